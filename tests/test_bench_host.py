"""Host-side measurement code of the benchmark, checked on the CPU against the oracle.

The path roofline reports how many exponentials the fused kernel evaluates: each 128-row
tile runs its readout over the union of its rows' admitted cells (eq. (8)), two cells per
64-key chunk, and its window over the band in 64-key chunks.  The count is recomputed here
independently: with K as large as W + P every admitted cell is selected, so the union of
the oracle's selections over a tile's rows is that tile's admitted union."""
import numpy as np

import bench
from workloads import generate, small
from tests._parity import oracle_for


def brute_executed_exps(wl, idx_all):
    q0 = wl.Nk - wl.Nq
    total = 0
    for b in range(wl.B):
        for h in range(wl.H):
            for r0 in range(0, wl.Nq, 128):
                nrows = min(128, wl.Nq - r0)
                sel = idx_all[b, h, r0:r0 + nrows]
                n_u = len(np.unique(sel[sel >= 0]))
                pb = q0 + r0
                lo, hi = max(0, pb - wl.w), pb + nrows - 1       # the tile's band of keys
                first = (pb - wl.w) + 64 * ((lo - (pb - wl.w)) // 64)
                n_w = (hi - first) // 64 + 1
                total += 128 * 64 * ((n_u + 1) // 2 + n_w)
    return total


def test_fused_executed_exps_matches_oracle_unions():
    for kw in (dict(Nq=1536, Nk=1536, K=6, W=4, P=9), dict(Nq=300, Nk=1700, K=6, W=3, P=5, w=96),
               dict(Nq=700, Nk=700, K=4, W=-1, P=-1)):
        inp = generate(small("exps", H=2, seed=71, **kw))
        wl = inp.wl
        k_all = wl.W + wl.P if wl.W >= 0 else wl.Nk // wl.s
        prob = oracle_for(inp, K=min(64, k_all))
        kbar, amax = prob.summaries()
        idx = prob.select_all(kbar, amax)
        assert bench.fused_executed_exps(wl, amax) == brute_executed_exps(wl, idx), kw

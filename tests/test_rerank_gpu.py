"""GPU parity of the eq. (12) token-level rerank (fs_select_topk_rerank) against the
float64 oracle's rerank_row, and of the forward pass run on the reranked cells.

Acceptance as for eq. (7): the selected cells equal the oracle's except where a
near-tie explains the difference (eq. (12) scores within 1e-4 relative of the K-th; with a
shortlist, eq. (7) scores within 1e-4 of the shortlist's boundary), and the output is
within the dtype's tolerance of the oracle's on the GPU's own cells."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from workloads import Inputs, generate, small
from tests._parity import TIE, TOL, DeviceRun, expected_output, oracle_for

pytestmark = pytest.mark.gpu


def check_rerank(prob, kbar, amax, gidx, rows, shortlist):
    exact = tie = 0
    for (b, h, r) in rows:
        Sg = [int(c) for c in gidx[b, h, r] if c >= 0]
        o_idx, cells, sc = prob.rerank_row(kbar, amax, b, h, r, shortlist)
        So = [int(c) for c in o_idx if c >= 0]
        assert Sg == sorted(Sg) and len(set(Sg)) == len(Sg), (b, h, r, Sg)
        if Sg == So:
            exact += 1
            continue
        assert len(Sg) == len(So), (b, h, r, Sg, So)
        score = dict(zip(cells.tolist(), sc.tolist()))
        _, acells, a7 = prob.select_row(kbar, amax, b, h, r)
        s7 = dict(zip(acells.tolist(), a7.tolist()))
        assert all(c in s7 for c in Sg), ("outside A_i", b, h, r)
        if shortlist and shortlist < len(acells):
            bound = sorted(a7.tolist(), reverse=True)[shortlist - 1]
            tol7 = TIE * max(abs(bound), 1e-6)
            assert all(c in score or s7[c] >= bound - tol7 for c in Sg), ("outside the shortlist", b, h, r)
        kth = min(score[c] for c in So)
        tol = TIE * max(abs(kth), 1e-6)
        kept = [score[c] for c in Sg if c in score]
        worst = min(kept) if kept else kth
        for c in set(score) - set(Sg):
            assert score[c] <= worst + tol, ("dropped a better cell", b, h, r, c)
        tie += 1
    return exact, tie


def run_rerank(inp, shortlist=0, rows=None, **over):
    wl = inp.wl
    g = DeviceRun(inp, **over)
    prob = oracle_for(inp, **over)
    kbar_o, amax_o = prob.summaries()
    g.summaries()
    fs.select_topk_rerank(g.p, g.Q, g.K, g.kbar, g.amax, g.idx, g.ws, shortlist)
    fs.sync_status(g.ws)
    idx = g.numpy(g.idx)
    if rows is None:
        rows = [(b, h, r) for b in range(wl.B) for h in range(wl.H) for r in range(wl.Nq)]
    exact, tie = check_rerank(prob, kbar_o, amax_o, idx, rows, shortlist)
    assert tie <= max(2, len(rows) // 100), (exact, tie)
    O = g.numpy(g.forward(idx=g.idx)).reshape(wl.B, wl.H, wl.Nq, wl.d)
    got = np.stack([O[b, h, r] for b, h, r in rows])
    err = np.abs(got - expected_output(inp, prob, rows, idx)).max()
    assert err <= TOL[wl.dtype], err
    return idx


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [
    dict(),                                        # pruned, all of A_i reranked
    dict(shortlist=8),                             # a shortlist of 8 of A_i's 13
    dict(lam=0.6, sigma=300.0),                    # erf prior on
    dict(Nq=300, Nk=1700),                         # appended queries (decode shape)
    dict(W=-1, P=-1, K=5, Nq=1200, Nk=1200),       # base FS: A_i = C_i (<= 21 cells)
])
def test_rerank_small(dtype, case):
    kw = dict(B=1, H=2, Nq=1536, Nk=1536, K=6, W=4, P=9, dtype=dtype, seed=401)
    kw.update(case)
    shortlist = kw.pop("shortlist", 0)
    lam = kw.pop("lam", None)
    sigma = kw.pop("sigma", 1024.0)
    run_rerank(generate(small("rerank", lam=lam, sigma=sigma, **kw)), shortlist)


def test_rerank_rescues_hidden_tokens():
    """Cells whose mean key is orthogonal to a query but which hold one token along it with
    logit 10 (and its negative, so the mean cancels) are selected by eq. (12)."""
    inp = generate(small("hidden", B=1, H=2, Nq=1024, Nk=1024, K=4, W=2, P=20, dtype="bf16", seed=402))
    K = inp.K.copy()
    planted = []
    for h in range(2):
        for r, c0 in ((1000, 7), (900, 11), (1023, 14)):      # (c0 + 1) s <= r - w
            q = inp.Q[0, h, r].astype(np.float64)
            qn = np.linalg.norm(q)
            s, d = inp.wl.s, inp.wl.d
            K[0, h, c0 * s:(c0 + 1) * s] *= 0.05
            K[0, h, c0 * s] = (10.0 * np.sqrt(d) / qn) * (q / qn)     # logit q.k/sqrt(d) = 10
            K[0, h, c0 * s + 1] = -K[0, h, c0 * s]
            planted.append((h, r, c0))
    from workloads import round_bf16
    inp = Inputs(wl=inp.wl, Q=inp.Q, K=round_bf16(K), V=inp.V, alpha=inp.alpha, lam=None, sigma=None)
    idx = run_rerank(inp)
    for h, r, c0 in planted:
        assert c0 in idx[0, h, r], (h, r, c0, idx[0, h, r])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [dict(), dict(Nq=300, Nk=1700), dict(lam=0.6, sigma=300.0, shortlist=10)])
def test_forward_rerank(dtype, case):
    """fs_forward_rerank: the same cells as fs_select_topk_rerank, and the output of the
    readout (fused tensor-core kernel in bf16) on them within tolerance of the oracle's."""
    kw = dict(B=1, H=2, Nq=1536, Nk=1536, K=6, W=4, P=9, dtype=dtype, seed=403)
    kw.update(case)
    shortlist = kw.pop("shortlist", 0)
    lam = kw.pop("lam", None)
    sigma = kw.pop("sigma", 1024.0)
    inp = generate(small("fwd_rerank", lam=lam, sigma=sigma, **kw))
    wl = inp.wl
    g = DeviceRun(inp)
    prob = oracle_for(inp)
    g.summaries()
    fs.select_topk_rerank(g.p, g.Q, g.K, g.kbar, g.amax, g.idx, g.ws, shortlist)
    ref_idx = g.numpy(g.idx).copy()
    idx2 = torch.full_like(g.idx, -7)
    g.O.fill_(float("nan"))
    fs.forward_rerank(g.p, g.Q, g.K, g.V, g.O, g.ws, idx=idx2, shortlist=shortlist)
    fs.sync_status(g.ws)
    idx2 = g.numpy(idx2)
    assert np.array_equal(idx2, ref_idx)
    rows = [(b, h, r) for b in range(wl.B) for h in range(wl.H) for r in range(wl.Nq)]
    O = g.numpy(g.O).reshape(wl.B, wl.H, wl.Nq, wl.d)
    got = np.stack([O[b, h, r] for b, h, r in rows])
    err = np.abs(got - expected_output(inp, prob, rows, idx2)).max()
    assert err <= TOL[wl.dtype], err


def test_forward_rerank_full_size_sampled():
    """The 64k prefill workload through fs_forward_rerank, judged on sampled rows."""
    from workloads import CONFIGS
    from tests._parity import sample_rows
    inp = generate(CONFIGS["prefill64k"])
    wl = inp.wl
    g = DeviceRun(inp)
    prob = oracle_for(inp)
    idx = torch.empty((wl.B, wl.H, wl.Nq, wl.K), dtype=torch.int32, device="cuda")
    fs.forward_rerank(g.p, g.Q, g.K, g.V, g.O, g.ws, idx=idx)
    fs.sync_status(g.ws)
    idx = g.numpy(idx)
    rows = sample_rows(wl, 48, seed=7)
    kbar_o, amax_o = prob.summaries()
    exact, tie = check_rerank(prob, kbar_o, amax_o, idx, rows, 0)
    assert tie <= max(2, len(rows) // 20), (exact, tie)
    O = g.numpy(g.O).reshape(wl.B, wl.H, wl.Nq, wl.d)
    got = np.stack([O[b, h, r] for b, h, r in rows])
    err = np.abs(got - expected_output(inp, prob, rows, idx)).max()
    assert err <= TOL[wl.dtype], err

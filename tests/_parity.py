"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and
judge its results against the oracle with the stated acceptance rules.

Acceptance (from the method's own tolerance statement, "1e-4 relative"):
  * selected cells equal the oracle's, except where the difference is explained by a
    near-tie: a score within 1e-4 * max(|x_K|, s_i, 1e-6) of the K-th best score, where
    s_i is the largest |r_ic| over the row's admitted cells (the scale of the row's
    scores: a K-th score near zero is the difference of products of that size, which
    fp32 arithmetic resolves only to a fraction of s_i), or a norm a_c within
    1e-4 * max(|a_P|, 1e-6) of the P-th largest (pruning boundary);
  * outputs within max-abs 2e-2 for bf16 inputs (fp32 accumulation) and 1e-4 in fp32,
    the long-range part judged on the GPU's own selected cells (oracle readout on them).
"""
import numpy as np
import torch

import long_context_sparse_head_b200 as fs
import oracle

TOL = {"bf16": 2e-2, "f32": 1e-4}
TIE = 1e-4


def tdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def params_for(inp, **over):
    wl = inp.wl
    kw = dict(B=wl.B, H=wl.H, Nq=wl.Nq, Nk=wl.Nk, d=wl.d, w=wl.w, s=wl.s, K=wl.K, W=wl.W,
              P=wl.P, alpha=inp.alpha, lam=inp.lam, sigma=inp.sigma, rope_base=wl.rope_base,
              rms_eps=wl.rms_eps, dtype=wl.dtype)
    kw.update(over)
    return fs.Params(**kw)


def oracle_for(inp, **over):
    wl = inp.wl
    kw = dict(w=wl.w, s=wl.s, K_cells=wl.K, W=wl.W, P=wl.P, alpha=inp.alpha, lam=inp.lam,
              sigma=inp.sigma, rope_base=wl.rope_base, rms_eps=wl.rms_eps)
    for k_in, k_out in (("K", "K_cells"),):
        if k_in in over:
            over[k_out] = over.pop(k_in)
    kw.update(over)
    return oracle.Problem(inp.Q, inp.K, inp.V, **kw)


class DeviceRun:
    """Device copies of the inputs and the C-ABI calls on them."""

    def __init__(self, inp, **over):
        self.inp = inp
        self.p = params_for(inp, **over)
        dt = tdtype(inp.wl)
        dev = "cuda"
        self.Q = torch.from_numpy(inp.Q).to(dev).to(dt).contiguous()
        self.K = torch.from_numpy(inp.K).to(dev).to(dt).contiguous()
        self.V = torch.from_numpy(inp.V).to(dev).to(dt).contiguous()
        self.ws = fs.alloc_workspace(self.p)
        p = self.p
        self.kbar = torch.empty((p.B, p.H, p.C, p.d), dtype=torch.float32, device=dev)
        self.amax = torch.empty((p.B, p.H, p.C), dtype=torch.float32, device=dev)
        self.idx = torch.empty((p.B, p.H, p.Nq, p.K), dtype=torch.int32, device=dev)
        self.O = torch.empty_like(self.Q)

    def summaries(self):
        fs.cell_summaries(self.p, self.K, self.kbar, self.amax)
        return self.kbar, self.amax

    def select(self):
        self.summaries()
        fs.select_topk(self.p, self.Q, self.kbar, self.amax, self.idx, self.ws)
        return self.idx

    def forward(self, kbar=None, amax=None, idx=None):
        self.O.fill_(float("nan"))
        fs.forward(self.p, self.Q, self.K, self.V, self.O, self.ws, kbar=kbar, amax=amax, idx=idx)
        fs.sync_status(self.ws)
        return self.O

    def numpy(self, t):
        torch.cuda.synchronize()
        return t.float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def flat_rows(wl, rows_bhr):
    """(b, h, r) triples -> flat row indices (b*H + h)*Nq + r."""
    return np.array([(b * wl.H + h) * wl.Nq + r for b, h, r in rows_bhr], np.int64)


def sample_rows(wl, n, seed, extra=()):
    rng = np.random.default_rng(seed)
    b = rng.integers(0, wl.B, n)
    h = rng.integers(0, wl.H, n)
    r = rng.integers(0, wl.Nq, n)
    rows = set(zip(b.tolist(), h.tolist(), r.tolist())) | set(extra)
    # always include the first and last rows of a head (window edge, longest prefix)
    rows |= {(0, 0, 0), (wl.B - 1, wl.H - 1, wl.Nq - 1)}
    return sorted(rows)


def check_selection(inp, orc_sum, gpu_idx, rows_bhr, **over):
    """Judge GPU-selected cells against the oracle with the near-tie rule.

    Returns (#rows exact, #rows differing within the tie rule); raises on a violation."""
    wl = inp.wl
    K = over.get("K", wl.K)
    W = over.get("W", wl.W)
    P = over.get("P", wl.P)
    prune = not (W < 0 and P < 0)
    prob = oracle_for(inp, **over)
    allc = oracle_for(inp, **dict(over, W=-1, P=-1, K=1))       # scores over all of C_i
    kbar, amax = orc_sum
    exact = tie = 0
    for (b, h, r) in rows_bhr:
        g = gpu_idx[b, h, r]
        Sg = [int(c) for c in g if c >= 0]
        o_idx, _, a_scores = prob.select_row(kbar, amax, b, h, r)
        So = [int(c) for c in o_idx if c >= 0]
        assert Sg == sorted(Sg) and len(set(Sg)) == len(Sg), (b, h, r, Sg)
        assert all(c == -1 for c in g[len(Sg):]), (b, h, r, g)
        if Sg == So:
            exact += 1
            continue
        _, ccells, cscores = allc.select_row(kbar, amax, b, h, r)
        score = dict(zip(ccells.tolist(), cscores.tolist()))
        n = len(ccells)
        assert len(Sg) == len(So), (b, h, r, Sg, So)
        assert all(c in score for c in Sg), ("not a candidate", b, h, r, Sg)
        a = amax[b, h, :n]
        if prune and n > P:
            # hi: every cell a near-tie could admit (norm within tol of the P-th largest);
            # lo: the cells admitted under any near-tie (norm above the (P+1)-th largest by
            # more than tol), so the P-th cell itself counts unless another one ties with it
            desc = np.sort(a)[::-1]
            aP = desc[P - 1] if P > 0 else np.inf
            aP1 = desc[P]
            tolP = TIE * max(abs(aP), 1e-6) if P > 0 else 0.0
            tolP1 = TIE * max(abs(aP1), 1e-6)
            recent = set(range(max(0, n - W), n))
            lo = recent | {c for c in range(n) if a[c] > aP1 + tolP1}
            hi = recent | {c for c in range(n) if a[c] >= aP - tolP}
        else:
            lo = hi = set(range(n))
        assert set(Sg) <= hi, ("outside A_i", b, h, r)
        kth = sorted((score[c] for c in So), reverse=True)[-1]
        scale = float(np.abs(a_scores).max()) if len(a_scores) else 0.0
        tolK = TIE * max(abs(kth), scale, 1e-6)
        worst_kept = min(score[c] for c in Sg)
        for c in lo - set(Sg):
            assert score[c] <= worst_kept + tolK, ("dropped a better cell", b, h, r, c)
        tie += 1
    return exact, tie


def expected_output(inp, prob, rows_bhr, gpu_idx):
    """Oracle o^sr plus alpha_h * oracle readout on the GPU's own cells, for the rows."""
    wl = inp.wl
    flat = flat_rows(wl, rows_bhr)
    _, _, _, osr = prob.forward(rows=flat, want_idx=True, want_parts=True)
    sel = np.stack([gpu_idx[b, h, r] for b, h, r in rows_bhr]).astype(np.int32)
    _, olr = prob.readout_rows(flat, sel)
    alpha = np.array([inp.alpha[h] for _, h, _ in rows_bhr])[:, None]
    return osr + alpha * olr

"""Pins for the float64 oracle (CPU only).

The oracle is checked against things other than itself: a brute-force dense-mask
restatement on tiny inputs, library attention (torch SDPA in float64) in the special
cases where the method reduces to it, closed forms, invariants stated on the
"FreeSolo" summary page, and hand-worked fixtures under tests/golden/.  A final test
plants known mistakes in the oracle and checks that some pin catches each one.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import Workload, generate, small
from tests._brute import brute_forward, rope_complex, sel_to_idx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def make_problem(inp, mutation=0, **over):
    wl = inp.wl
    kw = dict(w=wl.w, s=wl.s, K_cells=wl.K, W=wl.W, P=wl.P, alpha=inp.alpha,
              lam=inp.lam, sigma=inp.sigma, rope_base=wl.rope_base, rms_eps=wl.rms_eps)
    kw.update(over)
    return oracle.Problem(inp.Q, inp.K, inp.V, mutation=mutation, **kw)


def tiny(**kw):
    base = dict(B=1, H=2, Nq=192, Nk=192, d=8, w=32, s=8, K=3, W=2, P=3, seed=5)
    base.update(kw)
    return generate(small("tiny", **base))


TINY_CASES = {
    "prune": dict(),
    "noprune": dict(W=-1, P=-1),
    "prior": dict(lam=0.5, sigma=24.0),
    "decode": dict(Nq=40, Nk=200),
    "bigK": dict(K=40, W=-1, P=-1),
    "needles": dict(needles=2, needle_queries=6, Nq=256, Nk=256),
    "rag": dict(Nq=150, Nk=203),
}


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("case", sorted(TINY_CASES))
def test_oracle_matches_bruteforce(case):
    inp = tiny(**TINY_CASES[case])
    wl = inp.wl
    prob = make_problem(inp)
    O, idx = prob.forward(want_idx=True)
    Ob, sel, _, _, _ = brute_forward(inp.Q, inp.K, inp.V, w=wl.w, s=wl.s, K_cells=wl.K,
                                     W=wl.W, P=wl.P, alpha=inp.alpha, lam=inp.lam,
                                     sigma=inp.sigma, rope_base=wl.rope_base,
                                     rms_eps=wl.rms_eps)
    np.testing.assert_array_equal(idx, sel_to_idx(sel, wl.K))
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)


def test_oracle_matches_bruteforce_with_exact_ties():
    """Duplicated cells give exact ties in a_c and in the scores (tie rule G9)."""
    inp = tiny(H=1, Nq=160, Nk=160, seed=9)
    K = inp.K.copy()
    s = inp.wl.s
    for c in (1, 4, 7, 10):                     # four identical cells
        K[0, 0, c * s:(c + 1) * s] = K[0, 0, 0:s]
    inp.K = K
    wl = inp.wl
    for W_, P_ in ((2, 3), (0, 2), (-1, -1)):
        prob = make_problem(inp, W=W_, P=P_)
        O, idx = prob.forward(want_idx=True)
        Ob, sel, _, _, _ = brute_forward(inp.Q, inp.K, inp.V, w=wl.w, s=s, K_cells=wl.K,
                                         W=W_, P=P_, alpha=inp.alpha)
        np.testing.assert_array_equal(idx, sel_to_idx(sel, wl.K))
        np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- eq. (3) identity
def test_rope_relative_identity():
    """(R(i)q)^T (R(j)k) = q^T R(j-i) k, and R preserves norms (eq. (3))."""
    inp = tiny(d=64, seed=3)
    prob = make_problem(inp)
    rng = np.random.default_rng(0)
    for _ in range(20):
        q = rng.standard_normal(64).astype(np.float32)
        k = rng.standard_normal(64).astype(np.float32)
        i, j = (int(v) for v in rng.integers(0, 300000, 2))
        lhs = prob.rope(q, i) @ prob.rope(k, j)
        rhs = q.astype(np.float64) @ prob.rope(k, j - i)
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(lhs))
        assert abs(np.linalg.norm(prob.rope(q, i)) - np.linalg.norm(q.astype(np.float64))) < 1e-12


def test_rope_against_complex_rotation():
    inp = tiny(d=64, seed=4)
    prob = make_problem(inp)
    x = np.random.default_rng(1).standard_normal(64).astype(np.float32)
    for pos in (0, 1, 17, 4096, 262271):
        ref = rope_complex(x[None, :].astype(np.float64), np.array([pos]), 64, 10000.0)[0]
        # theta_m rounding (1e-16 relative) times pos ~ 2.6e5 bounds the difference
        np.testing.assert_allclose(prob.rope(x, pos), ref, rtol=0, atol=1e-9)


# ---------------------------------------------------------------- library reductions
def _sdpa(q, k, v, mask):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v),
                                                           attn_mask=t(mask).bool())
    return out[0, 0].numpy()


def test_full_window_is_causal_rope_attention():
    """w >= N and alpha = 0: the output is full causal RoPE attention."""
    inp = generate(small("full", Nq=256, Nk=256, d=64, w=10_000, s=32, K=4, seed=21))
    prob = make_problem(inp, alpha=np.zeros(2))
    O = prob.forward()
    N = 256
    mask = np.tril(np.ones((N, N), bool))
    for h in range(2):
        pos = np.arange(N)
        qr = rope_complex(inp.Q[0, h].astype(np.float64), pos, 64, 10000.0)
        kr = rope_complex(inp.K[0, h].astype(np.float64), pos, 64, 10000.0)
        ref = _sdpa(qr, kr, inp.V[0, h], mask)
        np.testing.assert_allclose(O[0, h], ref, rtol=0, atol=1e-12)


def test_alpha_zero_is_sliding_window_attention():
    inp = generate(small("sw", Nq=300, Nk=300, d=64, w=64, s=16, K=4, seed=22))
    prob = make_problem(inp, alpha=np.zeros(2))
    O = prob.forward()
    i = np.arange(300)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] >= i[:, None] - 64)
    for h in range(2):
        qr = rope_complex(inp.Q[0, h].astype(np.float64), i, 64, 10000.0)
        kr = rope_complex(inp.K[0, h].astype(np.float64), i, 64, 10000.0)
        np.testing.assert_allclose(O[0, h], _sdpa(qr, kr, inp.V[0, h], mask), rtol=0, atol=1e-12)


def test_long_range_with_all_cells_is_dense_nope_attention():
    """No pruning, K >= |C_i|, lambda = 0: u_i is dense NoPE attention over the prefix."""
    inp = generate(small("dense", Nq=400, Nk=400, d=64, w=64, s=16, K=64, W=-1, P=-1,
                         seed=23))
    prob = make_problem(inp)
    _, _, olr, _ = prob.forward(want_idx=True, want_parts=True)
    N, s, w = 400, 16, 64
    i = np.arange(N)
    n = np.where(i - w >= s, (i - w) // s, 0)
    mask = np.arange(N)[None, :] < (n * s)[:, None]
    has = n > 0
    for h in range(2):
        q = inp.Q[0, h].astype(np.float64)
        k = inp.K[0, h].astype(np.float64)
        # SDPA rows with an empty mask are undefined; give them one dummy key
        m2 = mask.copy()
        m2[~has, 0] = True
        u = _sdpa(q, k, inp.V[0, h], m2)
        ms = (u ** 2).mean(axis=1, keepdims=True)
        ref = np.where(has[:, None], u / np.sqrt(ms + 1e-6), 0.0)
        np.testing.assert_allclose(olr[0, h], ref, rtol=0, atol=1e-11)


# ---------------------------------------------------------------- closed forms
def test_softmax_rows_sum_to_one():
    """V = 1: o^sr = 1 and o^lr = 1/sqrt(1+eps) wherever a cell is selected (eqs. (4), (9))."""
    inp = tiny(d=16, Nq=200, Nk=200, seed=8)
    inp.V = np.ones_like(inp.V)
    prob = make_problem(inp)
    O, idx, olr, osr = prob.forward(want_idx=True, want_parts=True)
    np.testing.assert_allclose(osr, 1.0, rtol=0, atol=1e-13)
    has = (idx >= 0).any(axis=-1)
    assert has.any() and (~has).any()
    np.testing.assert_allclose(olr[has], 1.0 / math.sqrt(1.0 + 1e-6), rtol=0, atol=1e-13)
    np.testing.assert_array_equal(olr[~has], 0.0)
    a = inp.alpha[None, :, None, None]
    np.testing.assert_allclose(O, osr + a * olr, rtol=0, atol=1e-13)


def test_rmsnorm_closed_form():
    """mean(o_lr^2) = mean(u^2) / (mean(u^2) + eps) for the oracle's own u (eq. (9))."""
    inp = tiny(d=64, Nq=256, Nk=256, seed=12)
    prob = make_problem(inp, rms_eps=1e-4)
    _, idx = prob.forward(want_idx=True)
    rows = np.arange(inp.wl.B * inp.wl.H * inp.wl.Nq)
    u, olr = prob.readout_rows(rows, idx.reshape(-1, inp.wl.K))
    has = (idx.reshape(-1, inp.wl.K) >= 0).any(axis=1)
    mu = (u[has] ** 2).mean(axis=1)
    np.testing.assert_allclose((olr[has] ** 2).mean(axis=1), mu / (mu + 1e-4), rtol=1e-12)


def test_summaries_closed_form():
    """eq. (5): a cell of identical keys has kbar = that key and a_c = its norm;
    a cell with one long key has a_c = that key's norm."""
    inp = tiny(H=1, Nq=64, Nk=64, d=8, s=8, seed=2)
    K = inp.K.copy()
    K[0, 0, 0:8] = K[0, 0, 3]
    K[0, 0, 8:16] *= 0.01
    K[0, 0, 13] = np.float32([3, 4, 0, 0, 0, 0, 0, 0])
    inp.K = K
    kbar, amax = make_problem(inp).summaries()
    np.testing.assert_allclose(kbar[0, 0, 0], K[0, 0, 3], rtol=1e-7)
    assert abs(amax[0, 0, 0] - np.linalg.norm(K[0, 0, 3].astype(np.float64))) < 1e-12
    assert abs(amax[0, 0, 1] - 5.0) < 1e-12
    np.testing.assert_allclose(kbar[0, 0, 2], K[0, 0, 16:24].astype(np.float64).mean(0), rtol=1e-12)


def test_candidate_count_closed_form():
    """C_i = {c : (c+1)s <= i - w}: empty before i = w + s, then one cell per s tokens."""
    prob = make_problem(tiny(w=512, s=32, Nq=2048, Nk=2048, d=8))
    assert prob.candidate_count(0) == 0
    assert prob.candidate_count(512 + 31) == 0
    assert prob.candidate_count(512 + 32) == 1
    assert prob.candidate_count(512 + 63) == 1
    assert prob.candidate_count(512 + 64) == 2
    assert prob.candidate_count(2047) == (2047 - 512) // 32


def test_admitted_set_invariants():
    """|A_i| <= W + P, Recent_W is inside A_i, A_i is inside C_i (eq. (8))."""
    inp = tiny(Nq=512, Nk=512, seed=14)
    prob = make_problem(inp, W=3, P=5)
    _, amax = prob.summaries()
    for n in range(0, prob.C + 1):
        A = prob.admitted(amax[0, 0], n)
        assert len(A) <= 8 and len(A) == len(set(A.tolist()))
        assert all(0 <= c < n for c in A)
        assert set(range(max(0, n - 3), n)) <= set(A.tolist())
        if n <= 5:                               # TopP alone already covers C_i
            assert len(A) == n


def test_shift_invariance():
    """Shifting tokens, cells and queries together by a multiple of s leaves o unchanged
    ("Position Independence": RoPE is relative, the erf prior depends on i - p_c)."""
    inp = tiny(d=64, Nq=64, Nk=256, w=48, s=8, K=4, lam=0.7, sigma=20.0, seed=15)
    base = make_problem(inp).forward()
    for pos0 in (8, 800, 123456):
        shifted = make_problem(inp, pos0=pos0).forward()
        np.testing.assert_allclose(shifted, base, rtol=0, atol=1e-11)


def test_needles_are_selected():
    """Planted high-norm cells aligned with a query are selected by that query."""
    inp = generate(small("needle", B=1, H=2, Nq=2048, Nk=2048, d=64, w=512, s=32, K=4,
                         W=4, P=8, needles=3, needle_queries=5, seed=31))
    _, idx = make_problem(inp).forward(want_idx=True)
    assert len(inp.needle_cells) == 6
    for b, h, c, rows in inp.needle_cells:
        for r in rows:
            assert c in idx[b, h, r], (b, h, c, r)


# ---------------------------------------------------------------- golden fixtures
def _read_fixture(name):
    hdr, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            if ":" in line:
                k, v = line.split(":")
                rows.append((int(k), [int(t) for t in v.split()]))
            else:
                toks = line.split()
                hdr[toks[0]] = [float(t) for t in toks[1:]]
    return hdr, rows


def test_golden_prune_eq8():
    hdr, rows = _read_fixture("prune_eq8.txt")
    a = np.array(hdr["a"], np.float64)
    inp = tiny(H=1, Nq=8, Nk=64, d=8, s=8)
    prob = make_problem(inp, W=int(hdr["W"][0]), P=int(hdr["P"][0]))
    for n, cells in rows:
        assert prob.admitted(a, n).tolist() == cells, n


def test_golden_select_ties_eq7():
    hdr, rows = _read_fixture("select_ties_eq7.txt")
    x = np.array(hdr["x"], np.float32)
    Q = np.zeros((1, 1, 1, 2), np.float32)
    Q[..., 0] = 1.0
    K = np.zeros((1, 1, 8, 2), np.float32)
    K[0, 0, :, 0] = x
    V = np.zeros_like(K)
    for Kc, cells in rows:
        prob = oracle.Problem(Q, K, V, w=0, s=1, K_cells=Kc, W=-1, P=-1, alpha=[1.0])
        kbar, amax = prob.summaries()
        idx, acells, scores = prob.select_row(kbar, amax, 0, 0, 0)
        assert acells.tolist() == list(range(7))
        np.testing.assert_allclose(scores, x[:7].astype(np.float64) / math.sqrt(2), rtol=1e-15)
        assert idx.tolist() == cells, Kc


# ---------------------------------------------------------------- eq. (12) rerank
def _constant_cells(inp):
    """The same problem with every cell's keys replaced by one vector (its mean)."""
    K = inp.K.copy()
    s = inp.wl.s
    C = K.shape[2] // s
    for c in range(C):
        K[:, :, c * s:(c + 1) * s] = K[:, :, c * s:(c + 1) * s].mean(axis=2, keepdims=True)
    return type(inp)(wl=inp.wl, Q=inp.Q, K=np.ascontiguousarray(K), V=inp.V, alpha=inp.alpha,
                     lam=None, sigma=None)


def _rerank_pin_failures(mutation=0):
    """Pins of the eq. (12) rerank; returns the names of those that fail."""
    fails = []
    # (a) constant cells: log-sum-exp over s equal logits is that logit + log s, so the
    #     rerank keeps exactly eq. (7)'s cells and its scores sit log s above eq. (7)'s
    inp = _constant_cells(tiny(d=16, Nq=200, Nk=200, seed=43))
    prob = make_problem(inp, mutation=mutation, lam=None, sigma=None)
    kb, am = prob.summaries()
    wl = inp.wl
    for r in range(0, wl.Nq, 7):
        i7, cells7, sc7 = prob.select_row(kb, am, 0, 1, r)
        i12, cells12, sc12 = prob.rerank_row(kb, am, 0, 1, r)
        if i7.tolist() != i12.tolist():
            fails.append("constant_cells_selection")
            break
        want = {c: v + math.log(wl.s) for c, v in zip(cells7.tolist(), sc7.tolist())}
        if any(abs(want[c] - v) > 1e-9 for c, v in zip(cells12.tolist(), sc12.tolist())):
            fails.append("constant_cells_offset")
            break
    # (b) bounds: max_j logit <= log-sum-exp <= max_j logit + log s, logits from numpy
    inp = tiny(d=16, Nq=200, Nk=200, seed=44)
    prob = make_problem(inp, mutation=mutation, lam=None, sigma=None)
    kb, am = prob.summaries()
    wl = inp.wl
    for r in range(wl.s + wl.w, wl.Nq, 11):
        _, cells, sc = prob.rerank_row(kb, am, 0, 0, r)
        q = inp.Q[0, 0, r].astype(np.float64)
        for c, v in zip(cells.tolist(), sc.tolist()):
            lg = inp.K[0, 0, c * wl.s:(c + 1) * wl.s].astype(np.float64) @ q / math.sqrt(wl.d)
            if not (lg.max() - 1e-9 <= v <= lg.max() + math.log(wl.s) + 1e-9):
                fails.append("lse_bounds")
                break
        if "lse_bounds" in fails:
            break
    # (c) a shortlist of exactly K keeps eq. (7)'s set (the rerank only reorders it)
    for r in range(wl.s + wl.w, wl.Nq, 13):
        if prob.select_row(kb, am, 0, 0, r)[0].tolist() != prob.rerank_row(kb, am, 0, 0, r, wl.K)[0].tolist():
            fails.append("shortlist_K")
            break
    # (d) rescue: a cell whose mean key is orthogonal to q but which holds one token along
    #     q (and its negative, so the mean cancels) is missed by eq. (7) and kept by eq. (12)
    inp = tiny(d=16, Nq=160, Nk=160, K=2, W=-1, P=-1, seed=45)
    K = inp.K.copy()
    q = inp.Q[0, 0, 159].astype(np.float64)
    u = q / np.linalg.norm(q)
    c0, s_ = 3, inp.wl.s
    K[0, 0, c0 * s_:(c0 + 1) * s_] = 0.0
    K[0, 0, c0 * s_] = 6.0 * u
    K[0, 0, c0 * s_ + 1] = -6.0 * u
    inp = type(inp)(wl=inp.wl, Q=inp.Q, K=np.ascontiguousarray(K, np.float32), V=inp.V,
                    alpha=inp.alpha, lam=None, sigma=None)
    prob = make_problem(inp, mutation=mutation, lam=None, sigma=None, W=-1, P=-1)
    kb, am = prob.summaries()
    if c0 in prob.select_row(kb, am, 0, 0, 159)[0].tolist() or \
            c0 not in prob.rerank_row(kb, am, 0, 0, 159)[0].tolist():
        fails.append("rescue")
    return fails


def test_rerank_pins():
    assert _rerank_pin_failures() == []


# ---------------------------------------------------------------- backward
def _fd_failures(mutation=0, n_entries=12):
    """Gradients of L = sum(dO * O) from the oracle's backward against central finite
    differences of its forward (selection held fixed: perturbations that change it are
    skipped).  Returns the names of the inputs whose check fails."""
    inp = tiny(d=8, Nq=96, Nk=96, w=16, s=8, K=3, W=2, P=3, lam=0.5, sigma=16.0, seed=47)
    wl = inp.wl

    def problem(Q, K, V, alpha):
        return oracle.Problem(Q, K, V, w=wl.w, s=wl.s, K_cells=wl.K, W=wl.W, P=wl.P, alpha=alpha,
                              lam=inp.lam, sigma=inp.sigma, rope_base=wl.rope_base,
                              rms_eps=wl.rms_eps, mutation=mutation)
    O, idx = problem(inp.Q, inp.K, inp.V, inp.alpha).forward(want_idx=True)
    dO = np.random.default_rng(48).standard_normal(O.shape)
    grads = problem(inp.Q, inp.K, inp.V, inp.alpha).backward(idx, dO)
    rng = np.random.default_rng(49)
    fails = []
    for name, arr_i, g in (("Q", 0, grads[0]), ("K", 1, grads[1]), ("V", 2, grads[2])):
        base = [inp.Q, inp.K, inp.V]
        for _ in range(n_entries):
            e = tuple(int(rng.integers(0, n)) for n in base[arr_i].shape)
            vals = []
            for sgn in (1, -1):
                arrs = [a.copy() for a in base]
                arrs[arr_i][e] = np.float32(arrs[arr_i][e] + sgn * 2.0 ** -10)
                O2, idx2 = problem(*arrs, inp.alpha).forward(want_idx=True)
                vals.append((float((dO * O2).sum()), float(arrs[arr_i][e]), np.array_equal(idx2, idx)))
            if not (vals[0][2] and vals[1][2]):
                continue
            fd = (vals[0][0] - vals[1][0]) / (vals[0][1] - vals[1][1])
            if abs(fd - g[e]) > 1e-4 * max(1.0, abs(g[e])):
                fails.append(name)
                break
    for h in range(wl.H):
        vals = []
        for sgn in (1, -1):
            al = np.array(inp.alpha, np.float64)
            al[h] += sgn * 1e-4
            O2, _ = problem(inp.Q, inp.K, inp.V, al).forward(want_idx=True)
            vals.append(float((dO * O2).sum()))
        if abs((vals[0] - vals[1]) / 2e-4 - grads[3][h]) > 1e-4 * max(1.0, abs(grads[3][h])):
            fails.append("alpha")
            break
    return fails


def test_backward_matches_finite_differences():
    assert _fd_failures(n_entries=20) == []


def test_backward_sampled_matches_full_backward():
    """The sampled backward (rows' dQ, keys' dK and dV, for full-size checks) equals the
    whole backward pass, itself pinned by finite differences, on every row and key; and
    the all-rows selection equals the forward pass's."""
    inp = tiny(d=16, Nq=150, Nk=260, w=32, s=8, K=3, W=2, P=3, lam=0.5, sigma=30.0, seed=71)
    prob = make_problem(inp)
    _, idx = prob.forward(want_idx=True)
    kb, am = prob.summaries()
    assert np.array_equal(prob.select_all(kb, am), idx)
    dO = np.random.default_rng(72).standard_normal((inp.wl.B, inp.wl.H, inp.wl.Nq, inp.wl.d))
    dQ, dK, dV, _ = prob.backward(idx, dO)
    rows = np.arange(inp.wl.B * inp.wl.H * inp.wl.Nq)
    keys = np.arange(inp.wl.B * inp.wl.H * inp.wl.Nk)
    sq, sk, sv = prob.backward_sampled(idx, dO, rows, keys)
    d = inp.wl.d
    assert np.abs(sq - dQ.reshape(-1, d)).max() <= 1e-12
    assert np.abs(sk - dK.reshape(-1, d)).max() <= 1e-12
    assert np.abs(sv - dV.reshape(-1, d)).max() <= 1e-12


# ---------------------------------------------------------------- FS-B (eqs. (10)-(11))
def _codes(kbar_bh):
    """16-bit code of each cell: the signs of its mean key's first 16 coordinates,
    coordinate 0 the most significant bit."""
    nb = min(16, kbar_bh.shape[1])
    bits = (kbar_bh[:, :nb] > 0).astype(np.int64)
    return (bits * (1 << np.arange(nb - 1, -1, -1))).sum(axis=1)


def _eq7(q, kbar_bh, amax_bh, i, c, s, lam, sigma):
    r = float(q.astype(np.float64) @ kbar_bh[c]) / math.sqrt(q.shape[0])
    if lam:
        r += lam * amax_bh[c] * math.erf((i - (c + 0.5) * s) / (2.0 * sigma))
    return r


def _tree_pin_failures(mutation=0):
    """Pins of the FS-B oracle; returns the names of those that fail."""
    fails = set()
    inp = tiny(d=16, Nq=160, Nk=400, w=32, s=8, K=4, W=-1, P=-1, lam=0.7, sigma=40.0, seed=61)
    wl = inp.wl
    prob = make_problem(inp, mutation=mutation)
    kb, am = prob.summaries()
    tau = np.array([np.median(am[0, 0]), np.quantile(am[0, 1], 0.7)])
    # (a) an exhaustive beam keeps every leaf: S_i is eq. (7)'s top-K over C_i (brute force)
    _, sel, _, _, _ = brute_forward(inp.Q, inp.K, inp.V, w=wl.w, s=wl.s, K_cells=wl.K, W=-1, P=-1,
                                    alpha=inp.alpha, lam=inp.lam, sigma=inp.sigma,
                                    rope_base=wl.rope_base, rms_eps=wl.rms_eps)
    want = sel_to_idx(sel, wl.K).reshape(-1, wl.K)
    for t in (None, tau):
        idx, _ = prob.tree_select(kb, am, beam=64, tau=t)
        if not np.array_equal(idx, want):
            fails.add("exhaustive")
    lam, sig = inp.lam[0], inp.sigma[0]
    for h in range(wl.H):
        kbh, amh = kb[0, h], am[0, h]
        code = _codes(kbh)
        for forest in (0, 1):
            seq = np.arange(kbh.shape[0]) if forest == 0 else np.nonzero(amh >= tau[h])[0]
            n = len(seq)
            _, _, nseq = prob.tree_node(kb, am, 0, h, forest, 0, 0, 1, 0, tau=tau)
            if nseq != n:
                fails.add("sequence")
            k = 0
            while (1 << k) <= n:
                for blk in range(n >> k):
                    cells = seq[blk << k:(blk + 1) << k]
                    order = cells[np.lexsort((np.arange(len(cells)), code[cells]))]
                    leaves, _, _ = prob.tree_node(kb, am, 0, h, forest, k, blk, 1, 0, tau=tau)
                    if leaves is None or leaves.tolist() != order.tolist():   # (b) radix order
                        fails.add("leaf_order")
                k += 1
            # (c) node statistics and eq. (11): closed forms per node, for a few rows
            for r in (wl.Nq - 1, wl.Nq // 2):
                i = wl.Nk - wl.Nq + r
                ncand = prob.candidate_count(i)
                q = inp.Q[0, h, r].astype(np.float64)
                for k in range(0, 5):
                    for blk in range(n >> k):
                        for v in range(1, 2 << k):
                            leaves, U1, _ = prob.tree_node(kb, am, 0, h, forest, k, blk, v, r, 1.0, tau)
                            _, U0, _ = prob.tree_node(kb, am, 0, h, forest, k, blk, v, r, 0.0, tau)
                            mu = kbh[leaves].mean(axis=0)
                            rho = np.sqrt(((kbh[leaves] - mu) ** 2).sum(axis=1)).max()
                            prior = lam * amh[leaves].max() * math.erf(
                                (i - (leaves.min() + 0.5) * wl.s) / (2.0 * sig))
                            if abs(U0 - (q @ mu / math.sqrt(wl.d) + prior)) > 1e-12:
                                fails.add("mu_prior")
                            if abs((U1 - U0) - np.linalg.norm(q) * rho / math.sqrt(wl.d)) > 1e-12:
                                fails.add("rho")
                            best = max(_eq7(q, kbh, amh, i, c, wl.s, lam, sig) for c in leaves)
                            # (d) U_v bounds its leaves (nodes of the row's prefix: there
                            #     the erf argument is positive)
                            if leaves.max() < ncand and U1 < best - 1e-12:
                                fails.add("bound")
                            if len(leaves) == 1 and abs(U1 - best) > 1e-12:
                                fails.add("leaf_is_eq7")
    # (e) a beam of width 1 descends greedily: one cell per forest, and on the path from
    #     its root every node beats its sibling
    idx, _ = prob.tree_select(kb, am, beam=1)
    for h in range(wl.H):
        for r in (wl.Nq - 1, 60, 100):
            row = (0 * wl.H + h) * wl.Nq + r
            got = [c for c in idx[row] if c >= 0]
            n = prob.candidate_count(wl.Nk - wl.Nq + r)
            if n == 0:
                continue
            if len(got) != 1:
                fails.add("greedy")
                continue
            c = got[0]
            k = max(kk for kk in range(12) if (n >> kk) & 1 and ((n >> kk) - 1) << kk <= c)
            blk = (n >> k) - 1
            roots = [(kk, (n >> kk) - 1) for kk in range(12) if (n >> kk) & 1]
            Uroot = {rt: prob.tree_node(kb, am, 0, h, 0, rt[0], rt[1], 1, r)[1] for rt in roots}
            if max(Uroot.values()) != Uroot[(k, blk)]:
                fails.add("greedy")
            v = 1
            while v < (1 << k):
                kids = [prob.tree_node(kb, am, 0, h, 0, k, blk, 2 * v + e, r) for e in (0, 1)]
                e = 0 if c in kids[0][0] else 1
                if kids[e][1] < kids[1 - e][1]:
                    fails.add("greedy")
                v = 2 * v + e
    return sorted(fails)


def test_tree_pins():
    assert _tree_pin_failures() == []


# ---------------------------------------------------------------- sensitivity
def _pins_fail(mutation):
    """Run a compact set of the pins above against a mutated oracle; True if any fails."""
    failures = []
    inp = tiny(d=16, Nq=200, Nk=200, lam=0.8, sigma=16.0, seed=41)
    wl = inp.wl
    for W_, P_ in ((2, 3), (-1, -1)):
        prob = make_problem(inp, mutation=mutation, W=W_, P=P_)
        O, idx = prob.forward(want_idx=True)
        Ob, sel, _, _, _ = brute_forward(inp.Q, inp.K, inp.V, w=wl.w, s=wl.s, K_cells=wl.K,
                                         W=W_, P=P_, alpha=inp.alpha, lam=inp.lam,
                                         sigma=inp.sigma)
        if not np.array_equal(idx, sel_to_idx(sel, wl.K)) or np.abs(O - Ob).max() > 1e-12:
            failures.append("brute")
    try:
        hdr, rows = _read_fixture("prune_eq8.txt")
        p2 = make_problem(tiny(H=1, Nq=8, Nk=64, d=8, s=8), mutation=mutation, W=2, P=3)
        if any(p2.admitted(np.array(hdr["a"]), n).tolist() != c for n, c in rows):
            failures.append("golden_prune")
    except Exception:
        failures.append("golden_prune")
    failures += _rerank_pin_failures(mutation)
    failures += _fd_failures(mutation, n_entries=6)
    failures += _tree_pin_failures(mutation)
    return failures


@pytest.mark.parametrize("mutation", sorted(oracle.MUTATIONS))
def test_planted_mistakes_are_caught(mutation):
    assert _pins_fail(mutation), "mutation %s passed every pin" % mutation


def test_unmutated_oracle_passes_the_sensitivity_pins():
    assert _pins_fail(0) == []

"""FreeSolo float64 CPU oracle: ctypes wrapper around oracle/freesolo_oracle.c.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this package; the CUDA library and its Python binding never do.

It follows the "FreeSolo" technical summary, §3.1 eq. (2),
§3.2 eqs. (3)-(4), §3.3 eqs. (5), (7)-(9) and §3.4 eqs. (10)-(12); the readings taken where the page is
silent are stated at the top of the C source.  Inputs are float32 arrays holding
the exact input values (bf16 inputs widened); all arithmetic is float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


class OrcParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("Nq", ctypes.c_int), ("Nk", ctypes.c_int),
        ("d", ctypes.c_int), ("w", ctypes.c_int), ("s", ctypes.c_int), ("K", ctypes.c_int),
        ("W", ctypes.c_int), ("P", ctypes.c_int),
        ("rope_base", ctypes.c_double), ("rms_eps", ctypes.c_double),
        ("pos0", ctypes.c_longlong),
        ("alpha", ctypes.POINTER(ctypes.c_double)),
        ("lambda_", ctypes.POINTER(ctypes.c_double)),
        ("sigma", ctypes.POINTER(ctypes.c_double)),
        ("mutation", ctypes.c_int),
    ]


# planted mistakes, for the pin-sensitivity tests only
MUTATIONS = {
    "rope_key_sign": 1, "drop_prior": 2, "window_short": 3, "cand_loose": 4,
    "amax_mean": 5, "no_eps": 6, "alpha_on_sr": 7, "rope_in_readout": 8,
    "scale_d": 9, "tie_high_index": 10, "rerank_mean": 11, "rerank_rope": 12,
    "bwd_no_rms": 13, "tree_no_rho": 14, "tree_pmax": 15, "tree_sort_desc": 16,
}


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(OrcParams)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        L.orc_num_cells.argtypes = [P]
        L.orc_candidate_count.argtypes = [P, ctypes.c_longlong]
        L.orc_cell_summaries.argtypes = [P, f32p, f64p, f64p]
        L.orc_cell_summaries.restype = None
        L.orc_admitted.argtypes = [P, f64p, ctypes.c_int, i32p]
        L.orc_forward.argtypes = [P, f32p, f32p, f32p, ctypes.c_longlong, ctypes.c_void_p,
                                  f64p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_select_row.argtypes = [P, f32p, f64p, f64p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, i32p, i32p, f64p]
        L.orc_rerank_row.argtypes = [P, f32p, f32p, f64p, f64p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, i32p, i32p, f64p]
        L.orc_backward.argtypes = [P, f32p, f32p, f32p, i32p, f64p, f64p, f64p, f64p, f64p]
        L.orc_readout_rows.argtypes = [P, f32p, f32p, f32p, ctypes.c_longlong, i64p, i32p,
                                       ctypes.c_void_p, f64p]
        L.orc_readout_rows.restype = None
        L.orc_tree_select_rows.argtypes = [P, f32p, f64p, f64p, ctypes.c_void_p, ctypes.c_int,
                                           ctypes.c_double, ctypes.c_longlong, ctypes.c_void_p,
                                           i32p, f64p]
        L.orc_tree_node.argtypes = [P, f32p, f64p, f64p, ctypes.c_void_p] + [ctypes.c_int] * 7 + [
            ctypes.c_double, i32p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]
        L.orc_backward_sampled.argtypes = [P, f32p, f32p, f32p, i32p, f64p, ctypes.c_longlong, i64p, f64p,
                                           ctypes.c_longlong, i64p, f64p, f64p]
        L.orc_select_all.argtypes = [P, f32p, f64p, f64p, i32p]
        L.orc_rope.argtypes = [P, f32p, ctypes.c_longlong, f64p]
        L.orc_rope.restype = None
        _lib = L
    return _lib


class Problem:
    """One oracle problem: shapes, parameters and float32 input arrays.

    Q [B,H,Nq,d], K/V [B,H,Nk,d]; query row r sits at key-index position Nk-Nq+r.
    W = P = -1 means no pruning (base FS).  lam/sigma may be None (prior off).
    """

    def __init__(self, Q, K, V, *, w, s, K_cells, W, P, alpha, lam=None, sigma=None,
                 rope_base=10000.0, rms_eps=1e-6, pos0=0, mutation=0):
        self.Q = np.ascontiguousarray(Q, dtype=np.float32)
        self.K = np.ascontiguousarray(K, dtype=np.float32)
        self.V = np.ascontiguousarray(V, dtype=np.float32)
        self.B, self.H, self.Nq, self.d = self.Q.shape
        self.Nk = self.K.shape[2]
        self.alpha = np.ascontiguousarray(alpha, dtype=np.float64)
        self.lam = None if lam is None else np.ascontiguousarray(lam, dtype=np.float64)
        self.sigma = None if sigma is None else np.ascontiguousarray(sigma, dtype=np.float64)
        self.p = OrcParams()
        p = self.p
        p.B, p.H, p.Nq, p.Nk, p.d = self.B, self.H, self.Nq, self.Nk, self.d
        p.w, p.s, p.K, p.W, p.P = w, s, K_cells, W, P
        p.rope_base, p.rms_eps, p.pos0 = rope_base, rms_eps, pos0
        dp = ctypes.POINTER(ctypes.c_double)
        p.alpha = self.alpha.ctypes.data_as(dp)
        p.lambda_ = self.lam.ctypes.data_as(dp) if self.lam is not None else dp()
        p.sigma = self.sigma.ctypes.data_as(dp) if self.sigma is not None else dp()
        p.mutation = MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)

    @property
    def C(self):
        return lib().orc_num_cells(ctypes.byref(self.p))

    def candidate_count(self, i):
        return lib().orc_candidate_count(ctypes.byref(self.p), int(i))

    def summaries(self):
        """eq. (5): kbar [B,H,C,d], amax [B,H,C] (float64)."""
        C = self.C
        kbar = np.zeros((self.B, self.H, max(C, 1), self.d), np.float64)[:, :, :C]
        kbar = np.ascontiguousarray(kbar)
        amax = np.zeros((self.B, self.H, C), np.float64)
        if C > 0:
            lib().orc_cell_summaries(ctypes.byref(self.p), self.K, kbar, amax)
        return kbar, amax

    def admitted(self, amax_bh, n):
        """eq. (8): admitted cells for a candidate prefix of n cells, ascending."""
        out = np.zeros(max(n, 1), np.int32)
        a = np.ascontiguousarray(amax_bh, dtype=np.float64)
        cnt = lib().orc_admitted(ctypes.byref(self.p), a, int(n), out)
        return out[:cnt].copy()

    def forward(self, rows=None, want_idx=False, want_parts=False):
        """eq. (2) for the given flat rows ((b*H+h)*Nq + r), or all rows.

        Returns O [n,d] (or [B,H,Nq,d] when rows is None), plus idx/olr/osr on request.
        """
        if rows is None:
            n = self.B * self.H * self.Nq
            rows_arr = None
        else:
            rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
            n = rows_arr.shape[0]
        O = np.zeros((n, self.d), np.float64)
        idx = np.zeros((n, max(self.p.K, 1)), np.int32) if want_idx else None
        olr = np.zeros((n, self.d), np.float64) if want_parts else None
        osr = np.zeros((n, self.d), np.float64) if want_parts else None
        vp = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
        rc = lib().orc_forward(ctypes.byref(self.p), self.Q, self.K, self.V, n,
                               vp(rows_arr), O, vp(idx), vp(olr), vp(osr))
        if rc != 0:
            raise ValueError("oracle rejected the problem (rc=%d)" % rc)
        shape = (self.B, self.H, self.Nq) if rows is None else (n,)
        out = [O.reshape(shape + (self.d,))]
        if want_idx:
            out.append(idx[:, :self.p.K].reshape(shape + (self.p.K,)))
        if want_parts:
            out += [olr.reshape(shape + (self.d,)), osr.reshape(shape + (self.d,))]
        return out[0] if len(out) == 1 else tuple(out)

    def select_row(self, kbar, amax, b, h, r):
        """eq. (7) + top-K for one row: (idx[K], A_i cells, scores r_ic over A_i)."""
        C = self.C
        idx = np.zeros(max(self.p.K, 1), np.int32)
        acells = np.zeros(max(C, 1), np.int32)
        ascores = np.zeros(max(C, 1), np.float64)
        nA = lib().orc_select_row(ctypes.byref(self.p), self.Q,
                                  np.ascontiguousarray(kbar, np.float64),
                                  np.ascontiguousarray(amax, np.float64),
                                  b, h, r, idx, acells, ascores)
        return idx[:self.p.K].copy(), acells[:nA].copy(), ascores[:nA].copy()

    def rerank_row(self, kbar, amax, b, h, r, shortlist=0):
        """eq. (12) token-level rerank for one row: the `shortlist` best cells of A_i by
        eq. (7) (0: all of A_i) rescored by the log-sum-exp of their tokens' logits plus
        the prior; returns (idx[K], shortlist cells ascending, their eq. (12) scores)."""
        C = self.C
        idx = np.zeros(max(self.p.K, 1), np.int32)
        cells = np.zeros(max(C, 1), np.int32)
        scores = np.zeros(max(C, 1), np.float64)
        ns = lib().orc_rerank_row(ctypes.byref(self.p), self.Q, self.K,
                                  np.ascontiguousarray(kbar, np.float64),
                                  np.ascontiguousarray(amax, np.float64),
                                  b, h, r, int(shortlist), idx, cells, scores)
        return idx[:self.p.K].copy(), cells[:ns].copy(), scores[:ns].copy()

    def backward(self, idx, dO):
        """Gradients of eq. (2) with the selection idx [B,H,Nq,K] held fixed, for the
        upstream gradient dO [B,H,Nq,d]: (dQ, dK, dV, dalpha) in float64."""
        B, H, Nq, Nk, d = self.p.B, self.p.H, self.p.Nq, self.p.Nk, self.d
        dQ = np.zeros((B, H, Nq, d)); dK = np.zeros((B, H, Nk, d)); dV = np.zeros((B, H, Nk, d))
        dal = np.zeros(H)
        lib().orc_backward(ctypes.byref(self.p), self.Q, self.K, self.V,
                           np.ascontiguousarray(idx, np.int32).reshape(-1),
                           np.ascontiguousarray(dO, np.float64).reshape(-1),
                           dQ.reshape(-1), dK.reshape(-1), dV.reshape(-1), dal)
        return dQ, dK, dV, dal

    def tree_select(self, kbar, amax, beam, c_explore=1.0, tau=None, rows=None):
        """FS-B selection (eqs. (10)-(11), readings in the C source) for flat rows (or all):
        (idx [n,K] ascending -1 padded, margin [n]: smallest relative gap at a beam cut)."""
        n = self.B * self.H * self.Nq if rows is None else len(rows)
        rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        tau_arr = None if tau is None else np.ascontiguousarray(tau, dtype=np.float64)
        idx = np.zeros((max(n, 1), max(self.p.K, 1)), np.int32)
        margin = np.ones(max(n, 1), np.float64)
        vp = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
        rc = lib().orc_tree_select_rows(ctypes.byref(self.p), self.Q,
                                        np.ascontiguousarray(kbar, np.float64).reshape(-1),
                                        np.ascontiguousarray(amax, np.float64).reshape(-1),
                                        vp(tau_arr), int(beam), float(c_explore), n, vp(rows_arr),
                                        idx.reshape(-1), margin)
        if rc != 0:
            raise ValueError("oracle rejected the FS-B problem")
        return idx[:n, :self.p.K], margin[:n]

    def tree_node(self, kbar, amax, b, h, forest, k, blk, v, r, c_explore=1.0, tau=None):
        """One FS-B tree node: (leaf cells in code order, U_v of eq. (11) for row r,
        forest sequence length), or (None, None, n) if the node does not exist."""
        leaves = np.zeros(1 << max(k, 0), np.int32)
        U = ctypes.c_double()
        nseq = ctypes.c_int()
        tau_arr = None if tau is None else np.ascontiguousarray(tau, dtype=np.float64)
        cnt = lib().orc_tree_node(ctypes.byref(self.p), self.Q,
                                  np.ascontiguousarray(kbar, np.float64).reshape(-1),
                                  np.ascontiguousarray(amax, np.float64).reshape(-1),
                                  None if tau_arr is None else tau_arr.ctypes.data_as(ctypes.c_void_p),
                                  b, h, forest, k, blk, v, r, float(c_explore), leaves,
                                  ctypes.byref(U), ctypes.byref(nseq))
        if cnt < 0:
            return None, None, nseq.value
        return leaves[:cnt].copy(), U.value, nseq.value

    def backward_sampled(self, idx, dO, rows, keys):
        """Gradients of eq. (2) on samples: dQ [len(rows), d] of flat rows (b*H + h)*Nq + r
        and dK, dV [len(keys), d] of flat keys (b*H + h)*Nk + j, for every row's cells idx
        [B,H,Nq,K] and upstream gradient dO [B,H,Nq,d] (float64)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        keys = np.ascontiguousarray(keys, dtype=np.int64)
        dQ = np.zeros((max(len(rows), 1), self.d)); dK = np.zeros((max(len(keys), 1), self.d))
        dV = np.zeros_like(dK)
        lib().orc_backward_sampled(ctypes.byref(self.p), self.Q, self.K, self.V,
                                   np.ascontiguousarray(idx, np.int32).reshape(-1),
                                   np.ascontiguousarray(dO, np.float64).reshape(-1),
                                   len(rows), rows if len(rows) else np.zeros(1, np.int64), dQ.reshape(-1),
                                   len(keys), keys if len(keys) else np.zeros(1, np.int64), dK.reshape(-1),
                                   dV.reshape(-1))
        return dQ[:len(rows)], dK[:len(keys)], dV[:len(keys)]

    def select_all(self, kbar, amax):
        """eq. (7) selection of every row: idx [B,H,Nq,K] (ascending, -1 padded)."""
        idx = np.zeros((self.B, self.H, self.Nq, max(self.p.K, 1)), np.int32)
        lib().orc_select_all(ctypes.byref(self.p), self.Q, np.ascontiguousarray(kbar, np.float64).reshape(-1),
                             np.ascontiguousarray(amax, np.float64).reshape(-1), idx.reshape(-1))
        return idx[..., :self.p.K]

    def readout_rows(self, rows, idx):
        """eq. (9) for the given flat rows on caller-given cells idx [n,K]: (u, o^lr)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(rows.shape[0], self.p.K)
        u = np.zeros((rows.shape[0], self.d), np.float64)
        olr = np.zeros((rows.shape[0], self.d), np.float64)
        lib().orc_readout_rows(ctypes.byref(self.p), self.Q, self.K, self.V, rows.shape[0],
                               rows, idx, u.ctypes.data_as(ctypes.c_void_p), olr)
        return u, olr

    def rope(self, x, pos):
        """RoPE rotation of one d-vector at absolute position pos (float64)."""
        out = np.zeros(self.d, np.float64)
        lib().orc_rope(ctypes.byref(self.p), np.ascontiguousarray(x, np.float32), int(pos), out)
        return out

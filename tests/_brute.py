"""Brute-force float64 restatement of the FreeSolo forward pass, for tiny inputs.

Independent of the oracle: dense [Nq, Nk] score matrices with boolean masks, RoPE as
complex multiplication, and TopP / top-K decided by counting how many cells beat each
cell (no sorting).  Memory is O(Nq * C^2), so keep the inputs tiny.

Follows the "FreeSolo" technical summary, §3.1 eq. (2), §3.2 eqs. (3)-(4),
§3.3 eqs. (5), (7)-(9), with the same readings as the oracle for the unstated steps.
"""
import math

import numpy as np


def rope_complex(X, pos, d, base):
    """Rotate rows of X [n, d]: pair (2m, 2m+1) as a complex number times e^{i pos theta_m}."""
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    z = X[:, 0::2] + 1j * X[:, 1::2]
    z = z * np.exp(1j * np.outer(pos, theta))
    out = np.empty(X.shape, np.float64)
    out[:, 0::2] = z.real
    out[:, 1::2] = z.imag
    return out


def masked_softmax_rows(S, M):
    """Row softmax of S over the True entries of M; rows without any entry give zeros."""
    S = np.where(M, S, -np.inf)
    mx = S.max(axis=1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    E = np.where(M, np.exp(S - mx), 0.0)
    den = E.sum(axis=1, keepdims=True)
    return np.divide(E, den, out=np.zeros_like(E), where=den > 0)


def brute_forward(Q, K, V, *, w, s, K_cells, W, P, alpha, lam=None, sigma=None,
                  rope_base=10000.0, rms_eps=1e-6, pos0=0):
    """Returns O [B,H,Nq,d], sel [B,H,Nq,C] (bool), adm [B,H,Nq,C] (bool), olr, osr."""
    Q = Q.astype(np.float64)
    K = K.astype(np.float64)
    V = V.astype(np.float64)
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    C = Nk // s
    idx_q = (Nk - Nq) + np.arange(Nq)          # key-index position of each query row
    idx_k = np.arange(Nk)
    prune = not (W < 0 and P < 0)
    O = np.zeros((B, H, Nq, d))
    OLR = np.zeros((B, H, Nq, d))
    OSR = np.zeros((B, H, Nq, d))
    SEL = np.zeros((B, H, Nq, C), bool)
    ADM = np.zeros((B, H, Nq, C), bool)
    win = (idx_k[None, :] <= idx_q[:, None]) & (idx_k[None, :] >= idx_q[:, None] - w)
    cells = np.arange(C)
    cand = (cells[None, :] + 1) * s <= (idx_q[:, None] - w)           # [Nq, C]
    ncand = cand.sum(axis=1)
    for b in range(B):
        for h in range(H):
            q, k, v = Q[b, h], K[b, h], V[b, h]
            # eqs. (3)-(4)
            qr = rope_complex(q, pos0 + idx_q, d, rope_base)
            kr = rope_complex(k, pos0 + idx_k, d, rope_base)
            osr = masked_softmax_rows(qr @ kr.T / math.sqrt(d), win) @ v
            # eq. (5)
            kc = k[:C * s].reshape(C, s, d)
            kbar = kc.mean(axis=1)
            amax = np.sqrt((kc ** 2).sum(axis=2)).max(axis=1)
            # eq. (8): rank of each cell by a_c among the candidates (ties: lower index wins)
            beat_a = (amax[:, None] > amax[None, :]) | (
                (amax[:, None] == amax[None, :]) & (cells[:, None] < cells[None, :]))
            if prune:
                rankP = (cand[:, :, None] & beat_a[None, :, :]).sum(axis=1)   # [Nq, C]
                recent = cells[None, :] >= (ncand[:, None] - max(W, 0))
                adm = cand & (recent | (rankP < max(P, 0)))
            else:
                adm = cand.copy()
            # eq. (7)
            score = q @ kbar.T / math.sqrt(d)
            if lam is not None and lam[h] != 0.0:
                p_c = pos0 + (cells + 0.5) * s
                dlt = (pos0 + idx_q)[:, None] - p_c[None, :]
                erf = np.vectorize(math.erf)(dlt / (2.0 * sigma[h]))
                score = score + lam[h] * amax[None, :] * erf
            beat_s = (score[:, :, None] > score[:, None, :]) | (
                (score[:, :, None] == score[:, None, :]) & (cells[None, :, None] < cells[None, None, :]))
            rankK = (adm[:, :, None] & beat_s).sum(axis=1)
            sel = adm & (rankK < K_cells)
            # eq. (9)
            tok = np.zeros((Nq, Nk), bool)
            tok[:, :C * s] = np.repeat(sel, s, axis=1)
            u = masked_softmax_rows(q @ k.T / math.sqrt(d), tok) @ v
            ms = (u ** 2).mean(axis=1, keepdims=True)
            has = sel.any(axis=1, keepdims=True)
            olr = np.where(has, u / np.sqrt(ms + rms_eps), 0.0)
            O[b, h] = osr + alpha[h] * olr
            OLR[b, h], OSR[b, h], SEL[b, h], ADM[b, h] = olr, osr, sel, adm
    return O, SEL, ADM, OLR, OSR


def sel_to_idx(sel, K_cells):
    """Boolean selection [..., C] -> ascending cell lists padded with -1 [..., K]."""
    flat = sel.reshape(-1, sel.shape[-1])
    out = -np.ones((flat.shape[0], K_cells), np.int32)
    for t in range(flat.shape[0]):
        c = np.nonzero(flat[t])[0]
        out[t, :len(c)] = c
    return out.reshape(sel.shape[:-1] + (K_cells,))

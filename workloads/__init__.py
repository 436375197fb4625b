"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws random numbers and shapes arrays; it holds none of the method's
arithmetic.  Both sides receive the same float32 arrays (for bf16 workloads the
values are rounded to bf16 first, so the widening on either side is exact).

The workloads stand in for the long-context retrieval evaluations the FreeSolo
summary reports (RULER / single-needle retrieval at 4k-256k, "Empirical Validation"),
which are not available here.  Each recipe is stated in `CONFIGS` and `generate`.
"""
import concurrent.futures as cf
import os
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

RECIPE_NOTE = (
    "Q,K,V ~ N(0,1)/sqrt(d) (PCG64 streams spawned from the workload seed, one per "
    "(array, b, h)); bf16 workloads round to bf16 "
    "(nearest-even). Planted needles: a cell's keys become 3*|k_j|*u for a random unit u, "
    "and query rows placed after that cell's window edge become |q|*u. The 64k workload "
    "scales each cell's keys by LogNormal(0, 0.5)."
)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int = 64
    w: int = 512
    s: int = 32
    K: int = 16
    W: int = 16
    P: int = 48
    dtype: str = "bf16"           # "bf16" or "f32": type of Q, K, V and O
    seed: int = 0
    needles: int = 0              # planted needle cells per (b, h)
    needle_queries: int = 8       # query rows aligned with each needle (-1: all rows)
    cell_scale_sigma: float = 0.0  # log-normal sigma of a per-cell key scale (0: off)
    alpha: Optional[tuple] = None  # fixed per-head alpha, else U(0,1) per head
    lam: Optional[float] = None   # prior weight lambda_h (None: prior off)
    sigma: float = 1024.0         # prior width sigma_h
    rope_base: float = 10000.0
    rms_eps: float = 1e-6

    def with_(self, **kw):
        return replace(self, **kw)

    @property
    def queries(self):
        """Query tokens of one forward pass (B * Nq)."""
        return self.B * self.Nq


CONFIGS = {
    # tiny oracle check: fp32, K=8; also run with no pruning and K covering every cell
    "tiny2k": Workload("tiny2k", B=1, H=2, Nq=2048, Nk=2048, K=8, dtype="f32", seed=0,
                       alpha=(0.5, 1.0)),
    # training-length prefill with 4 planted needles per sequence
    "prefill4k": Workload("prefill4k", B=4, H=16, Nq=4096, Nk=4096, K=16, seed=1, needles=4),
    # 4x extrapolation prefill, 16 planted needles
    "prefill16k": Workload("prefill16k", B=2, H=16, Nq=16384, Nk=16384, K=16, seed=2,
                           needles=16),
    # long prefill: log-normal per-cell key scale, 64 planted needles
    "prefill64k": Workload("prefill64k", B=1, H=16, Nq=65536, Nk=65536, K=32, seed=3,
                           needles=64, cell_scale_sigma=0.5),
    # decode: 128 new queries appended to a 256k archive, one needle seen by every query
    "decode256k": Workload("decode256k", B=1, H=16, Nq=128, Nk=262144 + 128, K=32, seed=4,
                           needles=1, needle_queries=-1),
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even), kept as float32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _normal_fill(ss_children, shape, scale):
    """N(0,1)*scale float32 array; one independent stream per leading (b, h) slice,
    filled by a thread pool (deterministic whatever the scheduling)."""
    out = np.empty(shape, np.float32)
    flat = out.reshape(shape[0] * shape[1], *shape[2:])

    def fill(t):
        g = np.random.Generator(np.random.PCG64(ss_children[t]))
        g.standard_normal(out=flat[t], dtype=np.float32)
        flat[t] *= scale

    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(flat.shape[0])))
    return out


@dataclass
class Inputs:
    wl: Workload
    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    alpha: np.ndarray
    lam: Optional[np.ndarray]
    sigma: Optional[np.ndarray]
    needle_cells: list = field(default_factory=list)   # (b, h, cell, [rows])


def _unit(rng, d):
    u = rng.standard_normal(d)
    return (u / np.linalg.norm(u)).astype(np.float64)


def generate(wl: Workload) -> Inputs:
    """Draw the inputs of a workload.  Deterministic in (wl, wl.seed)."""
    B, H, Nq, Nk, d, s, w = wl.B, wl.H, wl.Nq, wl.Nk, wl.d, wl.s, wl.w
    kids = np.random.SeedSequence(wl.seed).spawn(3 * B * H + 1)
    rng = np.random.Generator(np.random.PCG64(kids[-1]))
    scale = np.float32(1.0 / np.sqrt(d))
    Q = _normal_fill(kids[0:B * H], (B, H, Nq, d), scale)
    K = _normal_fill(kids[B * H:2 * B * H], (B, H, Nk, d), scale)
    V = _normal_fill(kids[2 * B * H:3 * B * H], (B, H, Nk, d), scale)
    if wl.alpha is not None:
        alpha = np.asarray(wl.alpha, np.float64)
    else:
        alpha = rng.uniform(0.0, 1.0, H)
    C = Nk // s
    if wl.cell_scale_sigma > 0 and C > 0:
        f = rng.lognormal(0.0, wl.cell_scale_sigma, (B, H, C)).astype(np.float32)
        Kc = K[:, :, :C * s].reshape(B, H, C, s, d) * f[..., None, None]
        K[:, :, :C * s] = Kc.reshape(B, H, C * s, d)
    needles = []
    q0 = Nk - Nq                        # key-index position of query row 0
    if wl.needles > 0:
        # a needle cell c is a long-range candidate for positions i >= (c+1)s + w
        for b in range(B):
            for h in range(H):
                if wl.needle_queries < 0:
                    c_hi = (q0 - w) // s          # candidate for every query row
                else:
                    c_hi = (Nk - 1 - w) // s      # candidate for at least the last row
                if c_hi <= 0:
                    continue
                cells = rng.choice(c_hi, size=min(wl.needles, c_hi), replace=False)
                used = set()                      # a query row serves one needle only
                for c in cells:
                    c = int(c)
                    u = _unit(rng, d)
                    ks = K[b, h, c * s:(c + 1) * s].astype(np.float64)
                    nrm = np.linalg.norm(ks, axis=1, keepdims=True)
                    K[b, h, c * s:(c + 1) * s] = (3.0 * nrm * u[None, :]).astype(np.float32)
                    first = max((c + 1) * s + w - q0, 0)  # first row that sees the cell
                    if wl.needle_queries < 0:
                        rows = np.arange(first, Nq)
                    else:
                        want = min(wl.needle_queries, Nq - first - len(used))
                        picked = []
                        while len(picked) < want:
                            r = int(rng.integers(first, Nq))
                            if r not in used:
                                used.add(r)
                                picked.append(r)
                        rows = np.array(sorted(picked), np.int64)
                    for r in rows:
                        qn = np.linalg.norm(Q[b, h, r].astype(np.float64))
                        Q[b, h, r] = (qn * u).astype(np.float32)
                    needles.append((b, h, c, [int(r) for r in rows]))
    if wl.dtype == "bf16":
        Q, K, V = round_bf16(Q), round_bf16(K), round_bf16(V)
    lam = sig = None
    if wl.lam is not None:
        lam = np.full(H, wl.lam, np.float64)
        sig = np.full(H, wl.sigma, np.float64)
    return Inputs(wl, Q, K, V, alpha, lam, sig, needles)


def upstream_grad(wl: Workload, seed: int) -> np.ndarray:
    """A seeded N(0,1) upstream gradient dO [B,H,Nq,d] for the backward pass (bf16 values
    for bf16 workloads), float32."""
    g = np.random.default_rng(seed).standard_normal((wl.B, wl.H, wl.Nq, wl.d)).astype(np.float32)
    return round_bf16(g) if wl.dtype == "bf16" else g


def small(name="small", **kw) -> Workload:
    """A small workload for tests (defaults: 1x2 heads, 1024 tokens, fp32)."""
    base = dict(B=1, H=2, Nq=1024, Nk=1024, K=8, dtype="f32", seed=11)
    base.update(kw)
    return Workload(name, **base)

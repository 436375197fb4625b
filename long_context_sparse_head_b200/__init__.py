"""FreeSolo sparse-attention forward pass on NVIDIA B200 (sm_100a).

Thin Python binding of the C-ABI library libfreesolo.so (include/freesolo.h): it only
marshals arguments (tensor pointers, sizes, the current CUDA stream).  Every step of the
computation runs in the library's CUDA kernels; there is no Python or CPU fallback, and
loading fails loudly if the library has not been built (python -m
long_context_sparse_head_b200.build).

The entry points mirror the C names: `workspace_size`, `cell_summaries`, `select_topk`,
`forward`, `host_scratch_size`, `forward_host`, `sync_status`, `status_string`, and the
FS-L streaming cache `cache_bytes`, `cache_reset`, `cache_append`, `cache_attend`,
`cache_status`.
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfreesolo.so")

FS_BF16, FS_F32 = 0, 1
STATUS = {0: "FS_OK", 1: "FS_ERR_INVALID_ARG", 2: "FS_ERR_UNSUPPORTED", 3: "FS_ERR_WORKSPACE",
          4: "FS_ERR_CUDA", 5: "FS_ERR_TIMEOUT", 6: "FS_ERR_KERNEL_CHECK"}
EXPORTS = ("fs_workspace_size", "fs_cell_summaries", "fs_select_topk", "fs_forward",
           "fs_host_scratch_size", "fs_forward_host", "fs_sync_status", "fs_status_string",
           "fs_launch_count", "fs_timing_enable", "fs_kernel_times", "fs_kernel_name",
           "fs_select_topk_noalloc", "fs_cache_bytes", "fs_cache_reset", "fs_cache_append",
           "fs_cache_attend", "fs_cache_status", "fs_select_topk_rerank", "fs_forward_rerank",
           "fs_backward_workspace_size", "fs_backward", "fs_forest_bytes", "fs_forest_build",
           "fs_select_topk_tree", "fs_forward_tree", "fs_forest_append", "fs_selftest_timeout")


class FsError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s: %s (%s)" % (where, STATUS.get(code, code), status_string(code)))


class FsParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("Nq", ctypes.c_int), ("Nk", ctypes.c_int),
        ("d", ctypes.c_int), ("w", ctypes.c_int), ("s", ctypes.c_int), ("K", ctypes.c_int),
        ("W", ctypes.c_int), ("P", ctypes.c_int),
        ("rope_base", ctypes.c_float),
        ("alpha", ctypes.POINTER(ctypes.c_float)),
        ("lambda_", ctypes.POINTER(ctypes.c_float)),
        ("sigma", ctypes.POINTER(ctypes.c_float)),
        ("rms_eps", ctypes.c_float),
        ("dtype", ctypes.c_int),
    ]


_lib = None


def load():
    """Load libfreesolo.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfreesolo.so is not built; run "
                               "`python -m long_context_sparse_head_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(FsParams)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L.fs_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.fs_cell_summaries.argtypes = [P, vp, vp, vp, vp]
        L.fs_select_topk.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        L.fs_select_topk_noalloc.argtypes = [P, vp, vp, vp, vp, vp]
        L.fs_select_topk_rerank.argtypes = [P, vp, vp, vp, vp, ctypes.c_int, vp, vp, sz, vp]
        L.fs_forward_rerank.argtypes = [P, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp, sz, vp]
        L.fs_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.fs_host_scratch_size.argtypes = [P, ctypes.POINTER(sz)]
        L.fs_forward_host.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        L.fs_sync_status.argtypes = [vp, vp]
        L.fs_status_string.argtypes = [ctypes.c_int]
        L.fs_status_string.restype = ctypes.c_char_p
        L.fs_launch_count.argtypes = []
        L.fs_launch_count.restype = ctypes.c_longlong
        L.fs_timing_enable.argtypes = [ctypes.c_int]
        L.fs_kernel_times.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_longlong),
                                      ctypes.POINTER(ctypes.c_double)]
        L.fs_cache_bytes.argtypes = [P, ctypes.c_int, ctypes.POINTER(sz)]
        L.fs_cache_reset.argtypes = [P, ctypes.c_int, vp, sz, vp]
        L.fs_cache_append.argtypes = [P, ctypes.c_int, vp, sz, vp, vp, ctypes.c_int, vp]
        L.fs_cache_attend.argtypes = [P, ctypes.c_int, vp, sz, vp, ctypes.c_int, vp, vp, vp]
        L.fs_cache_status.argtypes = [vp, vp]
        L.fs_kernel_name.argtypes = [ctypes.c_int]
        L.fs_kernel_name.restype = ctypes.c_char_p
        L.fs_backward_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.fs_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        fp = ctypes.POINTER(ctypes.c_float)
        L.fs_forest_bytes.argtypes = [P, ctypes.POINTER(sz)]
        L.fs_forest_build.argtypes = [P, vp, vp, fp, vp, sz, vp]
        L.fs_forest_append.argtypes = [P, ctypes.c_int, vp, vp, fp, vp, sz, vp]
        L.fs_select_topk_tree.argtypes = [P, vp, vp, sz, ctypes.c_int, ctypes.c_float, vp, vp, sz, vp]
        L.fs_forward_tree.argtypes = [P, vp, vp, vp, fp, ctypes.c_int, ctypes.c_float, vp, vp, vp, sz, vp,
                                      sz, vp]
        L.fs_selftest_timeout.argtypes = [vp, vp]
        for name in EXPORTS:
            if name not in ("fs_status_string", "fs_launch_count", "fs_kernel_name"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code):
    return load().fs_status_string(int(code)).decode()


class Params:
    """fs_params plus the host arrays it points to (kept alive with it).

    Q [B,H,Nq,d], K/V [B,H,Nk,d]; W = P = -1 turns pruning off; lam/sigma None turns the
    erf prior off.  dtype: "bf16" or "f32".
    """

    def __init__(self, *, B, H, Nq, Nk, d=64, w=512, s=32, K=16, W=16, P=48, alpha,
                 lam=None, sigma=None, rope_base=10000.0, rms_eps=1e-6, dtype="bf16"):
        self.alpha = np.ascontiguousarray(alpha, np.float32)
        self.lam = None if lam is None else np.ascontiguousarray(lam, np.float32)
        self.sigma = None if sigma is None else np.ascontiguousarray(sigma, np.float32)
        fp = ctypes.POINTER(ctypes.c_float)
        c = FsParams()
        c.B, c.H, c.Nq, c.Nk, c.d, c.w, c.s, c.K, c.W, c.P = B, H, Nq, Nk, d, w, s, K, W, P
        c.rope_base, c.rms_eps = rope_base, rms_eps
        c.alpha = self.alpha.ctypes.data_as(fp)
        c.lambda_ = self.lam.ctypes.data_as(fp) if self.lam is not None else fp()
        c.sigma = self.sigma.ctypes.data_as(fp) if self.sigma is not None else fp()
        c.dtype = FS_BF16 if dtype == "bf16" else FS_F32
        self.c = c
        self.B, self.H, self.Nq, self.Nk, self.d, self.s, self.K = B, H, Nq, Nk, d, s, K
        self.dtype = dtype

    @property
    def C(self):
        return self.Nk // self.s

    def ref(self):
        return ctypes.byref(self.c)


def _ptr(t):
    # a plain int converts to void * through the argtypes (cheaper than a c_void_p object)
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream)


def _check(code, where):
    if code != 0:
        raise FsError(code, where)


def workspace_size(params):
    n = ctypes.c_size_t()
    _check(load().fs_workspace_size(params.ref(), ctypes.byref(n)), "fs_workspace_size")
    return n.value


def host_scratch_size(params):
    n = ctypes.c_size_t()
    _check(load().fs_host_scratch_size(params.ref(), ctypes.byref(n)), "fs_host_scratch_size")
    return n.value


def alloc_workspace(params, device="cuda"):
    """A zero-filled workspace (the device error flag must start at zero)."""
    import torch
    return torch.zeros(workspace_size(params), dtype=torch.uint8, device=device)


def cell_summaries(params, K, kbar, amax, stream=None):
    _check(load().fs_cell_summaries(params.ref(), _ptr(K), _ptr(kbar), _ptr(amax),
                                    _stream(stream)), "fs_cell_summaries")


def select_topk(params, Q, kbar, amax, idx, ws, stream=None):
    _check(load().fs_select_topk(params.ref(), _ptr(Q), _ptr(kbar), _ptr(amax), _ptr(idx),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "fs_select_topk")


def select_topk_rerank(params, Q, K, kbar, amax, idx, ws, shortlist=0, stream=None):
    """Selection by the eq. (12) token-level rerank of a shortlist of A_i (0: all of A_i)."""
    _check(load().fs_select_topk_rerank(params.ref(), _ptr(Q), _ptr(K), _ptr(kbar), _ptr(amax),
                                        int(shortlist), _ptr(idx), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)),
           "fs_select_topk_rerank")


def forward_rerank(params, Q, K, V, O, ws, kbar=None, amax=None, idx=None, shortlist=0, stream=None):
    """The forward pass with the eq. (12) rerank as its selection (idx: optional output)."""
    _check(load().fs_forward_rerank(params.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(amax),
                                    int(shortlist), _ptr(idx), _ptr(O), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "fs_forward_rerank")


def select_topk_noalloc(params, Q, kbar, amax, idx, stream=None):
    """fs_select_topk without a workspace, for callers that cannot allocate device memory:
    its scratch is a fixed array inside the library (see include/freesolo.h)."""
    _check(load().fs_select_topk_noalloc(params.ref(), _ptr(Q), _ptr(kbar), _ptr(amax),
                                         _ptr(idx), _stream(stream)), "fs_select_topk_noalloc")


def forward(params, Q, K, V, O, ws, kbar=None, amax=None, idx=None, stream=None):
    _check(load().fs_forward(params.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(amax),
                             _ptr(idx), _ptr(O), _ptr(ws), ws.numel() * ws.element_size(),
                             _stream(stream)), "fs_forward")


def forward_host(params, hQ, hK, hV, hO, dscratch, stream=None):
    _check(load().fs_forward_host(params.ref(), _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO),
                                  _ptr(dscratch), dscratch.numel() * dscratch.element_size(),
                                  _stream(stream)), "fs_forward_host")


# ---- FS-B: balanced-tree search (eqs. (10)-(11)) --------------------------------------
def forest_bytes(params):
    n = ctypes.c_size_t()
    _check(load().fs_forest_bytes(params.ref(), ctypes.byref(n)), "fs_forest_bytes")
    return n.value


def alloc_forest(params, device="cuda"):
    import torch
    return torch.empty(forest_bytes(params), dtype=torch.uint8, device=device)


def _tau(params, tau):
    if tau is None:
        return None
    arr = (ctypes.c_float * params.H)(*[float(x) for x in tau])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_float)), arr


def forest_build(params, kbar, amax, forest, tau=None, stream=None):
    """Both FS-B forests from the cell summaries; tau: per-head thresholds (None: forest 0 only)."""
    t = _tau(params, tau)
    _check(load().fs_forest_build(params.ref(), _ptr(kbar), _ptr(amax), t[0] if t else None, _ptr(forest),
                                  forest.numel() * forest.element_size(), _stream(stream)), "fs_forest_build")


def forest_append(params, prev_cells, kbar, amax, forest, tau=None, stream=None):
    """Rebuild only the trees whose blocks end after cell prev_cells (growing archive)."""
    t = _tau(params, tau)
    _check(load().fs_forest_append(params.ref(), int(prev_cells), _ptr(kbar), _ptr(amax), t[0] if t else None,
                                   _ptr(forest), forest.numel() * forest.element_size(), _stream(stream)),
           "fs_forest_append")


def select_topk_tree(params, Q, forest, idx, ws, beam, c_explore=1.0, stream=None):
    _check(load().fs_select_topk_tree(params.ref(), _ptr(Q), _ptr(forest), forest.numel() * forest.element_size(),
                                      int(beam), ctypes.c_float(c_explore), _ptr(idx), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)), "fs_select_topk_tree")


def forward_tree(params, Q, K, V, O, ws, forest, beam, c_explore=1.0, tau=None, idx=None, stream=None):
    """The forward pass with the FS-B selection (idx: optional output of the selection)."""
    t = _tau(params, tau)
    _check(load().fs_forward_tree(params.ref(), _ptr(Q), _ptr(K), _ptr(V), t[0] if t else None, int(beam),
                                  ctypes.c_float(c_explore), _ptr(idx), _ptr(O), _ptr(ws),
                                  ws.numel() * ws.element_size(), _ptr(forest),
                                  forest.numel() * forest.element_size(), _stream(stream)), "fs_forward_tree")


def backward_workspace_size(params):
    n = ctypes.c_size_t()
    _check(load().fs_backward_workspace_size(params.ref(), ctypes.byref(n)), "fs_backward_workspace_size")
    return n.value


def alloc_backward_workspace(params, device="cuda"):
    """A zero-filled backward workspace (its device error flag must start at zero)."""
    import torch
    return torch.zeros(backward_workspace_size(params), dtype=torch.uint8, device=device)


def backward(params, Q, K, V, idx, dO, dQ, dK, dV, dalpha, bws, stream=None):
    """Gradients of eq. (2) for the upstream gradient dO with the cells idx held fixed:
    dQ, dK, dV (float32, [B,H,N,d]) and dalpha (float32 [H], or None)."""
    _check(load().fs_backward(params.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(dO),
                              _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dalpha), _ptr(bws),
                              bws.numel() * bws.element_size(), _stream(stream)), "fs_backward")


def selftest_timeout(ws, stream=None):
    """Enqueue a kernel whose bounded wait runs out (about 2 s): the next sync_status(ws)
    raises FsError with FS_ERR_TIMEOUT."""
    _check(load().fs_selftest_timeout(_ptr(ws), _stream(stream)), "fs_selftest_timeout")


def sync_status(ws, stream=None):
    code = load().fs_sync_status(_ptr(ws), _stream(stream))
    _check(code, "fs_sync_status")


# ---- FS-L streaming cache ----------------------------------------------------------
def cache_bytes(params, max_block):
    n = ctypes.c_size_t()
    _check(load().fs_cache_bytes(params.ref(), int(max_block), ctypes.byref(n)), "fs_cache_bytes")
    return n.value


def alloc_cache(params, max_block, device="cuda", stream=None):
    """A cache buffer of cache_bytes(params, max_block) bytes, emptied by fs_cache_reset."""
    import torch
    cache = torch.empty(cache_bytes(params, max_block), dtype=torch.uint8, device=device)
    cache_reset(params, max_block, cache, stream)
    return cache


def cache_reset(params, max_block, cache, stream=None):
    _check(load().fs_cache_reset(params.ref(), int(max_block), _ptr(cache), cache.numel(),
                                 _stream(stream)), "fs_cache_reset")


def cache_append(params, max_block, cache, K_new, V_new, stream=None):
    """Appends K_new, V_new [B,H,n_new,d] (n_new <= max_block) to the stream."""
    _check(load().fs_cache_append(params.ref(), int(max_block), _ptr(cache), cache.numel(),
                                  _ptr(K_new), _ptr(V_new), int(K_new.shape[2]), _stream(stream)),
           "fs_cache_append")


def cache_attend(params, max_block, cache, Q_new, O, idx=None, stream=None):
    """O [B,H,n_q,d] for the n_q = Q_new.shape[2] most recent positions."""
    _check(load().fs_cache_attend(params.ref(), int(max_block), _ptr(cache), cache.numel(),
                                  _ptr(Q_new), int(Q_new.shape[2]), _ptr(idx), _ptr(O),
                                  _stream(stream)), "fs_cache_attend")


def cache_status(cache, stream=None):
    _check(load().fs_cache_status(_ptr(cache), _stream(stream)), "fs_cache_status")


# ---- diagnostics -------------------------------------------------------------------
def launch_count():
    """Kernels the library has launched since it was loaded."""
    return load().fs_launch_count()


def timing_enable(on=True):
    load().fs_timing_enable(1 if on else 0)


def kernel_times():
    """{kernel name: (launches, summed device ms)} since the previous read (then cleared)."""
    n = 32
    cnt = (ctypes.c_longlong * n)()
    ms = (ctypes.c_double * n)()
    k = load().fs_kernel_times(n, cnt, ms)
    out = {}
    for i in range(min(k, n)):
        name = load().fs_kernel_name(i).decode()
        out[name] = (cnt[i], ms[i])
    return out

"""GPU parity of the backward pass of eq. (2) (fs_backward) against the float64 oracle's
Problem.backward, on the oracle's own selection (the cells are an input held fixed).

Both sides see the same bf16-representable inputs; the GPU accumulates in float32.  The
bar is the dtype's output tolerance (2e-2 bf16, 1e-4 f32) relative to the gradient's scale
max(1, max|ref|), for dQ, dK, dV and dalpha separately."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from workloads import generate, small, upstream_grad
from tests._parity import TOL, oracle_for, params_for, tdtype

pytestmark = pytest.mark.gpu


def gpu_backward(inp, idx, dO, with_dalpha=True):
    wl = inp.wl
    p = params_for(inp)
    dt = tdtype(wl)
    Q, K, V, G = (torch.from_numpy(np.ascontiguousarray(x)).cuda().to(dt) for x in (inp.Q, inp.K, inp.V, dO))
    I = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    dQ = torch.full((wl.B, wl.H, wl.Nq, wl.d), float("nan"), device="cuda")
    dK = torch.full((wl.B, wl.H, wl.Nk, wl.d), float("nan"), device="cuda")
    dV = torch.full_like(dK, float("nan"))
    dal = torch.full((wl.H,), float("nan"), device="cuda") if with_dalpha else None
    bws = fs.alloc_backward_workspace(p)
    fs.backward(p, Q, K, V, I, G, dQ, dK, dV, dal, bws)
    fs.sync_status(bws)                            # no bounded wait ran out, no check failed
    torch.cuda.synchronize()
    out = [t.cpu().numpy().astype(np.float64) for t in (dQ, dK, dV)]
    return out + [dal.cpu().numpy().astype(np.float64) if with_dalpha else None]


def compare(got, ref, dtype):
    for name, g, r in zip(("dQ", "dK", "dV", "dalpha"), got, ref):
        if g is None:
            continue
        assert np.isfinite(g).all(), name
        scale = max(1.0, float(np.abs(r).max()) if r.size else 1.0)
        err = float(np.abs(g - r).max()) if r.size else 0.0
        assert err <= TOL[dtype] * scale, (name, err, scale)


def run_case(inp, seed=77):
    prob = oracle_for(inp)
    _, idx = prob.forward(want_idx=True)
    dO = upstream_grad(inp.wl, seed)
    ref = prob.backward(idx, dO)
    got = gpu_backward(inp, idx, dO)
    compare(got, ref, inp.wl.dtype)
    return idx


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [
    dict(),                                        # FS-L, early rows with -1 padding
    dict(lam=0.6, sigma=300.0),                    # erf prior on (a different selection)
    dict(Nq=300, Nk=1700),                         # appended queries, ragged last cell
    dict(W=-1, P=-1, K=5, Nq=1200, Nk=1200),       # base FS
    dict(w=64, K=4, W=2, P=5, Nq=777, Nk=1001),    # short window, ragged everything
    dict(B=2, H=3, K=3, Nq=640, Nk=640),           # several (b, h)
])
def test_backward_small(dtype, case):
    kw = dict(B=1, H=2, Nq=1536, Nk=1536, K=6, W=4, P=9, dtype=dtype, seed=501)
    kw.update(case)
    lam = kw.pop("lam", None)
    sigma = kw.pop("sigma", 1024.0)
    run_case(generate(small("bwd", lam=lam, sigma=sigma, **kw)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_no_cells_and_no_dalpha(dtype):
    """Rows with no candidate cell (prefix shorter than w + s) have y = 0: only the window
    carries gradient; dalpha = NULL is accepted (bf16: tiles with an empty union)."""
    inp = generate(small("bwd_short", Nq=500, Nk=500, K=4, W=2, P=3, dtype=dtype, seed=502))
    prob = oracle_for(inp)
    _, idx = prob.forward(want_idx=True)
    assert (idx < 0).all()
    dO = upstream_grad(inp.wl, 5)
    ref = prob.backward(idx, dO)
    got = gpu_backward(inp, idx, dO, with_dalpha=False)
    compare(got[:3], ref[:3], dtype)
    assert np.abs(ref[3]).max() == 0.0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_empty_queries(dtype):
    """Nq = 0: nothing to differentiate; dK = dV = 0 for every key."""
    inp = generate(small("bwd_empty", Nq=0, Nk=256, dtype=dtype, seed=503))
    got = gpu_backward(inp, np.zeros((1, 2, 0, inp.wl.K), np.int32), np.zeros((1, 2, 0, 64), np.float32))
    assert np.abs(got[1]).max() == 0.0 and np.abs(got[2]).max() == 0.0 and np.abs(got[3]).max() == 0.0


def test_backward_full_size_sampled():
    """The 16k prefill workload (B=2, H=16, 16384 tokens) at full size, on the oracle's own
    selection of every row: dQ of sampled rows and dK, dV of sampled keys (each gathering
    every row whose window or cells hold it) against the float64 oracle."""
    from workloads import CONFIGS
    inp = generate(CONFIGS["prefill16k"])
    wl = inp.wl
    prob = oracle_for(inp)
    kb, am = prob.summaries()
    idx = prob.select_all(kb, am)
    dO = upstream_grad(wl, 91)
    got = gpu_backward(inp, idx, dO)
    rng = np.random.default_rng(92)
    rows = rng.integers(0, wl.B * wl.H * wl.Nq, 48)
    # keys: some inside needle cells and frequently selected cells, the rest uniform
    flat = idx.reshape(wl.B * wl.H, -1)
    keys = []
    for _ in range(12):
        bh = int(rng.integers(0, wl.B * wl.H))
        cells = flat[bh][flat[bh] >= 0]
        c = int(rng.choice(cells)) if len(cells) else int(rng.integers(0, wl.Nk // wl.s))
        keys.append(bh * wl.Nk + c * wl.s + int(rng.integers(0, wl.s)))
    keys += rng.integers(0, wl.B * wl.H * wl.Nk, 8).tolist()
    keys = np.array(keys, np.int64)
    sq, sk, sv = prob.backward_sampled(idx, dO, rows, keys)
    d = wl.d
    gq, gk, gv = got[0].reshape(-1, d)[rows], got[1].reshape(-1, d)[keys], got[2].reshape(-1, d)[keys]
    for name, g, r in (("dQ", gq, sq), ("dK", gk, sk), ("dV", gv, sv)):
        scale = max(1.0, float(np.abs(r).max()))
        assert np.abs(g - r).max() <= TOL[wl.dtype] * scale, (name, float(np.abs(g - r).max()), scale)


def test_backward_union_overflow_sets_flag():
    """bf16 with pruning takes the tensor-core path, which holds at most 128 distinct cells
    per 128-row tile (true of any selection from A_i).  Cells drawn at random from the whole
    prefix exceed that: the call still completes, and the workspace flag reports the
    failed check (FS_ERR_KERNEL_CHECK) through fs_sync_status."""
    inp = generate(small("bwd_over", Nq=256, Nk=8192, K=6, W=4, P=9, dtype="bf16", seed=504))
    wl = inp.wl
    C = wl.Nk // wl.s
    rng = np.random.default_rng(505)
    idx = np.stack([np.sort(rng.choice(C, wl.K, replace=False)) for _ in range(wl.B * wl.H * wl.Nq)])
    idx = idx.reshape(wl.B, wl.H, wl.Nq, wl.K).astype(np.int32)
    p = params_for(inp)
    dt = tdtype(wl)
    dO = upstream_grad(wl, 6)
    Q, K, V, G = (torch.from_numpy(np.ascontiguousarray(x)).cuda().to(dt) for x in (inp.Q, inp.K, inp.V, dO))
    I = torch.from_numpy(idx).cuda()
    dQ = torch.empty((wl.B, wl.H, wl.Nq, wl.d), device="cuda")
    dK = torch.empty((wl.B, wl.H, wl.Nk, wl.d), device="cuda")
    dV = torch.empty_like(dK)
    bws = fs.alloc_backward_workspace(p)
    fs.backward(p, Q, K, V, I, G, dQ, dK, dV, None, bws)
    with pytest.raises(fs.FsError) as err:
        fs.sync_status(bws)
    assert err.value.code == 6
    fs.sync_status(bws)                            # the flag was cleared by the first read

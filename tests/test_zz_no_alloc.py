"""fs_select_topk_noalloc: selection for callers that cannot allocate device memory.

Such callers (a fixed device-memory budget planned in advance, a host framework that owns
every allocation, loops that must not stall on cudaMalloc/cudaFree) cannot pass a
workspace, so this entry point keeps its scratch in a fixed array inside the library.
These tests call it through the C ABI and require its cell indices to equal, bit for bit
(the tolerance for index results), those of fs_select_topk on the same inputs, on two
calls in a row with different problems, so stale contents of the shared array from the
previous call cannot leak into the next; the fp32, unpruned and exactly-at-the-limit
shapes take the call's other branches.  After each call the status word read by
fs_sync_status(NULL, ...) must be clear.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from tests._parity import DeviceRun
from workloads import CONFIGS, generate, small


def _problems():
    big = generate(small("noalloc-a", B=2, H=3, Nq=3000, Nk=3000, K=7, W=5, P=11,
                         dtype="bf16", seed=211, needles=2, needle_queries=4))
    little = generate(small("noalloc-b", B=1, H=2, Nq=700, Nk=1900, K=4, W=3, P=6,
                            dtype="bf16", seed=212, lam=0.5, sigma=200.0))
    return big, little


def _check_against_workspace_call(g):
    want = g.select().clone()        # fs_select_topk with a workspace
    got = torch.full_like(want, -7)
    fs.select_topk_noalloc(g.p, g.Q, g.kbar, g.amax, got)
    fs.sync_status(None)             # the status word: no timeout, no failed check
    assert torch.equal(got, want)
    assert (got >= -1).all()


@pytest.mark.gpu
def test_noalloc_matches_workspace_selection_twice():
    for inp in _problems():          # two calls in a row: large problem, then small one
        _check_against_workspace_call(DeviceRun(inp))


@pytest.mark.gpu
def test_noalloc_f32_and_unpruned_paths():
    # fp32 inputs take the CUDA-core selection; W = P = -1 (no pruning) skips the exit
    # table altogether; both must still equal fs_select_topk
    f32 = generate(small("noalloc-f32", B=1, H=2, Nq=1500, Nk=2500, K=6, W=4, P=9,
                         dtype="f32", seed=213, needles=1))
    _check_against_workspace_call(DeviceRun(f32))
    unpruned = generate(small("noalloc-base", B=1, H=2, Nq=2048, Nk=2048, K=9, W=-1, P=-1,
                              dtype="bf16", seed=214))
    _check_against_workspace_call(DeviceRun(unpruned))


@pytest.mark.gpu
def test_noalloc_exactly_at_the_limit():
    # B * H * floor(Nk / s) == FS_NOALLOC_MAX_CELLS: accepted, every entry of the array in
    # use.  The selection reads only Q, kbar and amax, so those are drawn on the device
    # (no keys needed): 4 x 256 heads x 1024 cells, 128 appended queries per head.
    B, H, Nk, Nq, K = 4, 256, 32768, 128, 8
    assert B * H * (Nk // 32) == 1 << 20
    gen = torch.Generator(device="cuda").manual_seed(215)
    p = fs.Params(B=B, H=H, Nq=Nq, Nk=Nk, K=K, alpha=np.ones(H))
    Q = (torch.randn((B, H, Nq, 64), generator=gen, device="cuda") / 8).to(torch.bfloat16)
    kbar = torch.randn((B, H, Nk // 32, 64), generator=gen, device="cuda") / 64
    amax = torch.rand((B, H, Nk // 32), generator=gen, device="cuda") + 0.5
    want = torch.empty((B, H, Nq, K), dtype=torch.int32, device="cuda")
    ws = fs.alloc_workspace(p)
    fs.select_topk(p, Q, kbar, amax, want, ws)
    fs.sync_status(ws)
    got = torch.full_like(want, -7)
    fs.select_topk_noalloc(p, Q, kbar, amax, got)
    fs.sync_status(None)
    assert torch.equal(got, want)
    assert (got >= 0).all()          # every query has more than K admitted cells here


@pytest.mark.gpu
def test_noalloc_full_size_prefill_matches():
    inp = generate(CONFIGS["prefill16k"])
    g = DeviceRun(inp)
    want = g.select().clone()
    got = torch.full_like(want, -7)
    fs.select_topk_noalloc(g.p, g.Q, g.kbar, g.amax, got)
    torch.cuda.synchronize()
    assert torch.equal(got, want)


def test_noalloc_rejects_tables_past_the_limit():
    # 2 x 256 heads x 2048 cells = 1,048,576 + 2048 > FS_NOALLOC_MAX_CELLS: refused before
    # anything touches a device
    p = fs.Params(B=2, H=256, Nq=128, Nk=65536 + 64, K=8, alpha=np.ones(256))
    with pytest.raises(fs.FsError) as e:
        fs.select_topk_noalloc(p, None, None, None, None, stream=0)
    assert e.value.code in (1, 2)


class _Ptr:
    def __init__(self, v):
        self.v = v

    def data_ptr(self):
        return self.v


def test_noalloc_limit_is_checked_before_pointers():
    p = fs.Params(B=2, H=256, Nq=128, Nk=65536 + 64, K=8, alpha=np.ones(256))
    t = _Ptr(0x1000)
    with pytest.raises(fs.FsError) as e:
        fs.select_topk_noalloc(p, t, t, t, t, stream=0)
    assert e.value.code == 2

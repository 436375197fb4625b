"""fs_forward_host: the forward pass on host buffers, pipelined over chunks of heads on
internal streams.  In fp32 (no fused kernel) its output must equal fs_forward's on device
copies of the same inputs bit for bit.  In bf16 a chunk is a smaller call, so the fused
kernel may split its tiles over a different number of CTAs: each split rounds its P to
bf16 against its own running maximum, so the two agree within the bf16 output tolerance,
not bit for bit.  Both must match the oracle on sampled rows."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from workloads import generate, small
from tests._parity import TOL, DeviceRun, check_selection, expected_output, oracle_for, sample_rows, tdtype

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [
    dict(B=2, H=6),                                  # 4 chunks per batch entry: 2, 2, 2 heads
    dict(B=1, H=3),                                  # one head per chunk
    dict(B=9, H=2, Nq=512, Nk=640),                  # chunks of whole batch entries
    dict(B=1, H=9, lam=0.7, sigma=200.0),           # per-head prior offsets, ragged chunk
    dict(B=3, H=4, Nq=700, Nk=1900),                 # decode shape
])
def test_forward_host_matches_device(dtype, case):
    kw = dict(Nq=1024, Nk=1024, K=6, W=4, P=9, dtype=dtype, seed=701)
    kw.update(case)
    lam = kw.pop("lam", None)
    sigma = kw.pop("sigma", 1024.0)
    inp = generate(small("host", lam=lam, sigma=sigma, **kw))
    wl = inp.wl
    g = DeviceRun(inp)
    ref = g.numpy(g.forward()).copy()
    dt = tdtype(wl)
    hQ, hK, hV = (torch.from_numpy(x).to(dt).pin_memory() for x in (inp.Q, inp.K, inp.V))
    hO = torch.full(hQ.shape, float("nan"), dtype=dt).pin_memory()
    scratch = torch.zeros(fs.host_scratch_size(g.p), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        fs.forward_host(g.p, hQ, hK, hV, hO, scratch, stream)
    stream.synchronize()
    got = hO.float().numpy()
    if wl.dtype == "f32":
        assert np.array_equal(got, ref)
    else:
        assert np.abs(got - ref).max() <= TOL["bf16"], np.abs(got - ref).max()
    prob = oracle_for(inp)
    rows = sample_rows(wl, 24, seed=3)
    idx = g.numpy(g.select())
    check_selection(inp, prob.summaries(), idx, rows)
    err = np.abs(np.stack([got[b, h, r] for b, h, r in rows]) - expected_output(inp, prob, rows, idx)).max()
    assert err <= TOL[wl.dtype], err

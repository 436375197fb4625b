"""The device error flag, end to end on the GPU without a fault: a kernel whose bounded
wait runs out (the same wait the tensor-core kernels use) records FS_ERR_TIMEOUT, the
status call reports and clears it, and the context stays usable for a normal call."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from workloads import generate, small
from tests._parity import TOL, DeviceRun, oracle_for, expected_output

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    inp = generate(small("status", Nq=512, Nk=1024, K=4, W=2, P=5, dtype="bf16", seed=601))
    g = DeviceRun(inp)
    fs.sync_status(g.ws)                               # clean before
    fs.selftest_timeout(g.ws)
    with pytest.raises(fs.FsError) as err:
        fs.sync_status(g.ws)
    assert err.value.code == 5                         # FS_ERR_TIMEOUT
    fs.sync_status(g.ws)                               # the flag was cleared by the read
    # a normal forward call afterwards still matches the oracle
    g.summaries()
    idx = g.numpy(g.select())
    wl = inp.wl
    O = g.numpy(g.forward()).reshape(wl.B, wl.H, wl.Nq, wl.d)
    rows = [(0, h, r) for h in range(wl.H) for r in range(0, wl.Nq, 7)]
    want = expected_output(inp, oracle_for(inp), rows, idx)
    got = np.stack([O[b, h, r] for b, h, r in rows])
    assert np.abs(got - want).max() <= TOL[wl.dtype]
    fs.sync_status(g.ws)

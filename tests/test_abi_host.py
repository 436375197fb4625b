"""C-ABI checks that need no GPU: the library loads, exports every symbol its header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import long_context_sparse_head_b200 as fs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fs_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_function():
    L = fs.load()
    declared = header_functions()
    assert "fs_forward" in declared and "fs_select_topk" in declared
    for name in declared:
        assert hasattr(L, name), name
    assert set(fs.EXPORTS) <= set(declared)


def test_binding_declares_every_signature():
    """Every declared function is in the binding with its argument types set (an
    undeclared size_t would be passed as a 32-bit int)."""
    L = fs.load()
    assert set(header_functions()) <= set(fs.EXPORTS)
    for name in fs.EXPORTS:
        assert getattr(L, name).argtypes is not None, name


def test_tree_arguments_rejected_on_host():
    p = params(W=-1, P=-1)
    n = fs.forest_bytes(p)
    assert n > 0
    big = fs.Params(B=1, H=2, Nq=256, Nk=4096, alpha=[0.5, 1.0], W=-1, P=-1)
    assert fs.forest_bytes(big) > n
    for beam in (0, 65):
        with pytest.raises(fs.FsError) as e:
            fs.select_topk_tree(p, _FakeTensor(1), _FakeTensor(n), _FakeTensor(1), _FakeTensor(1 << 20), beam,
                                stream=0)
        assert e.value.code == 1
    with pytest.raises(fs.FsError) as e:          # forest buffer too small
        fs.select_topk_tree(p, _FakeTensor(1), _FakeTensor(n - 1), _FakeTensor(1), _FakeTensor(1 << 20), 8,
                            stream=0)
    assert e.value.code == 3


class _FakeTensor:
    """Stands in for a device tensor in calls that must fail before any launch."""

    def __init__(self, nbytes):
        self.nbytes = nbytes

    def data_ptr(self):
        return 0x1000

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def test_status_strings():
    for code in range(7):
        assert fs.status_string(code)
    assert fs.status_string(99) == "unknown status"


def params(**kw):
    base = dict(B=1, H=2, Nq=256, Nk=256, alpha=[0.5, 1.0])
    base.update(kw)
    return fs.Params(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(Nq=300, Nk=256), 1), (dict(K=-1), 1), (dict(W=-1, P=4), 1),
    (dict(d=32), 2), (dict(s=16), 2), (dict(w=500), 2), (dict(K=65), 2),
    (dict(W=1024, P=1025), 2), (dict(w=-1), 1),
])
def test_invalid_params_are_rejected(kw, code):
    with pytest.raises(fs.FsError) as e:
        fs.workspace_size(params(**kw))
    assert e.value.code == code


def test_prior_needs_positive_sigma():
    with pytest.raises(fs.FsError) as e:
        fs.workspace_size(params(lam=[0.5, 0.5], sigma=[1.0, 0.0]))
    assert e.value.code == 1
    with pytest.raises(fs.FsError):
        fs.workspace_size(params(lam=[0.5, 0.5]))
    fs.workspace_size(params(lam=[0.5, 0.5], sigma=[1.0, 2.0]))


class FakeTensor:
    """A stand-in with a device pointer: argument checks fail before any use."""

    def __init__(self, ptr, n=1):
        self.ptr, self.n = ptr, n

    def data_ptr(self):
        return self.ptr

    def numel(self):
        return self.n

    def element_size(self):
        return 1


def test_forward_rejects_small_workspace_before_launch():
    p = params()
    need = fs.workspace_size(p)
    t = FakeTensor(0x1000)
    with pytest.raises(fs.FsError) as e:
        fs.forward(p, t, t, t, t, FakeTensor(0x2000, need - 1), stream=0)
    assert e.value.code == 3
    with pytest.raises(fs.FsError) as e:
        fs.forward(p, None, t, t, t, FakeTensor(0x2000, need), stream=0)
    assert e.value.code == 1
    with pytest.raises(fs.FsError) as e:      # summaries must come as a pair
        fs.forward(p, t, t, t, t, FakeTensor(0x2000, need), kbar=t, stream=0)
    assert e.value.code == 1


def test_workspace_size_grows_with_problem():
    a = fs.workspace_size(params())
    b = fs.workspace_size(params(Nq=4096, Nk=4096))
    assert 0 < a < b
    assert fs.host_scratch_size(params()) > a


def test_cache_memory_is_bounded():
    """The FS-L streaming cache's size depends on the budgets and the block size, never on
    how many tokens pass through it; base FS (no pruning) has no bounded state."""
    import numpy as np
    p = fs.Params(B=1, H=16, Nq=1, Nk=1, K=32, W=16, P=48, alpha=np.ones(16), dtype="bf16")
    assert fs.cache_bytes(p, 1) < fs.cache_bytes(p, 64) < fs.cache_bytes(p, 4096)
    q = fs.Params(B=1, H=16, Nq=1, Nk=1, K=32, W=-1, P=-1, alpha=np.ones(16), dtype="bf16")
    with pytest.raises(fs.FsError) as e:
        fs.cache_bytes(q, 1)
    assert e.value.code == 2
    with pytest.raises(fs.FsError) as e:
        fs.cache_bytes(p, 0)
    assert e.value.code == 1

"""GPU parity of the FS-L streaming cache: tokens are appended block by block and each
block's queries are attended from the cache alone; the answer must be the batch
forward pass's on the whole prefix so far, judged against the float64 oracle run on
that prefix (same acceptance rules as the batch parity tests: selected cells up to
near-ties, output within the dtype's tolerance)."""
import numpy as np
import pytest
import torch

import long_context_sparse_head_b200 as fs
from workloads import Inputs, generate, small
from tests._parity import TOL, check_selection, expected_output, oracle_for, params_for, tdtype

pytestmark = pytest.mark.gpu


def sub_inputs(inp, t, n_q):
    """The batch problem the cache answers after t tokens: keys and values 0..t-1 and
    the queries at the n_q most recent positions (query row r at position t - n_q + r)."""
    wl = inp.wl.with_(Nq=n_q, Nk=t)
    return Inputs(wl=wl, Q=np.ascontiguousarray(inp.Q[:, :, t - n_q:t]),
                  K=np.ascontiguousarray(inp.K[:, :, :t]), V=np.ascontiguousarray(inp.V[:, :, :t]),
                  alpha=inp.alpha, lam=inp.lam, sigma=inp.sigma)


def stream(inp, blocks, max_block, attend=None, check_every=1):
    """Append `blocks` tokens at a time; after a block, attend its last min(n, attend)
    positions and compare with the oracle (every `check_every`-th block)."""
    wl = inp.wl
    p = params_for(inp)
    cache = fs.alloc_cache(p, max_block)
    dt = tdtype(wl)
    Qd, Kd, Vd = (torch.from_numpy(x).cuda().to(dt) for x in (inp.Q, inp.K, inp.V))
    t, checked, ties = 0, 0, 0
    for step, nb in enumerate(blocks):
        fs.cache_append(p, max_block, cache, Kd[:, :, t:t + nb].contiguous(), Vd[:, :, t:t + nb].contiguous())
        t += nb
        if step % check_every:
            continue
        n_q = nb if attend is None else max(1, min(nb, attend))
        Qn = Qd[:, :, t - n_q:t].contiguous()
        O = torch.full_like(Qn, float("nan"))
        idx = torch.empty((wl.B, wl.H, n_q, wl.K), dtype=torch.int32, device="cuda")
        fs.cache_attend(p, max_block, cache, Qn, O, idx)
        fs.cache_status(cache)
        sub = sub_inputs(inp, t, n_q)
        prob = oracle_for(sub)
        rows = [(b, h, r) for b in range(wl.B) for h in range(wl.H) for r in range(n_q)]
        idx_n = idx.cpu().numpy()
        exact, tie = check_selection(sub, prob.summaries(), idx_n, rows)
        ties += tie
        got = O.float().cpu().numpy()
        assert np.isfinite(got).all(), t
        want = expected_output(sub, prob, rows, idx_n)
        err = np.abs(np.stack([got[b, h, r] for b, h, r in rows]) - want).max()
        assert err <= TOL[wl.dtype], (t, n_q, err)
        checked += len(rows)
    assert ties <= max(2, checked // 100), (ties, checked)
    return t


BLOCKS = [600, 1, 1, 1, 37, 130, 200, 1, 64, 500, 3, 17, 600, 90]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [
    dict(),                                   # W + P well below the prefix: evictions
    dict(lam=0.6, sigma=300.0),               # erf prior on
    dict(W=0, P=7),                           # TopP only
    dict(W=6, P=0),                           # recent cells only
    dict(B=2, H=3, K=3, needles=2, needle_queries=4),
])
def test_cache_stream_blocks(dtype, case):
    kw = dict(B=1, H=2, Nq=2245, Nk=2245, K=6, W=4, P=9, dtype=dtype, seed=301)
    kw.update(case)
    lam = kw.pop("lam", None)
    sigma = kw.pop("sigma", 1024.0)
    inp = generate(small("cache", lam=lam, sigma=sigma, **kw))
    assert stream(inp, BLOCKS, max_block=600) == sum(BLOCKS)


def test_cache_decode_one_token_at_a_time():
    """max_block = 1: the decode loop; every 97th position checked."""
    inp = generate(small("decode", Nq=1800, Nk=1800, K=5, W=3, P=6, dtype="bf16", seed=302))
    stream(inp, [1] * 1800, max_block=1, check_every=97)


def test_cache_short_window():
    """w = 64: cells become candidates soon after they complete."""
    inp = generate(small("shortw", Nq=1500, Nk=1500, w=64, K=4, W=2, P=5, dtype="f32", seed=303))
    stream(inp, [100, 1, 31, 32, 33, 200, 1, 1, 100, 500, 1, 499], max_block=500)


def test_cache_attend_past_the_stream_is_reported():
    """Attending more positions than were appended is caught by the kernel's own check."""
    inp = generate(small("early", Nq=64, Nk=64, dtype="f32", seed=305))
    p = params_for(inp)
    cache = fs.alloc_cache(p, 64)
    Kd = torch.from_numpy(inp.K[:, :, :5].copy()).cuda()
    fs.cache_append(p, 64, cache, Kd, Kd)
    Q = torch.zeros((1, 2, 6, 64), device="cuda")
    O = torch.empty_like(Q)
    fs.cache_attend(p, 64, cache, Q, O)
    with pytest.raises(fs.FsError) as e:
        fs.cache_status(cache)
    assert e.value.code == 6
    fs.cache_status(cache)          # the flag was cleared


def test_cache_full_size_decode_sampled():
    """The 256k-token decode workload through the streaming cache: the archive appended in
    blocks of 128, then the 128 new tokens appended and their queries attended in one call;
    selection (near-tie rule) and output judged against the float64 oracle on sampled rows
    (the same rows the batch decode test uses)."""
    from workloads import CONFIGS
    from tests._parity import sample_rows
    inp = generate(CONFIGS["decode256k"])
    wl = inp.wl
    p = params_for(inp)
    mb = 128
    cache = fs.alloc_cache(p, mb)
    dt = tdtype(wl)
    K, V = (torch.from_numpy(x).cuda().to(dt) for x in (inp.K, inp.V))
    for a in range(0, wl.Nk, mb):
        fs.cache_append(p, mb, cache, K[:, :, a:a + mb].contiguous(), V[:, :, a:a + mb].contiguous())
    Qd = torch.from_numpy(inp.Q).cuda().to(dt)
    O = torch.full_like(Qd, float("nan"))
    idx = torch.empty((wl.B, wl.H, wl.Nq, wl.K), dtype=torch.int32, device="cuda")
    fs.cache_attend(p, mb, cache, Qd, O, idx)
    fs.cache_status(cache)
    prob = oracle_for(inp)
    rows = sample_rows(wl, 200, seed=1)
    idx_n = idx.cpu().numpy()
    exact, tie = check_selection(inp, prob.summaries(), idx_n, rows)
    assert tie <= max(2, len(rows) // 50), (exact, tie)
    got = O.float().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(np.stack([got[b, h, r] for b, h, r in rows]) - expected_output(inp, prob, rows, idx_n)).max()
    assert err <= TOL[wl.dtype], err

"""The GPU parity judge itself, checked on the CPU: it accepts the oracle's own
selections and rejects plausible wrong ones (a worse cell swapped in, the best unselected
cell swapped for the K-th where their gap exceeds the near-tie tolerance, a
non-candidate, unsorted output, a missing pad)."""
import numpy as np
import pytest

from tests._parity import check_selection, oracle_for, sample_rows
from workloads import generate, small


@pytest.fixture(scope="module")
def case():
    inp = generate(small("judge", B=1, H=2, Nq=2048, Nk=2048, K=6, W=4, P=9, dtype="bf16",
                         seed=77))
    wl = inp.wl
    prob = oracle_for(inp)
    kbar, amax = prob.summaries()
    rows = [r for r in sample_rows(wl, 60, 3) if prob.candidate_count(wl.Nk - wl.Nq + r[2]) > 12]
    flat = np.array([(b * wl.H + h) * wl.Nq + r for b, h, r in rows])
    _, idx = prob.forward(rows=flat, want_idx=True)
    full = -np.ones((wl.B, wl.H, wl.Nq, wl.K), np.int32)
    for t, (b, h, r) in enumerate(rows):
        full[b, h, r] = idx[t]
    return inp, prob, (kbar, amax), full, rows


def test_accepts_oracle_selection(case):
    inp, _, sums, full, rows = case
    exact, tie = check_selection(inp, sums, full, rows)
    assert exact == len(rows) and tie == 0


def test_rejects_worse_cell(case):
    inp, prob, sums, full, rows = case
    b, h, r = rows[0]
    _, acells, scores = prob.select_row(sums[0], sums[1], b, h, r)
    chosen = set(full[b, h, r].tolist())
    worst = min((c for c in acells if c not in chosen), key=lambda c: scores[list(acells).index(c)])
    bad = full.copy()
    row = sorted([c for c in chosen if c >= 0][1:] + [int(worst)])
    bad[b, h, r, :len(row)] = row
    with pytest.raises(AssertionError):
        check_selection(inp, sums, bad, [(b, h, r)])


def test_rejects_non_candidate_and_bad_layout(case):
    inp, _, sums, full, rows = case
    b, h, r = rows[0]
    n = inp.wl.Nk - inp.wl.Nq + r
    bad = full.copy()
    bad[b, h, r, -1] = n // 32 + 5                       # a cell inside the window
    bad[b, h, r] = np.sort(bad[b, h, r])
    with pytest.raises(AssertionError):
        check_selection(inp, sums, bad, [(b, h, r)])
    bad = full.copy()
    bad[b, h, r] = bad[b, h, r][::-1]                     # descending
    with pytest.raises(AssertionError):
        check_selection(inp, sums, bad, [(b, h, r)])


def test_rejects_boundary_swap_outside_tolerance(case):
    # the K-th selected cell traded for the best unselected one: a near-tie only if their
    # scores lie within 1e-4 of the row's score scale; rows with a wider gap must fail
    inp, prob, sums, full, rows = case
    tested = 0
    for b, h, r in rows:
        _, acells, scores = prob.select_row(sums[0], sums[1], b, h, r)
        sc = dict(zip(acells.tolist(), scores.tolist()))
        chosen = [int(c) for c in full[b, h, r] if c >= 0]
        rest = [c for c in sc if c not in chosen]
        if not rest:
            continue
        kth = min(chosen, key=lambda c: sc[c])
        best_out = max(rest, key=lambda c: sc[c])
        if sc[kth] - sc[best_out] <= 1e-4 * max(np.abs(scores).max(), abs(sc[kth])):
            continue
        bad = full.copy()
        row = sorted([c for c in chosen if c != kth] + [best_out])
        bad[b, h, r, :len(row)] = row
        with pytest.raises(AssertionError):
            check_selection(inp, sums, bad, [(b, h, r)])
        tested += 1
    assert tested >= 10, tested

"""The parity checkers themselves, on the CPU: they accept the oracle's own answers
and reject planted mistakes (a swapped kept position, a retained list that is not
the closure of its candidates, a budget off by one).  The "GPU" outputs here are
oracle outputs, altered by hand."""
import numpy as np
import pytest

import synth
from focus_testutil import (TIE_TOL, check_dynamic_budget, check_selection_all, check_structured,
                            selection_margin)


def test_selection_margin_hand_case():
    # raw delta of a 6-token block; pooled = MaxPool1D(k=3) of it, nothing decoded
    raw = np.array([0.10, 0.50, 0.20, 0.30, 0.45, 0.00])
    pooled = np.array([0.50, 0.50, 0.50, 0.45, 0.45, 0.45])
    dec = np.zeros(6, np.uint8)
    # k = 3: the cut is at 0.50 (a plateau of copies of raw[1]); nearest other raw value 0.45
    assert selection_margin(raw, pooled, dec, 3) == pytest.approx(0.05)
    # k = 4: the cut is at 0.45; nearest other raw value 0.50 (0.30 is further)
    assert selection_margin(raw, pooled, dec, 4) == pytest.approx(0.05)
    # a raw value hidden inside a window still counts: 0.499 never appears pooled
    raw2 = raw.copy()
    raw2[2] = 0.499
    assert selection_margin(raw2, pooled, dec, 3) == pytest.approx(0.001)
    # two raw positions holding exactly the value at the cut (duplicated keys): a tie
    raw3 = np.array([0.10, 0.50, 0.20, 0.30, 0.50, 0.00])
    pooled3 = np.array([0.50, 0.50, 0.50, 0.50, 0.50, 0.50])
    assert selection_margin(raw3, pooled3, dec, 3) == 0.0
    # nothing to decide: k = 0 or every masked position kept
    assert selection_margin(raw, pooled, dec, 0) == np.inf
    dec2 = np.array([1, 1, 1, 0, 0, 1], np.uint8)
    assert selection_margin(raw, pooled, dec2, 2) == np.inf


@pytest.fixture(scope="module")
def case(orc):
    p = synth.make_problem(1, seed=31, wide_logits=True, overrides=dict(R=8, prefix=("uniform", 0, 300)))
    ref = orc.evict(p)
    return p, ref


def test_selection_checker_accepts_the_oracle_and_rejects_a_swap(case, orc):
    p, ref = case
    dec, bud = p.decoded.numpy(), p.budget.numpy()
    rep = check_selection_all(ref["kept"], ref["cu_seqlens"], ref, dec, bud, orc)
    assert rep["exact"] == rep["requests"] == p.R
    assert rep["decided"] >= 1
    # swap one kept position of a decided request for a masked position not kept
    from focus_testutil import selection_margins
    m = selection_margins(ref, dec, bud)
    r = int(np.flatnonzero(m > TIE_TOL)[0])
    a, b = int(ref["cu_seqlens"][r]), int(ref["cu_seqlens"][r + 1])
    assert b > a
    spare = np.setdiff1d(np.flatnonzero(dec[r] == 0), ref["kept"][a:b])
    assert spare.size
    bad = ref["kept"].copy()
    bad[a:b] = np.sort(np.concatenate([ref["kept"][a:b - 1], spare[-1:]]))
    with pytest.raises(AssertionError):
        check_selection_all(bad, ref["cu_seqlens"], ref, dec, bud, orc)


def test_structured_checker_accepts_the_oracle_and_rejects_a_broken_closure(case, orc):
    p, ref = case
    dec, bud = p.decoded.numpy(), p.budget.numpy()
    kept3, cu3, _ = orc.select_structured(ref["pooled"], dec, bud, 3)
    rep = check_structured(kept3, cu3, ref["kept"], ref["cu_seqlens"], ref, dec, bud, 3, orc)
    assert rep["structured_exact"] == p.R
    # drop one retained position that is not a candidate (a predecessor or a filler)
    for r in range(p.R):
        seg = kept3[cu3[r]:cu3[r + 1]]
        extra = np.setdiff1d(seg, ref["kept"][ref["cu_seqlens"][r]:ref["cu_seqlens"][r + 1]])
        if extra.size:
            break
    else:
        pytest.fail("no request retains more than its candidates")
    drop = cu3[r] + int(np.flatnonzero(seg == extra[0])[0])
    bad = np.delete(kept3, drop)
    bad_cu = cu3.copy()
    bad_cu[r + 1:] -= 1
    with pytest.raises(AssertionError):
        check_structured(bad, bad_cu, ref["kept"], ref["cu_seqlens"], ref, dec, bud, 3, orc)


def test_budget_checker_accepts_the_oracle_and_rejects_off_by_one(case, orc):
    p, ref = case
    dec = p.decoded.numpy()
    avg = np.random.default_rng(5).uniform(0.0, 4.0, size=p.R).astype(np.float32)
    k = orc.dynamic_budget(ref["pooled"], dec, avg.astype(np.float64))
    pinned = check_dynamic_budget(k, ref["pooled"], dec, avg)
    assert pinned >= 1
    # a request whose bounds meet: any other budget is rejected
    for r in range(p.R):
        bad = k.copy()
        bad[r] = k[r] + 1 if k[r] < int((dec[r] == 0).sum()) else k[r] - 1
        try:
            check_dynamic_budget(bad, ref["pooled"], dec, avg)
        except AssertionError:
            return
    pytest.fail("no budget change was caught")

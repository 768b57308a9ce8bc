"""CPU checks of the parity tests' own comparison rule (tests/s3r_testlib.py): the first
decision where a GPU round departs from the oracle's must be a boundary case of its own,
with everything before it identical. The "GPU" rounds here are the oracle's rounds with
one decision changed by hand."""
import numpy as np
import pytest

from tests.s3r_testlib import MARGIN, compare_round_decisions


def _res(drafts, tokens, margins, draft_margin):
    return dict(drafts=np.asarray(drafts), tokens=np.asarray(tokens), n_out=len(tokens),
                margins=np.asarray(margins, dtype=np.float64),
                draft_margin=np.asarray(draft_margin, dtype=np.float64))


K = 3
FAR = 0.3


def test_identical_round_is_exact():
    r = _res([5, 6, 7], [5, 9], [FAR, FAR, FAR], [FAR] * K)
    assert compare_round_decisions(r, [5, 6, 7], [5, 9, -1, -1], 2, K) is True


def test_a_different_draft_needs_its_own_draft_margin():
    r = _res([5, 6, 7], [5, 6, 7, 1], [FAR] * 4, [FAR, 1e-7, FAR])
    assert compare_round_decisions(r, [5, 8, 7], [5, 8, 7, 2], 4, K) is False
    # an earlier draft near its boundary does not excuse a later one that is not
    r = _res([5, 6, 7], [5, 6, 7, 1], [FAR] * 4, [1e-7, FAR, FAR])
    with pytest.raises(AssertionError):
        compare_round_decisions(r, [5, 6, 8], [5, 6, 8, 2], 4, K)


def test_a_flipped_accept_needs_that_tests_margin():
    # oracle: accepts draft 0, rejects draft 1 (margin m1), draws 4
    r = _res([5, 6, 7], [5, 4], [FAR, 1e-6, FAR], [FAR] * K)
    # GPU accepted draft 1 too: differs at position 1, excused by margins[1]
    assert compare_round_decisions(r, [5, 6, 7], [5, 6, 3], 3, K) is False
    # the same flip with a far margin fails
    r = _res([5, 6, 7], [5, 4], [FAR, FAR, FAR], [FAR] * K)
    with pytest.raises(AssertionError):
        compare_round_decisions(r, [5, 6, 7], [5, 6, 3], 3, K)
    # a near accept test EARLIER than the flip does not excuse it
    r = _res([5, 6, 7], [5, 6, 4], [1e-7, FAR, FAR, FAR], [FAR] * K)
    with pytest.raises(AssertionError):
        compare_round_decisions(r, [5, 6, 7], [5, 2], 2, K)


def test_a_different_draw_needs_the_draw_margin():
    r = _res([5, 6, 7], [5, 4], [FAR, FAR, 1e-6], [FAR] * K)
    assert compare_round_decisions(r, [5, 6, 7], [5, 3], 2, K) is False
    r = _res([5, 6, 7], [5, 4], [FAR, 1e-6, FAR], [FAR] * K)   # the accept margin is near,
    with pytest.raises(AssertionError):                        # but the draw differs
        compare_round_decisions(r, [5, 6, 7], [5, 3], 2, K)


def test_bonus_draw_after_all_accepted():
    r = _res([5, 6, 7], [5, 6, 7, 9], [FAR, FAR, FAR, 2e-6], [FAR] * K)
    assert compare_round_decisions(r, [5, 6, 7], [5, 6, 7, 8], 4, K) is False
    r = _res([5, 6, 7], [5, 6, 7, 9], [FAR, FAR, FAR, 2 * MARGIN], [FAR] * K)
    with pytest.raises(AssertionError):
        compare_round_decisions(r, [5, 6, 7], [5, 6, 7, 8], 4, K)

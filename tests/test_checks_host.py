"""The parity gate itself: the top-k comparison allows swaps only among entries
within rtol * |k-th oracle score| of the k-th oracle score, and nothing wider.

Each case builds an oracle row, its exact top-k and a "GPU" selection that
differs from it by one planted swap, then checks that the gate accepts or
rejects it as the stated band says.
"""
import numpy as np
import pytest

from tests._checks import assert_topk_equivalent


def _row():
    # 20 scores: a planted outlier (100) far above the rest, the k-th (k = 5) at 10.0
    s = np.array([100.0, 20.0, 15.0, 12.0, 10.0, 9.995, 9.5, 9.0, 1.0, 0.5,
                  0.1, -1.0, -2.0, -3.0, -4.0, -5.0, -6.0, -7.0, -8.0, -9.0])
    ref = np.sort(np.argsort(-s, kind="stable")[:5])
    return s, ref


def _swap(ref, out, inn):
    g = sorted((set(ref.tolist()) - {out}) | {inn})
    return np.array([g])


def test_identical_sets_pass_with_zero_swaps():
    s, ref = _row()
    assert assert_topk_equivalent(ref[None], ref[None], s[None], 1e-2) == 0


def test_swap_within_band_of_kth_passes_and_is_counted():
    s, ref = _row()
    # 9.995 is within 1e-2 * 10.0 = 0.1 of the k-th score 10.0
    rep = []
    n = assert_topk_equivalent(_swap(ref, 4, 5), ref[None], s[None], 1e-2, report=rep)
    assert n == 1 and rep == [(0, 1)]


def test_swap_outside_band_of_kth_fails_even_within_rtol_of_row_max():
    s, ref = _row()
    # 9.5 is 0.5 below the k-th score: outside 1e-2 * |10.0| = 0.1, but inside
    # 1e-2 * max|row| = 1.0, the wider band an earlier form of the gate allowed
    with pytest.raises(AssertionError):
        assert_topk_equivalent(_swap(ref, 4, 6), ref[None], s[None], 1e-2)


def test_swap_of_an_entry_far_above_kth_fails():
    s, ref = _row()
    # dropping the 12.0 entry for 9.995: the dropped entry is 2.0 above the k-th score
    with pytest.raises(AssertionError):
        assert_topk_equivalent(_swap(ref, 3, 5), ref[None], s[None], 1e-2)


def test_band_scales_with_the_kth_scores_magnitude_when_it_is_negative():
    s, ref = _row()
    neg = s - 20.0                 # same order; the k-th score is now -10.0
    assert assert_topk_equivalent(_swap(ref, 4, 5), ref[None], neg[None], 1e-2) == 1   # 0.005 from it
    with pytest.raises(AssertionError):
        assert_topk_equivalent(_swap(ref, 4, 6), ref[None], neg[None], 1e-2)           # 0.5 from it


def test_structure_checks_still_apply():
    s, ref = _row()
    with pytest.raises(AssertionError):  # not ascending
        assert_topk_equivalent(ref[::-1][None], ref[None], s[None], 1e-2)
    with pytest.raises(AssertionError):  # a selected position beyond the row's length
        assert_topk_equivalent(ref[None], ref[None], s[None], 1e-2, n_valid=np.array([3]))
    short = np.array([list(ref[:4]) + [-1]])
    with pytest.raises(AssertionError):  # fewer entries than the oracle
        assert_topk_equivalent(short, ref[None], s[None], 1e-2)

"""The comparison helpers themselves (CPU): a NaN, a one-sided infinity or a bad padding slot must
fail the parity checks that use them."""
import numpy as np
import pytest

from tests.cmp_utils import assert_close, check_topk_row


def test_assert_close_rejects_nan_and_one_sided_inf():
    ref = np.array([1.0, 2.0, -np.inf, np.nan])
    assert_close(ref.copy(), ref, 1e-3, 1e-3)                    # equal, with matching -inf and NaN
    for bad in (np.array([np.nan, 2.0, -np.inf, np.nan]),     # NaN where the reference is finite
                np.array([1.0, 2.0, -np.inf, 0.0]),           # a value where the reference is NaN
                np.array([1.0, np.inf, -np.inf, np.nan]),     # +inf where the reference is finite
                np.array([1.0, 2.0, 5.0, np.nan])):           # finite where the reference is -inf
        with pytest.raises(AssertionError):
            assert_close(bad, ref, 1e-3, 1e-3)


def test_check_topk_row_padding_contract():
    scores = np.array([5.0, 4.0, -np.inf, 3.0])
    ids = np.arange(4)
    # k = 5 > 3 visible candidates: 3 ids and exactly two -1 slots, in any order
    assert check_topk_row(np.array([-1, 3, 0, -1, 1]), scores, ids, 5) == 0
    with pytest.raises(AssertionError):
        check_topk_row(np.array([-2, 3, 0, -1, 1]), scores, ids, 5)     # a negative slot other than -1
    with pytest.raises(AssertionError):
        check_topk_row(np.array([3, 0, 1, 1, -1]), scores, ids, 5)      # a duplicate in place of padding
    with pytest.raises(AssertionError):
        check_topk_row(np.array([2, 0, 1, -1, -1]), scores, ids, 5)     # an invisible candidate

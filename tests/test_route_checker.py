"""The routing checker of the parity tests, against planted selections (CPU).

The rule it enforces: a GPU selection equals the oracle's top-k set unless the
token's k-th vs (k+1)-th key gap is below 1e-4, and its slot order equals the
oracle's except for swaps of keys within 1e-4; whatever that lets through must
still be a valid top-k within 1e-4.  Each planted mistake below is one a
wrong router could make; a checker that exempted every token with any small
gap (and then accepted any selection for it) would let the first three pass.
"""
import numpy as np
import pytest

from tests import harness as H

E, K = 8, 2


def keys_with(row):
    """One token's selection keys (float64)."""
    return np.asarray([row], dtype=np.float64)


def old_rule_accepts(idx_g, keys, k):
    """The earlier, wider exemption: any adjacent gap among the top k+1 keys
    below 1e-4 excused the token, whatever it selected."""
    srt = -np.sort(-keys, axis=1)[:, :k + 1]
    tie = ((srt[:, :-1] - srt[:, 1:]) < H.NEAR_TIE).any(axis=1)
    from oracle.moe_oracle import topk_select
    diff = (np.asarray(idx_g) != topk_select(keys, k)).any(axis=1)
    return not (diff & ~tie).any()


def test_exact_selection_passes():
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 0.5, 0.0, -2.0, 1.0])
    c = H.check_selection(np.array([[1, 3]]), keys, K)
    assert c == dict(set_ties=0, order_ties=0, set_flips=0, order_flips=0)


def test_wrong_expert_on_an_order_tie_is_rejected():
    # slots 0 and 1 nearly tie (3.0 vs 3.00005), the set gap (3.0 vs 1.0) is
    # wide: picking expert 7 (key 1.0) instead of expert 3 is a wrong set
    keys = keys_with([0.1, 3.00005, -1.0, 3.0, 0.5, 0.0, -2.0, 1.0])
    planted = np.array([[1, 7]])
    assert old_rule_accepts(planted, keys, K)
    with pytest.raises(AssertionError, match="different expert set"):
        H.check_selection(planted, keys, K)


def test_far_expert_on_a_set_tie_is_rejected():
    # the k-th and (k+1)-th keys tie (2.0 vs 2.00003), so either may be
    # chosen; expert 6 (key -2.0) may not
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 2.00003, 0.0, -2.0, 1.0])
    planted = np.array([[1, 6]])
    assert old_rule_accepts(planted, keys, K)
    with pytest.raises(AssertionError, match="below the k-th key"):
        H.check_selection(planted, keys, K)


def test_far_order_swap_on_a_tied_token_is_rejected():
    # a set tie lets the set differ, not the order of keys 3.0 and 2.0
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 2.00003, 0.0, -2.0, 1.0])
    planted = np.array([[4, 1]])
    assert old_rule_accepts(planted, keys, K)
    with pytest.raises(AssertionError, match="order their slots"):
        H.check_selection(planted, keys, K)


def test_valid_flip_on_a_set_tie_is_accepted_and_counted():
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 2.00003, 0.0, -2.0, 1.0])
    c = H.check_selection(np.array([[1, 3]]), keys, K)   # oracle picks 1, 4
    assert c["set_ties"] == 1 and c["set_flips"] == 1 and c["order_flips"] == 0


def test_near_order_swap_is_accepted_and_counted():
    keys = keys_with([0.1, 3.00005, -1.0, 3.0, 0.5, 0.0, -2.0, 1.0])
    c = H.check_selection(np.array([[3, 1]]), keys, K)
    assert c == dict(set_ties=0, order_ties=1, set_flips=0, order_flips=1)


def test_far_order_swap_is_rejected():
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 0.5, 0.0, -2.0, 1.0])
    with pytest.raises(AssertionError, match="order their slots"):
        H.check_selection(np.array([[3, 1]]), keys, K)


def test_duplicate_and_out_of_range_are_rejected():
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 0.5, 0.0, -2.0, 1.0])
    with pytest.raises(AssertionError, match="twice"):
        H.check_selection(np.array([[1, 1]]), keys, K)
    with pytest.raises(AssertionError, match="out of range"):
        H.check_selection(np.array([[1, 8]]), keys, K)


def test_equal_keys_may_take_either_expert():
    # exact ties: the oracle takes the lower index, any tied expert is valid
    keys = keys_with([0.1, 3.0, -1.0, 2.0, 2.0, 0.0, -2.0, 1.0])
    c = H.check_selection(np.array([[1, 4]]), keys, K)
    assert c["set_flips"] == 1


def test_many_tokens_random_keys():
    # random keys: the oracle's own selection passes with zero flips; a
    # selection shifted by one rank fails on every token with a wide gap
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((500, 64))
    from oracle.moe_oracle import topk_select
    k = 6
    idx = topk_select(keys, k)
    c = H.check_selection(idx, keys, k)
    assert c["set_flips"] == 0 and c["order_flips"] == 0
    shifted = np.argsort(-keys, axis=1, kind="stable")[:, 1:k + 1]
    with pytest.raises(AssertionError):
        H.check_selection(shifted, keys, k)

"""The GPU parity gates themselves, checked on the CPU: each planted mistake in a
result handed to the checkers must fail, and each allowed difference (a tie at
the k-th score, bf16 rounding of the output) must pass."""
import numpy as np
import pytest
import torch

from parity_util import check_attn, check_index_set


def scores_with_tie():
    """Top 4 = {1, 4, 6, 7}; the 4th (index 7) and 5th (index 2) differ by 1e-9."""
    return np.array([0.10, 0.90, 0.50, 0.20, 0.80, 0.05, 0.70, 0.50 + 1e-9, 0.01])


def test_index_exact_match_passes():
    s = scores_with_tie()
    assert check_index_set(np.array([1, 4, 6, 7]), s, 4) == 0


def test_index_tie_at_kth_score_is_tolerated():
    s = scores_with_tie()
    # the oracle keeps 7 (0.5 + 1e-9); index 2 (0.5) lies within 1e-6 of the k-th score
    assert check_index_set(np.array([1, 2, 4, 6]), s, 4) == 2


def test_index_dropped_top_entry_fails():
    s = scores_with_tie()
    with pytest.raises(AssertionError, match="beyond the tie window"):
        check_index_set(np.array([2, 4, 6, 7]), s, 4)  # lost index 1 (0.9)


def test_index_layout_errors_fail():
    s = scores_with_tie()
    with pytest.raises(AssertionError, match="not strictly ascending"):
        check_index_set(np.array([4, 1, 6, 7]), s, 4)
    with pytest.raises(AssertionError, match="not strictly ascending"):
        check_index_set(np.array([1, 4, 4, 7]), s, 4)
    with pytest.raises(AssertionError, match="range"):
        check_index_set(np.array([1, 4, 6, 9]), s, 4)
    with pytest.raises(AssertionError, match="padding"):
        check_index_set(np.array([1, 4, 6, 7, 3]), s, 4)
    # budget above the candidate count: all entries, then padding
    assert check_index_set(np.concatenate([np.arange(9), [-1, -1]]), s, 11) == 0


def test_index_window_scale_for_logits_near_zero():
    """Block logits straddle 0: the window follows the row's largest |score|."""
    s = np.array([2e-2, -1e-2, 1e-9, 0.0, 3e-3])
    # k = 3: oracle keeps {0, 4, 2}; index 3 (0.0) is 1e-9 from the k-th score
    assert check_index_set(np.array([0, 3, 4]), s, 3, window_scale=np.abs(s).max()) == 2
    with pytest.raises(AssertionError):
        check_index_set(np.array([0, 3, 4]), s, 3)  # relative to |1e-9| it is far


def test_attention_tolerances():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((64, 32)) * 0.1
    ok = torch.from_numpy(ref).to(torch.bfloat16)
    mx, mean = check_attn(ok, None, ref, None)
    assert mx <= 1e-3 and mean <= 1e-3
    one_off = ref.copy()
    one_off[5, 3] += 9e-3  # a single element inside max-abs
    check_attn(torch.from_numpy(one_off).float(), None, ref, None)
    far = ref.copy()
    far[5, 3] += 2e-2
    with pytest.raises(AssertionError, match="max abs"):
        check_attn(torch.from_numpy(far).float(), None, ref, None)
    drift = ref + 2e-3  # every element inside max-abs, the mean outside
    with pytest.raises(AssertionError, match="mean abs"):
        check_attn(torch.from_numpy(drift).float(), None, ref, None)
    bad = ref.copy()
    bad[0, 0] = np.nan
    with pytest.raises(AssertionError, match="non-finite"):
        check_attn(torch.from_numpy(bad).float(), None, ref, None)


def test_attention_lse_and_empty_rows():
    ref = np.zeros((3, 4))
    lse_ref = np.array([1.5, -np.inf, 0.25])
    out = torch.zeros(3, 4)
    check_attn(out, torch.tensor([1.5, -np.inf, 0.2502]), ref, lse_ref)
    with pytest.raises(AssertionError, match="empty rows"):
        check_attn(out, torch.tensor([1.5, 0.0, 0.25]), ref, lse_ref)
    with pytest.raises(AssertionError, match="lse max abs"):
        check_attn(out, torch.tensor([1.5, -np.inf, 0.26]), ref, lse_ref)

"""The comparison helpers every GPU parity test goes through fail when they
should (CPU): a parity test is only as strong as its checker, so each helper
is fed a planted difference just past its stated tolerance and one just
inside it."""
import numpy as np
import pytest
import torch

from parity import OUT_TOL, SCORE_FLOOR, SCORE_REL, assert_csr_equal, assert_out_close, assert_scores_close


def test_csr_equal_rejects_any_moved_or_missing_id():
    rp = np.array([0, 2, 2, 5])
    col = np.array([1, 3, 0, 2, 4])
    assert_csr_equal((rp, col), (rp.copy(), col.copy()))
    with pytest.raises(AssertionError):
        assert_csr_equal((rp, np.array([1, 3, 0, 2, 5])), (rp, col))            # one id differs
    with pytest.raises(AssertionError):
        assert_csr_equal((np.array([0, 1, 2, 5]), col), (rp, col))              # same ids, other rows
    with pytest.raises(AssertionError):
        assert_csr_equal((np.array([0, 2, 2, 4]), col[:4]), (rp, col))          # one id missing


def test_scores_close_holds_the_relative_bound_and_its_floor():
    ref = np.array([0.5, 1e-3, 1e-9, 0.0])
    assert_scores_close(ref * (1 + 0.9 * SCORE_REL), ref)
    bad = ref.copy()
    bad[1] *= 1 + 1.1 * SCORE_REL
    with pytest.raises(AssertionError):
        assert_scores_close(bad, ref)
    # below the floor the absolute bound applies: a tiny or zero reference still
    # rejects an error above 1e-12
    tiny = ref.copy()
    tiny[3] = 0.9 * SCORE_FLOOR
    assert_scores_close(tiny, ref)
    tiny[3] = 2 * SCORE_FLOOR
    with pytest.raises(AssertionError):
        assert_scores_close(tiny, ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_out_close_checks_max_abs_and_frobenius(dtype):
    abs_tol, fro_tol = OUT_TOL[dtype]
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((4, 64))
    # one element just inside the max-abs bound: both checks pass
    g = ref.copy()
    g[0, 0] += 0.9 * abs_tol
    assert_out_close(g, ref, dtype)
    # one element just past it
    g[0, 0] = ref[0, 0] + 1.1 * abs_tol
    with pytest.raises(AssertionError):
        assert_out_close(g, ref, dtype)
    # every element inside the max-abs bound, but together past the Frobenius one
    small = ref * (0.5 * abs_tol / np.abs(ref).max())
    g = small + 0.9 * abs_tol * np.sign(rng.standard_normal(small.shape))
    assert np.abs(g - small).max() <= abs_tol
    with pytest.raises(AssertionError):
        assert_out_close(g, small, dtype)
    # an all-zero reference (an empty row's output) accepts only outputs near zero
    zero = np.zeros((2, 8))
    assert_out_close(zero, zero, dtype)
    with pytest.raises(AssertionError):
        assert_out_close(zero + 2 * abs_tol, zero, dtype)

"""The parity bound itself (CPU only): |gpu - ref| <= 2^-7 |ref| + 2^-8 rms(ref),
checked by hand on small arrays, NaN rejected, and the statistics each passing
check records for the session summary."""
import numpy as np
import pytest

import gpu_util


def test_tolerance_formula_by_hand():
    ref = np.array([3.0, -4.0])                     # rms = sqrt((9 + 16) / 2) = 3.5355...
    rms = np.sqrt(12.5)
    assert np.allclose(gpu_util.tolerance(ref), [3 / 128 + rms / 256, 4 / 128 + rms / 256], rtol=0, atol=1e-15)


def test_check_close_passes_at_the_bound_and_fails_beyond_it():
    ref = np.array([1.0, 2.0, -8.0, 0.0])
    tol = gpu_util.tolerance(ref)
    n0 = len(gpu_util.PARITY_LOG)
    assert gpu_util.check_close(ref + tol, ref, "at bound") == pytest.approx(1.0)
    what, ratio, half, n = gpu_util.PARITY_LOG[n0]
    assert what == "at bound" and ratio == pytest.approx(1.0) and half == 1.0 and n == 4
    with pytest.raises(AssertionError):
        gpu_util.check_close(ref + 1.01 * tol, ref, "beyond")
    with pytest.raises(AssertionError):
        gpu_util.check_close(np.array([np.nan, 2.0, -8.0, 0.0]), ref, "nan")
    assert len(gpu_util.PARITY_LOG) == n0 + 1      # failures are not recorded
    del gpu_util.PARITY_LOG[n0:]                   # keep the session summary to real checks


def test_tolerance_takes_a_given_whole_matrix_rms():
    """Sampled checks pass the whole output's rms; the bound uses it in place of
    the sample's own."""
    ref = np.array([3.0, -4.0])
    assert np.allclose(gpu_util.tolerance(ref, rms=10.0), [3 / 128 + 10 / 256, 4 / 128 + 10 / 256],
                       rtol=0, atol=1e-15)
    with pytest.raises(AssertionError):
        gpu_util.check_close(ref + 3 / 128 + 0.5 / 256 + 1e-9, ref, "small rms", rms=0.5)


def test_whole_output_rms_is_lowered_below_the_exact_one():
    """The GPU output's rms lowered by 2^-6 stays below rms(ref) whenever every
    element is within the bound: the bound built on it is never looser."""
    import torch
    rng = np.random.default_rng(3)
    ref = rng.standard_normal(4000) * np.where(rng.random(4000) < 0.01, 50.0, 1.0)
    tol = gpu_util.tolerance(ref)
    worst = ref + np.sign(ref) * tol              # every element at the bound, pushed outward
    est = gpu_util.full_rms_from_gpu(torch.from_numpy(worst))
    assert est < float(np.sqrt(np.mean(ref * ref)))

"""Host logic of the parity comparison (no GPU): the per-tensor error measure
max|gpu - ref| / max|ref| and its rule for references below fp32's normal
range, which must accept only the fp32 rounding of the reference."""
import numpy as np

from tests.parity_util import FLT_SUBNORMAL_ULP, TOL, assert_within, rel_err


def test_relative_to_the_largest_reference_value():
    ref = np.array([1.0, -4.0, 0.5])
    gpu = ref + np.array([0.0, 0.02, -0.01])
    assert abs(rel_err(gpu, ref) - 0.02 / 4.0) < 1e-15
    assert rel_err(ref, ref) == 0.0
    assert rel_err(np.zeros((0, 3)), np.zeros((0, 3))) == 0.0


def test_all_zero_reference_needs_exact_zero():
    ref = np.zeros(5)
    assert rel_err(np.zeros(5), ref) == 0.0
    assert rel_err(np.array([0, 0, 1e-30, 0, 0]), ref) == float("inf")


def test_reference_below_fp32_normal_range():
    # a gradient that decayed to ~1e-189: zero in fp32, so the GPU value must be zero
    ref = np.full(8, 1e-189)
    assert rel_err(np.zeros(8), ref) == 0.0
    assert rel_err(np.full(8, 1e-3), ref) == float("inf")      # would pass a plain tol
    assert rel_err(np.full(8, 2e-2), ref) == float("inf")
    # a subnormal reference: its fp32 rounding, within one subnormal ulp
    sub = np.array([3.5 * FLT_SUBNORMAL_ULP, -7 * FLT_SUBNORMAL_ULP])
    r32 = sub.astype(np.float32).astype(np.float64)
    assert rel_err(r32, sub) == 0.0
    assert rel_err(r32 + FLT_SUBNORMAL_ULP, sub) == 0.0
    assert rel_err(r32 + 3 * FLT_SUBNORMAL_ULP, sub) == float("inf")


def test_assert_within_reports_every_tensor():
    assert_within({"y": 1e-3, "dW": 5e-3}, "bf16")
    try:
        assert_within({"y": 1e-3, "dW": 3e-2}, "bf16", "case")
    except AssertionError as e:
        assert "dW" in str(e) and str(TOL["bf16"]) in str(e)
    else:
        raise AssertionError("a tensor above the tolerance passed")
    try:
        assert_within({"dh0": float("inf")}, "fp32")
    except AssertionError:
        pass
    else:
        raise AssertionError("inf passed")

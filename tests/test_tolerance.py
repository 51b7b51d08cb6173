"""The comparison rules themselves (CPU)."""
import numpy as np

from synthetic import bf16_bits_to_f64, f32_to_bf16_bits
from tolerance import bf16_check, dw_fp32_check, rstd_check, ulp_bf16


def test_ulp_values():
    assert ulp_bf16(np.array([1.0]))[0] == 2.0 ** -7
    assert ulp_bf16(np.array([1.99]))[0] == 2.0 ** -7
    assert ulp_bf16(np.array([2.0]))[0] == 2.0 ** -6
    assert ulp_bf16(np.array([-0.75]))[0] == 2.0 ** -8


def test_bf16_rounding_passes_and_three_ulp_fails():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((8, 64))
    rounded = bf16_bits_to_f64(f32_to_bf16_bits(ref.astype(np.float32)))
    assert bf16_check(rounded, ref)["ok"]
    worse = ref + 3 * ulp_bf16(ref) * np.sign(ref)
    # 3 ulp exceeds both 2 ulp and (for values high in their binade) 1e-2 relative
    assert not bf16_check(worse, ref)["ok"]


def test_floor_covers_cancellation_only():
    ref = np.array([[1.0, -1.0, 1e-9, 2.0]])
    gpu = ref.copy()
    gpu[0, 2] = 1e-9 + 1e-6  # tiny absolute error on a near-zero element
    assert bf16_check(gpu, ref)["ok"]
    gpu[0, 2] = 1e-2  # large absolute error
    assert not bf16_check(gpu, ref)["ok"]


def test_dw_and_rstd_rules():
    ref = np.array([1.0, -2.0, 1e-8, 3.0])
    assert dw_fp32_check(ref * (1 + 5e-4), ref)["ok"]
    assert not dw_fp32_check(ref * (1 + 5e-3), ref)["ok"]
    assert rstd_check(ref[[0, 1, 3]] * (1 + 5e-6), ref[[0, 1, 3]])["ok"]
    assert not rstd_check(ref[[0, 1, 3]] * (1 + 5e-5), ref[[0, 1, 3]])["ok"]


def test_subnormal_results_may_flush_to_zero():
    ref = np.array([[1e-40, -3e-39, 0.0]])
    assert bf16_check(np.zeros_like(ref), ref)["ok"]
    assert not bf16_check(np.array([[1e-37, 0.0, 0.0]]), ref)["ok"]


def test_nonfinite_reference_must_be_matched():
    ref = np.array([[1.0, np.nan, np.inf, -np.inf, 2.0]])
    gpu = ref.copy()
    assert bf16_check(gpu, ref)["ok"]
    # a NaN turned into a number, an infinity of the wrong sign, a finite value for an
    # infinity, and an infinity or NaN where the oracle is finite are all failures
    for j, v in ((1, 0.0), (2, -np.inf), (3, 3e38), (0, np.inf), (4, np.nan)):
        g = ref.copy()
        g[0, j] = v
        assert not bf16_check(g, ref)["ok"], (j, v)
        assert not dw_fp32_check(g[0], ref[0])["ok"], (j, v)
    assert dw_fp32_check(ref[0], ref[0])["ok"]


def test_nan_elsewhere_in_a_row_does_not_void_the_rest():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((4, 32))
    ref[1, 5] = np.nan
    ref[2, 7] = np.inf
    gpu = ref.copy()
    assert bf16_check(gpu, ref)["ok"]
    gpu[1, 6] += 0.5  # a wrong finite element in the row that holds the NaN
    rep = bf16_check(gpu, ref)
    assert not rep["ok"] and rep["first_bad"] == [1, 6]
    gpu = ref.copy()
    gpu[2, 0] *= 1.2  # and in the row that holds the infinity
    assert not bf16_check(gpu, ref)["ok"]


def test_rstd_nonfinite():
    ref = np.array([1.0, np.nan, 3.0])
    assert rstd_check(ref.copy(), ref)["ok"]
    assert not rstd_check(np.array([1.0, 1.0, 3.0]), ref)["ok"]
    assert not rstd_check(np.array([1.0, np.nan, np.inf]), ref)["ok"]


def test_rstd_zero_reference_needs_zero():
    ref = np.array([0.0, 2.0])
    assert rstd_check(np.array([0.0, 2.0]), ref)["ok"]
    assert not rstd_check(np.array([1e-30, 2.0]), ref)["ok"]

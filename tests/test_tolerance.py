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

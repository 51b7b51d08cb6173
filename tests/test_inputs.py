"""The seeded input generator and the BF16 rounding helpers (CPU only)."""
import numpy as np
import torch

from synthetic import (WORKLOADS, bf16_bits_to_f32, bf16_bits_to_f64, f32_to_bf16_bits,
                       make_inputs, make_workload_inputs)


def test_bf16_rounding_special_values():
    vals = np.array([1.0, 1.00390625, 1.01171875, -2.5, 0.0, -0.0, np.inf, -np.inf,
                     np.finfo(np.float32).max, 1e-40], dtype=np.float32)
    bits = f32_to_bf16_bits(vals)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to even (1.0)
    assert bits[1] == 0x3F80
    # 1 + 3*2^-8 is a tie between 1+2^-7 and 1+2^-6: rounds to even (1+2^-6)
    assert bits[2] == 0x3F82
    assert bits[0] == 0x3F80 and bits[3] == 0xC020
    assert bits[4] == 0x0000 and bits[5] == 0x8000
    assert bits[6] == 0x7F80 and bits[7] == 0xFF80
    assert bits[8] == 0x7F80  # above the largest finite BF16 after rounding
    nan_bits = f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))
    assert np.isnan(bf16_bits_to_f32(nan_bits))[0]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        (rng.standard_normal(10000) * 1e30).astype(np.float32),
        (rng.standard_normal(10000) * 1e-38).astype(np.float32),
        rng.integers(0, 2**32, 10000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ])
    mine = f32_to_bf16_bits(a)
    theirs = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    finite = np.isfinite(a)
    assert np.array_equal(mine[finite], theirs[finite])
    assert np.array_equal(np.isnan(bf16_bits_to_f32(mine)), np.isnan(a))


def test_widening_is_exact():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    f32 = bf16_bits_to_f32(bits)
    f64 = bf16_bits_to_f64(bits)
    ok = ~np.isnan(f32)
    assert np.array_equal(f32[ok].astype(np.float64), f64[ok])
    assert np.array_equal(f32_to_bf16_bits(f32[ok]), bits[ok])


def test_generator_is_seeded_and_shaped():
    a = make_inputs(64, 32, seed=0)
    b = make_inputs(64, 32, seed=0)
    c = make_inputs(64, 32, seed=1)
    for k in ("x", "g", "dy", "w"):
        assert np.array_equal(a[k], b[k])
        assert a[k].dtype == np.uint16
    assert not np.array_equal(a["x"], c["x"])
    assert a["x"].shape == (64, 32) and a["w"].shape == (32,)


def test_distributions():
    d = make_inputs(4096, 256, seed=0, g_std=2.0)
    x, g, w = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "w"))
    assert abs(np.std(x) - 1.0) < 0.01 and abs(np.mean(x)) < 0.01
    assert abs(np.std(g) - 2.0) < 0.02  # g_std is a standard deviation
    assert abs(np.mean(w) - 1.0) < 0.03 and abs(np.std(w) - 0.1) < 0.02


def test_outlier_rows():
    wl = WORKLOADS["wide_16384x4096"].scaled(2000)
    d = make_workload_inputs(wl)
    rows = d["outlier_rows"]
    assert len(rows) == 20 and len(np.unique(rows)) == 20
    x = bf16_bits_to_f64(d["x"])
    rms = np.sqrt(np.mean(x * x, axis=1))
    mask = np.zeros(2000, bool); mask[rows] = True
    assert np.all(rms[mask] > 30) and np.all(rms[~mask] < 2)


def test_workload_table():
    assert [w.M for w in WORKLOADS.values()] == [1024, 65536, 368640, 16384, 262144]
    assert [w.N for w in WORKLOADS.values()] == [128, 128, 128, 4096, 256]
    assert int(round(0.01 * 16384)) == 164

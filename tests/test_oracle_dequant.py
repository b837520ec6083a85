"""Pins of the oracle's dequantization ([HS] holysheep.ai "FP8 混精度训练
DeepSeek 671B" (zh), 2.2: code value times the tile's scale) and of its
fp32 -> bf16 rounding."""
import numpy as np
import pytest
import torch


def test_unit_codes_reproduce_each_tiles_scale(orc):
    """Every code 0x38 (= 1.0) and a distinct scale per tile: the output is
    the tile's scale at every position of that tile (tile indexing, ragged
    last row block)."""
    rng = np.random.default_rng(1)
    for tile_rows, R, C in ((1, 5, 384), (128, 300, 256)):
        q = np.full((R, C), 0x38, dtype=np.uint8)
        s = rng.uniform(0.5, 2.0, ((R + tile_rows - 1) // tile_rows, C // 128)).astype(np.float32)
        out = orc.dequantize_fp32(q, s, tile_rows)
        for r in range(R):
            for c in range(0, C, 64):
                assert out[r, c] == s[r // tile_rows, c // 128]


def test_scale_one_gives_the_code_values(orc):
    q = np.arange(256, dtype=np.uint8).reshape(2, 128)
    out = orc.dequantize_fp32(q, np.ones((2, 1), np.float32), 1)
    ref = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).float().numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(out[finite], ref[finite])
    assert np.all(np.isnan(out[~finite]))


def test_power_of_two_scale_shifts_exactly(orc):
    q = np.arange(0, 0x7F, dtype=np.uint8)
    q = np.concatenate([q, q | 0x80, [0, 0]]).astype(np.uint8).reshape(2, 128)
    base = orc.dequantize_fp32(q, np.ones((2, 1), np.float32), 1)
    for k in (-20, -3, 5, 40):
        out = orc.dequantize_fp32(q, np.full((2, 1), 2.0 ** k, np.float32), 1)
        assert np.array_equal(out, (base.astype(np.float64) * 2.0 ** k).astype(np.float32))


def test_round_trip_within_half_a_code_step(orc):
    """dequantize(quantize(x)) differs from x by at most half the E4M3 step at
    |x| (2^-4 relative in the normal range, 2^-10 s in the subnormal one)."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.integers(-6, 6, (64, 1)))).astype(np.float32)
    q, s = orc.quantize_act_1x128(x)
    y = orc.dequantize_fp32(q, s, 1).astype(np.float64)
    srep = np.repeat(s.astype(np.float64), 128, axis=1)
    bound = np.maximum(2.0 ** -4 * np.abs(x.astype(np.float64)), 2.0 ** -10 * srep) * (1 + 1e-6)
    assert np.all(np.abs(y - x) <= bound)


def test_single_rounding_of_the_exact_product(orc):
    """The fp32 result is the exact product rounded once: checked against
    the product of the two factors as Python integers scaled by powers of
    two (exact rational arithmetic)."""
    from fractions import Fraction
    rng = np.random.default_rng(3)
    q = rng.integers(0, 0x7F, (1, 128)).astype(np.uint8)
    s = np.array([[np.float32(1.0) / np.float32(3.0)]], dtype=np.float32)
    out = orc.dequantize_fp32(q, s, 1)
    dec = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).float().numpy()
    for j in range(128):
        exact = Fraction(float(dec[0, j])) * Fraction(float(s[0, 0]))
        got = Fraction(float(out[0, j]))
        up = np.nextafter(out[0, j], np.float32(np.inf))
        dn = np.nextafter(out[0, j], np.float32(-np.inf))
        # no fp32 value is closer to the exact product
        assert abs(got - exact) <= abs(Fraction(float(up)) - exact)
        assert abs(got - exact) <= abs(Fraction(float(dn)) - exact)


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        # exact ties between two bf16 values, both parities
                        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        np.array([0.0, -0.0, 3.0e38, -1e-40], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16_bits(x), ref)

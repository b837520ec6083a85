"""Pins for the oracle's E4M3 codec (CPU only).

The codec is written from the E4M3 format definition; these tests pin it to
things other than itself: PyTorch's own float8_e4m3fn decoding and casting
(a library routine), the OCP FP8 format's published extreme values, the
constant the pages print, and properties round-to-nearest-even must have.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_constants.txt")


def load_golden():
    vals = {}
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, value = line.split()[:2]
            vals[key] = float(value)
    return vals


ALL = np.arange(256, dtype=np.uint8)
FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
NONNEG = np.arange(0x7F, dtype=np.uint8)          # 0x00..0x7E, increasing in value


def torch_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def torch_encode(values):
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_matches_torch_all_256(orc):
    mine = orc.e4m3_decode(ALL)
    ref = torch_decode(ALL)
    nan_m, nan_r = np.isnan(mine), np.isnan(ref)
    assert np.array_equal(nan_m, nan_r)
    assert set(np.flatnonzero(nan_m)) == {0x7F, 0xFF}
    assert np.array_equal(mine[~nan_m], ref[~nan_r])
    # signed zeros decode with their sign
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])


def test_decode_format_extremes(orc):
    """OCP OFP8 E4M3: max normal S.1111.110 = 448, min normal S.0001.000 = 2^-6,
    max subnormal S.0000.111 = 0.875 * 2^-6, min subnormal S.0000.001 = 2^-9."""
    d = orc.e4m3_decode
    assert d(np.uint8(0x7E)) == 448.0 and d(np.uint8(0xFE)) == -448.0
    assert d(np.uint8(0x08)) == 2.0 ** -6
    assert d(np.uint8(0x07)) == 0.875 * 2.0 ** -6
    assert d(np.uint8(0x01)) == 2.0 ** -9
    assert d(np.uint8(0x38)) == 1.0          # exponent field 7 = bias
    assert FINITE.size == 254
    fin = orc.e4m3_decode(FINITE)
    assert np.max(fin) == 448.0 and np.min(np.abs(fin[fin != 0])) == 2.0 ** -9


def test_pages_constant_448_is_e4m3_max(orc):
    g = load_golden()
    fin = orc.e4m3_decode(FINITE)
    assert np.max(fin) == g["e4m3_max"] == g["e4m3_range_abs"]


def test_encode_roundtrip_every_finite_code(orc):
    vals = orc.e4m3_decode(FINITE).astype(np.float32)
    # -0.0 decodes to -0.0 and must come back as 0x80
    assert np.array_equal(orc.e4m3_encode(vals), FINITE)


def test_nonnegative_codes_are_monotone(orc):
    v = orc.e4m3_decode(NONNEG)
    assert np.all(np.diff(v) > 0)


def test_midpoints_go_to_even_code(orc):
    v = orc.e4m3_decode(NONNEG)
    lo, hi = v[:-1], v[1:]
    mids = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (lo + hi) / 2)   # exact in fp32
    got = orc.e4m3_encode(mids).astype(np.int64)
    c = NONNEG[:-1].astype(np.int64)
    want = np.where(c % 2 == 0, c, c + 1)
    assert np.array_equal(got, want)
    # one fp32 ulp either side of the midpoint picks the nearer code
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(np.inf))
    assert np.array_equal(orc.e4m3_encode(below).astype(np.int64), c)
    assert np.array_equal(orc.e4m3_encode(above).astype(np.int64), c + 1)
    # negative side mirrors with the sign bit
    assert np.array_equal(orc.e4m3_encode(-mids).astype(np.int64), want | 0x80)


def test_encode_matches_torch_cast_below_464(orc):
    rng = np.random.default_rng(1234)
    n = 1_000_000
    mag = np.exp2(rng.uniform(-16.0, np.log2(463.99), size=n))
    v = (mag * rng.choice([-1.0, 1.0], size=n)).astype(np.float32)
    v = v[np.abs(v) < 464]
    v = np.concatenate([v, rng.standard_normal(100_000).astype(np.float32),
                        np.float32([0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 448.0, 463.9, -463.9])])
    assert np.array_equal(orc.e4m3_encode(v), torch_encode(v))


def test_saturates_where_torch_gives_nan(orc):
    """The pages' cast (float8_e4m3fn) turns |v| > 464 into NaN (464 itself is a
    tie that rounds to 448); the method's reading saturates every |v| >= 448,
    infinities included, to +-448."""
    assert torch_encode(np.float32([464.0]))[0] == 0x7E
    big = np.float32([464.00003, 470.0, 1e6, 3.4e38, np.inf])
    assert np.all(torch_encode(big) == 0x7F)
    assert np.all(orc.e4m3_encode(big) == 0x7E)
    assert np.all(orc.e4m3_encode(-big) == 0xFE)
    assert np.all(orc.e4m3_encode(np.float32([448.0, 450.0, 463.99])) == 0x7E)


def test_encode_is_nearest_by_brute_force(orc):
    """For every input the chosen code is at minimum distance from it."""
    rng = np.random.default_rng(7)
    v = (np.exp2(rng.uniform(-12, 9, size=20000)) * rng.choice([-1, 1], size=20000)).astype(np.float32)
    codes = orc.e4m3_encode(v)
    dec_all = orc.e4m3_decode(NONNEG)
    a = np.minimum(np.abs(v.astype(np.float64)), 448.0)
    best = np.min(np.abs(a[:, None] - dec_all[None, :]), axis=1)
    got = np.abs(orc.e4m3_decode(codes & 0x7F) - a)
    assert np.array_equal(got, best)
    assert np.array_equal(codes >> 7, np.signbit(v).astype(np.uint8))


def test_small_values_and_signed_zero(orc):
    e = orc.e4m3_encode
    assert e(np.float32(-0.0)) == 0x80 and e(np.float32(0.0)) == 0x00
    assert e(np.float32(-1e-9)) == 0x80
    assert e(np.float32(2.0 ** -10)) == 0x00        # tie between 0 and 2^-9 -> even (0)
    assert e(np.float32(3 * 2.0 ** -10)) == 0x02    # tie between 1 and 2 (x 2^-9) -> even
    assert e(np.float32(2.0 ** -10 * 1.0001)) == 0x01


@pytest.mark.parametrize("v", [np.nan, -np.nan])
def test_nan_encodes_to_nan(orc, v):
    c = int(orc.e4m3_encode(np.float32([v]))[0])
    assert c & 0x7F == 0x7F

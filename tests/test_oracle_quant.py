"""Pins for the oracle's online 1x128 / 128x128 quantizers (CPU only).

Pins: closed forms (exactly representable scaled inputs), invariants that
any correct implementation of scale = amax/448 with round-to-nearest E4M3
must satisfy (amax element -> +-448, power-of-two scale invariance, sign
symmetry, zero tiles, dequantization error bound), a library cross-check of
the per-element quotient (fp64 quotient rounded to fp32 -- exact division by
the double-rounding theorem for p' >= 2p + 2 -- then PyTorch's cast), and
relations between the two quantizers.
"""
import numpy as np
import pytest
import torch

from synth import normal, set_outliers, scale_outliers


def bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def rand_act(M, K, seed, dtype=torch.bfloat16, outliers=True):
    x = normal((M, K), 1.0, seed, "cpu", dtype)
    if outliers:
        scale_outliers(x, 1e-2, 100.0, seed + 1)
    return x


def as_np(t):
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.contiguous().numpy()


def values(arr):
    return bf16_to_f32(arr) if arr.dtype == np.uint16 else arr


# ----------------------------------------------------------------------------
# activation quantizer
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_act_amax_element_maps_to_448(orc, dtype):
    x = as_np(rand_act(64, 512, 11, dtype))
    q, sa = orc.quantize_act_1x128(x)
    v = values(x)
    for m in range(v.shape[0]):
        for kb in range(v.shape[1] // 128):
            tile = v[m, kb * 128:(kb + 1) * 128]
            qt = q[m, kb * 128:(kb + 1) * 128]
            amax = np.max(np.abs(tile))
            hit = np.abs(tile) == amax
            assert np.all(qt[hit] == np.where(tile[hit] > 0, 0x7E, 0xFE))
            assert np.all((qt[~hit] & 0x7F) < 0x7E + 1)


def test_act_scale_is_fp32_division_by_448(orc):
    x = as_np(rand_act(32, 384, 21))
    q, sa = orc.quantize_act_1x128(x)
    v = values(x).reshape(32, 3, 128)
    amax = np.max(np.abs(v), axis=2).astype(np.float32)
    assert np.array_equal(sa, amax / np.float32(448.0))


def test_act_codes_match_exact_quotient_then_torch_cast(orc):
    """q = cast(RN_fp32(x / s)): fp64 division rounded once to fp32 is the
    correctly rounded fp32 quotient; PyTorch's cast agrees with E4M3 RNE for
    |v| < 464; since s = fl(amax/448) may round down, a quotient can reach
    448 (1 + 2^-23) but never 464."""
    x = as_np(rand_act(48, 640, 31, torch.float32))
    q, sa = orc.quantize_act_1x128(x)
    s = np.repeat(sa, 128, axis=1).astype(np.float64)
    quot = (x.astype(np.float64) / s).astype(np.float32)
    assert np.max(np.abs(quot)) <= 448.0 * (1 + 2.0 ** -22)
    ref = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


@pytest.mark.parametrize("j", [-20, -3, 1, 7, 30])
def test_act_power_of_two_scale_invariance(orc, j):
    x = rand_act(16, 256, 41, torch.float32).numpy()
    q0, s0 = orc.quantize_act_1x128(x)
    q1, s1 = orc.quantize_act_1x128((x * np.float32(2.0 ** j)).astype(np.float32))
    assert np.array_equal(q0, q1)
    assert np.array_equal(s1, (s0 * np.float32(2.0 ** j)).astype(np.float32))


def test_act_sign_symmetry(orc):
    x = rand_act(16, 256, 51, torch.float32).numpy()
    q0, s0 = orc.quantize_act_1x128(x)
    q1, s1 = orc.quantize_act_1x128(-x)
    assert np.array_equal(s0, s1)
    assert np.array_equal(q1, q0 ^ 0x80)


def test_act_closed_form_exact_codes(orc):
    """x = 2^j * dec(c) with 448 present in every tile: then amax = 448 * 2^j,
    s = 2^j exactly, x / s = dec(c) exactly, so the codes come back unchanged."""
    rng = np.random.default_rng(5)
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    codes = rng.choice(fin, size=(8, 384)).astype(np.uint8)
    codes[:, ::128] = 0x7E                    # one +448 per tile
    codes[3, 130] = 0xFE                      # a -448 too
    dec = orc.e4m3_decode(codes)
    for j in (-6, 0, 5):
        x = (dec * 2.0 ** j).astype(np.float32)
        q, sa = orc.quantize_act_1x128(x)
        assert np.array_equal(q, codes)
        assert np.all(sa == np.float32(2.0 ** j))


def test_act_zero_tile_scale_one(orc):
    x = np.zeros((2, 256), dtype=np.float32)
    x[0, 5] = -0.0
    x[1, 128:] = np.float32(3.0)
    q, sa = orc.quantize_act_1x128(x)
    assert sa[0, 0] == 1.0 and sa[0, 1] == 1.0 and sa[1, 0] == 1.0
    assert np.all(q[0] == np.where(np.signbit(x[0]), 0x80, 0x00))
    assert sa[1, 1] == np.float32(3.0) / np.float32(448.0) and np.all(q[1, 128:] == 0x7E)


def test_act_underflowing_scale_reads_as_one(orc):
    """fp32 amax below 448 * 2^-150 makes amax/448 round to 0; the oracle reads
    "scale = 1 when amax = 0" as "scale = 1 when amax/448 = 0"."""
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 7] = np.float32(1e-44)               # subnormal, / 448 underflows to 0
    q, sa = orc.quantize_act_1x128(x)
    assert np.float32(1e-44) / np.float32(448.0) == 0.0
    assert sa[0, 0] == 1.0 and q[0, 7] == 0x00


def test_act_dequant_error_bound(orc):
    """|x - s dec(q)| <= max(2^-4 |x|, 2^-10 s) (half an E4M3 ulp, normal /
    subnormal range), up to the fp32 rounding of the quotient."""
    x = as_np(rand_act(64, 512, 61))
    q, sa = orc.quantize_act_1x128(x)
    v = values(x).astype(np.float64)
    dq = orc.dequantize(q, sa, 1, 128)
    s = np.repeat(sa, 128, axis=1).astype(np.float64)
    bound = np.maximum(2.0 ** -4 * np.abs(v), 2.0 ** -10 * s) * (1 + 2.0 ** -20)
    assert np.all(np.abs(v - dq) <= bound)


def test_act_tiles_are_independent_and_128_wide(orc):
    """Changing one element only changes its own 1x128 tile."""
    x = rand_act(4, 512, 71, torch.float32).numpy()
    q0, s0 = orc.quantize_act_1x128(x)
    y = x.copy()
    y[2, 300] = np.float32(1e4)               # tile (2, 2)
    q1, s1 = orc.quantize_act_1x128(y)
    diff_s = np.argwhere(s0 != s1)
    assert diff_s.tolist() == [[2, 2]]
    rows, cols = np.nonzero(q0 != q1)
    assert set(rows) == {2} and cols.min() >= 256 and cols.max() < 384


def test_act_tail_tile_equals_zero_padded_tile(orc):
    x = rand_act(6, 200, 81, torch.float32).numpy()
    q, sa = orc.quantize_act_1x128(x)
    xp = np.zeros((6, 256), dtype=np.float32)
    xp[:, :200] = x
    qp, sap = orc.quantize_act_1x128(xp)
    assert np.array_equal(sa, sap) and np.array_equal(q, qp[:, :200])


def test_act_bf16_matches_fp32_of_same_values(orc):
    xb = rand_act(8, 256, 91)
    q0, s0 = orc.quantize_act_1x128(bf16_bits(xb))
    q1, s1 = orc.quantize_act_1x128(xb.float().numpy())
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)


# ----------------------------------------------------------------------------
# weight quantizer
# ----------------------------------------------------------------------------

# ----------------------------------------------------------------------------
# 128x1 activation quantizer (1x128 tiles of X^T, for the weight gradient)
# ----------------------------------------------------------------------------

def test_act_128x1_scale_is_column_amax_over_448(orc):
    """st[k, mb] = fl32(max over rows 128 mb .. 128 mb + 127 of |x[m, k]| / 448),
    computed here along the columns of x directly."""
    x = as_np(rand_act(384, 256, 61))
    qt, st = orc.quantize_act_128x1(x)
    assert qt.shape == (256, 384) and st.shape == (256, 3)
    amax = np.max(np.abs(values(x).reshape(3, 128, 256)), axis=1).astype(np.float32)   # [mb, k]
    assert np.array_equal(st, (amax / np.float32(448.0)).T)


def test_act_128x1_codes_exact_quotient_then_torch_cast(orc):
    """qt[k, m] = cast(RN_fp32(x[m, k] / st[k, m / 128])), with the quotient
    from fp64 division and PyTorch's E4M3 cast; a column's largest element
    maps to +-448."""
    x = as_np(rand_act(256, 384, 71))
    qt, st = orc.quantize_act_128x1(x)
    v = values(x).astype(np.float64)                       # [m, k]
    s = np.repeat(st.T, 128, axis=0).astype(np.float64)    # [m, k]
    quot = (v / s).astype(np.float32)
    ref = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(qt, ref.T)
    blocks = np.abs(values(x)).reshape(2, 128, 384)
    top = blocks == blocks.max(axis=1, keepdims=True)
    codes = qt.T.reshape(2, 128, 384)
    assert np.all((codes[top] & 0x7F) == 0x7E)


def rand_weight(K, N, seed, dtype=torch.bfloat16):
    w = normal((K, N), 0.02, seed, "cpu", dtype)
    set_outliers(w, 1e-3, 1.0, seed + 1, seed + 2)
    return w


def test_weight_block_scale_is_max_of_row_tile_scales(orc):
    """amax over a 128x128 block is the max of its 128 row-tile amaxes, and
    x -> fl(x/448) is monotone, so sb[kb,nb] = max over the block's rows of
    the 1x128 scales of W's rows (no row here is all zero)."""
    w = as_np(rand_weight(256, 384, 101))
    qw, sb = orc.quantize_weight_128x128(w)
    qa, sa = orc.quantize_act_1x128(w)          # tiles along N of each row k
    assert np.array_equal(sb, sa.reshape(2, 128, 3).max(axis=1))


def test_weight_amax_element_maps_to_448(orc):
    w = rand_weight(256, 256, 111, torch.float32).numpy()
    q, sb = orc.quantize_weight_128x128(w)
    for kb in range(2):
        for nb in range(2):
            blk = w[kb * 128:(kb + 1) * 128, nb * 128:(nb + 1) * 128]
            qb = q[kb * 128:(kb + 1) * 128, nb * 128:(nb + 1) * 128]
            amax = np.max(np.abs(blk))
            hit = np.abs(blk) == amax
            assert np.all(qb[hit] == np.where(blk[hit] > 0, 0x7E, 0xFE))
            assert sb[kb, nb] == np.float32(amax) / np.float32(448.0)


def test_weight_transposed_output_is_transpose(orc):
    w = as_np(rand_weight(384, 256, 121))
    q0, s0 = orc.quantize_weight_128x128(w, transpose_out=False)
    q1, s1 = orc.quantize_weight_128x128(w, transpose_out=True)
    assert q1.shape == (256, 384)
    assert np.array_equal(q1, q0.T) and np.array_equal(s0, s1)


def test_weight_closed_form_and_symmetries(orc):
    rng = np.random.default_rng(9)
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    codes = rng.choice(fin, size=(256, 256)).astype(np.uint8)
    codes[0, 0] = codes[0, 128] = codes[200, 10] = codes[131, 250] = 0x7E
    x = (orc.e4m3_decode(codes) * 2.0 ** -3).astype(np.float32)
    q, sb = orc.quantize_weight_128x128(x)
    assert np.array_equal(q, codes) and np.all(sb == np.float32(0.125))
    qn, sbn = orc.quantize_weight_128x128(-x)
    assert np.array_equal(qn, q ^ 0x80) and np.array_equal(sbn, sb)


def test_weight_dequant_error_bound(orc):
    w = as_np(rand_weight(256, 384, 131))
    q, sb = orc.quantize_weight_128x128(w)
    v = values(w).astype(np.float64)
    dq = orc.dequantize(q, sb, 128, 128)
    s = np.repeat(np.repeat(sb, 128, 0), 128, 1).astype(np.float64)
    bound = np.maximum(2.0 ** -4 * np.abs(v), 2.0 ** -10 * s) * (1 + 2.0 ** -20)
    assert np.all(np.abs(v - dq) <= bound)


def test_weight_partial_blocks(orc):
    w = rand_weight(200, 136, 141, torch.float32).numpy()
    q, sb = orc.quantize_weight_128x128(w)
    wp = np.zeros((256, 256), dtype=np.float32)
    wp[:200, :136] = w
    qp, sbp = orc.quantize_weight_128x128(wp)
    assert sb.shape == (2, 2)
    assert np.array_equal(sb, sbp) and np.array_equal(q, qp[:200, :136])

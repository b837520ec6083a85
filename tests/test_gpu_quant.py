"""GPU parity of the online quantization kernels against the oracle:
codes and scales bit-identical, called through the C ABI."""
import numpy as np
import pytest
import torch

import synth
from _util import assert_codes_equal, assert_scales_equal, np_u8, to_oracle

pytestmark = pytest.mark.gpu


def act(M, K, dtype, seed, std=1.0, outliers=1e-2):
    return synth.act_input(M, K, std, outliers, 100.0, 7, "cpu", dtype, tensor_id=seed)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (130, 384), (257, 1024), (1000, 7168),
                                 (77, 2048)])
def test_act_quant_bit_exact(cuda_lib, orc, M, K, dtype):
    x = act(M, K, dtype, M + K)
    q, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qo, sao = orc.quantize_act_1x128(to_oracle(x))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa.cpu().numpy(), sao)


def test_act_quant_strided_layouts(cuda_lib, orc):
    """ldx > K, ldq > K and column-major ([K/128, M]) scales."""
    M, K = 200, 512
    big = act(M, 768, torch.bfloat16, 3).cuda()
    x = big[:, 128:128 + K]
    qbuf = torch.full((M, 640), 0xAB, dtype=torch.uint8, device="cuda")
    q = qbuf[:, 64:64 + K]
    sa_t = torch.full((K // 128, M), -1.0, device="cuda")
    cuda_lib.fp8_quantize_act_1x128(x, q=q, sa=sa_t.t())
    qo, sao = orc.quantize_act_1x128(to_oracle(x))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa_t.t().cpu().numpy(), sao)
    untouched = np_u8(qbuf)
    assert np.all(untouched[:, :64] == 0xAB) and np.all(untouched[:, 64 + K:] == 0xAB)


@pytest.mark.parametrize("M,K", [(1, 128), (31, 256), (33, 384), (1000, 1024)])
def test_act_quant_row_and_stream_paths_agree(cuda_lib, orc, M, K):
    """bf16 codes written with 32-byte alignment take the one-row-per-thread
    kernel; codes at a 16-byte offset (ldq a multiple of 16 only) take the
    streamed 128x128-box kernel.  Both equal the oracle bit for bit."""
    x = act(M, K, torch.bfloat16, 5 * M + K).cuda()
    qo, sao = orc.quantize_act_1x128(to_oracle(x))
    for offset, ld in ((0, K), (16, K + 16)):
        qbuf = torch.full((M, ld + offset), 0xCD, dtype=torch.uint8, device="cuda")
        q = qbuf[:, offset:offset + K]
        _, sa = cuda_lib.fp8_quantize_act_1x128(x, q=q)
        assert_codes_equal(np_u8(q), qo)
        assert_scales_equal(sa.cpu().numpy(), sao)
        rest = np_u8(qbuf)
        assert np.all(rest[:, :offset] == 0xCD) and np.all(rest[:, offset + K:] == 0xCD)


def test_act_quant_special_values(cuda_lib, orc):
    g = torch.Generator().manual_seed(123)
    x = torch.randn(8, 512, generator=g) * 3
    x[0, :128] = 0.0                               # zero tile -> scale 1
    x[0, 128:256] = -0.0
    x[1, :128] = 1e-42                             # subnormal fp32 amax: amax/448 underflows
    x[1, 5] = -1e-42
    x[2, :128] = torch.tensor(2.0 ** -130)         # subnormal scale, no underflow
    x[3, 130] = 3.0e38                             # huge amax
    x[4, 256:384] = 448.0                          # all at the maximum
    x[5, 384:] = torch.linspace(-1e-3, 1e-3, 128)
    for dtype in (torch.float32, torch.bfloat16):
        xd = x.to(dtype)
        q, sa = cuda_lib.fp8_quantize_act_1x128(xd.cuda())
        qo, sao = orc.quantize_act_1x128(to_oracle(xd))
        assert_codes_equal(np_u8(q), qo)
        assert_scales_equal(sa.cpu().numpy(), sao)


def test_cvt_rounding_matches_oracle_encoder(cuda_lib, orc):
    """Every tile holds 448 so its scale is exactly 1 and code = E4M3(x):
    checks the hardware conversion against the oracle's nearest-value
    encoder on random values and on every midpoint +-1 ulp."""
    dec = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((dec[:-1] + dec[1:]) / 2).astype(np.float32)
    special = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                              np.nextafter(mids, np.float32(np.inf)), dec.astype(np.float32)])
    special = np.concatenate([special, -special])
    rng = np.random.default_rng(42)
    rand = (np.exp2(rng.uniform(-14, np.log2(448), 2_000_000)) *
            rng.choice([-1, 1], 2_000_000)).astype(np.float32)
    vals = np.concatenate([special, rand])
    n_rows = (len(vals) + 126) // 127
    tiles = np.zeros((n_rows, 128), dtype=np.float32)
    tiles[:, 0] = 448.0
    tiles[:, 1:].flat[:len(vals)] = vals
    x = torch.from_numpy(tiles)
    q, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    assert torch.all(sa == 1.0)
    assert_codes_equal(np_u8(q), orc.e4m3_encode(tiles))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quotients_at_rounding_midpoints(cuda_lib, orc, dtype):
    """Tiles with non-power-of-two scales whose elements are (a few ulps
    around) E4M3 midpoints times the scale: x / s lands within a few fp32
    ulps of a rounding boundary, where a reciprocal-based quotient could
    round differently from the IEEE quotient."""
    rng = np.random.default_rng(7)
    dec = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (dec[:-1] + dec[1:]) / 2
    rows = 4096
    tiles = np.empty((rows, 128), dtype=np.float32)
    amax = (rng.uniform(0.5, 2.0, rows) * np.exp2(rng.integers(-30, 30, rows))).astype(np.float32)
    if dtype == torch.bfloat16:    # amax itself must survive the bf16 rounding
        amax = torch.from_numpy(amax).bfloat16().float().numpy()
    s = (amax / np.float32(448.0)).astype(np.float32)
    m = rng.choice(mids, size=(rows, 127)) * rng.choice([-1.0, 1.0], size=(rows, 127))
    x = (m * s[:, None].astype(np.float64)).astype(np.float32)
    jitter = rng.integers(-3, 4, size=x.shape).astype(np.int32)
    x = (x.view(np.int32) + jitter).view(np.float32)
    tiles[:, 0] = amax
    tiles[:, 1:] = np.clip(x, -amax[:, None], amax[:, None])
    xt = torch.from_numpy(tiles).to(dtype)
    q, sa = cuda_lib.fp8_quantize_act_1x128(xt.cuda())
    qo, sao = orc.quantize_act_1x128(to_oracle(xt))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa.cpu().numpy(), sao)
    w = xt[:1024].reshape(128, 1024)                # same values through the weight kernel
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=True)
    qwo, swo = orc.quantize_weight_128x128(to_oracle(w), transpose_out=True)
    assert_codes_equal(np_u8(qw), qwo)
    assert_scales_equal(sw.cpu().numpy(), swo)


def test_act_quant_nan_element_smoke(cuda_lib, orc):
    """Out of contract: a NaN element is skipped by amax and encodes to NaN
    (fp32 and bf16 inputs, both activation kernels)."""
    gen = torch.Generator().manual_seed(321)
    x = torch.randn(2, 256, generator=gen)
    x[1, 17] = float("nan")
    for dtype in (torch.float32, torch.bfloat16):
        xd = x.to(dtype)
        q, sa = cuda_lib.fp8_quantize_act_1x128(xd.cuda())
        qo, sao = orc.quantize_act_1x128(to_oracle(xd))
        g = np_u8(q)
        assert (g[1, 17] & 0x7F) == 0x7F
        g[1, 17] = qo[1, 17]
        assert_codes_equal(g, qo)
        assert_scales_equal(sa.cpu().numpy(), sao)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("K,N", [(128, 128), (256, 384), (384, 256), (1024, 2048)])
@pytest.mark.parametrize("transpose", [False, True])
def test_weight_quant_bit_exact(cuda_lib, orc, K, N, dtype, transpose):
    w = synth.normal((K, N), 0.02, 1000 + K + N, "cpu", dtype)
    synth.scale_outliers(w, 1e-3, 100.0, 77)
    q, sb = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=transpose)
    qo, sbo = orc.quantize_weight_128x128(to_oracle(w), transpose_out=transpose)
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sb.cpu().numpy(), sbo)


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("K,N", [(128, 128), (384, 640), (1024, 256)])
def test_weight_quant_row_and_stream_paths_agree(cuda_lib, orc, K, N, transpose):
    """bf16 codes written with 32-byte alignment take the one-block-row-per-
    thread kernel; codes at a 16-byte offset take the streamed box kernel.
    Both equal the oracle bit for bit and write nothing outside q."""
    w = synth.normal((K, N), 0.02, 2000 + K + N, "cpu", torch.bfloat16)
    synth.scale_outliers(w, 1e-3, 100.0, 78)
    qo, sbo = orc.quantize_weight_128x128(to_oracle(w), transpose_out=transpose)
    rows, cols = (N, K) if transpose else (K, N)
    for offset, ld in ((0, cols), (16, cols + 16)):
        qbuf = torch.full((rows, ld + offset), 0xCD, dtype=torch.uint8, device="cuda")
        q = qbuf[:, offset:offset + cols]
        _, sb = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=transpose, q=q)
        assert_codes_equal(np_u8(q), qo)
        assert_scales_equal(sb.cpu().numpy(), sbo)
        rest = np_u8(qbuf)
        assert np.all(rest[:, :offset] == 0xCD) and np.all(rest[:, offset + cols:] == 0xCD)


def test_weight_quant_zero_and_strided(cuda_lib, orc):
    K, N = 256, 384
    big = synth.normal((K, 512), 0.02, 5, "cpu", torch.float32)
    big[:128, 64:192] = 0.0                        # block (0, 0) of the slice below
    w = big[:, 64:64 + N].cuda()
    sbT = torch.zeros((N // 128, K // 128), device="cuda")
    for transpose in (False, True):
        q, _ = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=transpose, sb=sbT.t())
        qo, sbo = orc.quantize_weight_128x128(to_oracle(w), transpose_out=transpose)
        assert_codes_equal(np_u8(q), qo)
        assert_scales_equal(sbT.t().cpu().numpy(), sbo)
        assert sbo[0, 0] == 1.0


# ---------------------------------------------------------------- full sizes

def _sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, n)]))


@pytest.mark.slow
def test_quant_bandwidth_workload_sampled(cuda_lib, orc):
    """Activation [8192x7168] and weight [7168x18432] bf16, N(0, 0.02) with
    0.1% outliers x100, quantized as the bench does; sampled rows and
    blocks compared bit for bit with the oracle."""
    x, w = synth.quant_inputs("cuda")
    q, sa = cuda_lib.fp8_quantize_act_1x128(x)
    qw, sb = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
    torch.cuda.synchronize()
    rows = _sample_rows(8192, 96, 1)
    qo, sao = orc.quantize_act_1x128(to_oracle(x[torch.from_numpy(rows).cuda()]))
    assert_codes_equal(np_u8(q[torch.from_numpy(rows).cuda()]), qo)
    assert_scales_equal(sa[torch.from_numpy(rows).cuda()].cpu().numpy(), sao)
    rng = np.random.default_rng(2)
    for kb, nb in list(zip(rng.integers(0, 56, 24), rng.integers(0, 144, 24))) + [(55, 143)]:
        blk = w[kb * 128:(kb + 1) * 128, nb * 128:(nb + 1) * 128]
        qo, sbo = orc.quantize_weight_128x128(to_oracle(blk), transpose_out=True)
        assert_codes_equal(np_u8(qw[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]), qo)
        assert_scales_equal(sb[kb:kb + 1, nb:nb + 1].cpu().numpy(), sbo)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)) \
        .view(torch.bfloat16)


def test_act_bf16_quotient_sweep(cuda_lib, orc):
    """Every bf16 (amax, x) mantissa pair over 21 exponent steps, at amax
    exponents that put the scale near the bottom of the fast path, just
    below it, and across the range: codes of the fast quotient equal those
    of IEEE division."""
    from _util import bf16_quotient_sweep
    rows = []
    for lst in bf16_quotient_sweep():
        amax, xs = lst[0], lst[1:]
        for i in range(0, len(xs), 127):
            row = np.zeros(128, dtype=np.uint16)
            row[0] = amax
            chunk = xs[i:i + 127]
            row[1:1 + len(chunk)] = chunk
            rows.append(row)
    bits = np.stack(rows)
    x = _bf16(bits)
    q, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qo, sao = orc.quantize_act_1x128(bits)
    assert_scales_equal(sa.cpu().numpy(), sao)
    assert_codes_equal(np_u8(q), qo)


@pytest.mark.parametrize("transpose_out", [False, True])
def test_weight_bf16_quotient_sweep(cuda_lib, orc, transpose_out):
    """The same sweep through the 128x128 weight quantizer: one amax (and
    all its x) per block."""
    from _util import bf16_quotient_sweep
    lists = bf16_quotient_sweep()
    nb = len(lists)                       # 896 blocks: 28 x 32
    kb_n, nb_n = 28, 32
    assert nb == kb_n * nb_n
    w = np.zeros((kb_n * 128, nb_n * 128), dtype=np.uint16)
    for i, lst in enumerate(lists):
        blk = np.zeros(128 * 128, dtype=np.uint16)
        blk[:len(lst)] = lst
        r, c = divmod(i, nb_n)
        w[r * 128:(r + 1) * 128, c * 128:(c + 1) * 128] = blk.reshape(128, 128)
    q, sb = cuda_lib.fp8_quantize_weight_128x128(_bf16(w).cuda(), transpose_out=transpose_out)
    qo, sbo = orc.quantize_weight_128x128(w, transpose_out=transpose_out)
    assert_scales_equal(sb.cpu().numpy(), sbo)
    assert_codes_equal(np_u8(q), qo)

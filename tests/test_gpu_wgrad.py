"""GPU parity of the weight-gradient path dW = X^T dY: the 128x1 activation
quantizer (1x128 tiles of X^T and dY^T along the tokens, codes and scales
bit-identical to the oracle) and the block-scaled GEMM with per-column B
scales (within the GEMM bound of the oracle's fp64 reference), called
through the C ABI."""
import numpy as np
import pytest
import torch

import synth
from _util import (assert_codes_equal, assert_gemm_within_bound, assert_scales_equal, np_f32,
                   np_u8, to_oracle)

pytestmark = pytest.mark.gpu


def act(M, K, seed, std=1.0, outliers=1e-2):
    return synth.act_input(M, K, std, outliers, 100.0, 9, "cpu", torch.bfloat16, tensor_id=seed)


def cuda_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)) \
        .view(torch.bfloat16)


# ------------------------------------------------------------ 128x1 quantizer

@pytest.mark.parametrize("M,K", [(128, 128), (256, 384), (640, 2048), (2048, 4096),
                                 (4096, 1152)])
def test_act_128x1_bit_exact(cuda_lib, orc, M, K):
    """Tiles of one box, several boxes, and more boxes than the grid's two
    groups of CTAs cover in one pass."""
    x = act(M, K, M + K)
    qt, st = cuda_lib.fp8_quantize_act_128x1(x.cuda())
    qo, so = orc.quantize_act_128x1(to_oracle(x))
    assert qt.shape == (K, M) and st.shape == (K, M // 128)
    assert_codes_equal(np_u8(qt), qo)
    assert_scales_equal(st.cpu().numpy(), so)


def test_act_128x1_kb_major_scales_and_strides(cuda_lib, orc):
    """ldx > K, ldq > M, scales written [M/128, K]; bytes outside the
    output rows are left alone."""
    M, K = 384, 256
    big = act(M, 512, 5).cuda()
    x = big[:, 128:128 + K]
    qbuf = torch.full((K, M + 64), 0xAB, dtype=torch.uint8, device="cuda")
    qt = qbuf[:, 32:32 + M]
    qt, st = cuda_lib.fp8_quantize_act_128x1(x, qt=qt, st_kb_major=True)
    qo, so = orc.quantize_act_128x1(to_oracle(x))
    assert st.shape == (M // 128, K)
    assert_codes_equal(np_u8(qt), qo)
    assert_scales_equal(st.t().cpu().numpy(), so)
    untouched = np_u8(qbuf)
    assert np.all(untouched[:, :32] == 0xAB) and np.all(untouched[:, 32 + M:] == 0xAB)


@pytest.mark.parametrize("M,K", [(128, 128), (384, 640), (1024, 256)])
def test_act_128x1_column_and_stream_paths_agree(cuda_lib, orc, M, K):
    """Codes written with 32-byte alignment take the column-pair kernel,
    codes at a 16-byte offset the streamed box kernel: both equal the oracle
    (codes and scales, both scale layouts) and write nothing outside qt."""
    x = act(M, K, 3 * M + K).cuda()
    qo, so = orc.quantize_act_128x1(to_oracle(x))
    for offset, kb_major in ((0, False), (16, False), (0, True), (16, True)):
        qbuf = torch.full((K, M + 16 + offset), 0xAB, dtype=torch.uint8, device="cuda")
        qt = qbuf[:, offset:offset + M]
        _, st = cuda_lib.fp8_quantize_act_128x1(x, qt=qt, st_kb_major=kb_major)
        assert_codes_equal(np_u8(qt), qo)
        assert_scales_equal((st.t() if kb_major else st).cpu().numpy(), so)
        rest = np_u8(qbuf)
        assert np.all(rest[:, :offset] == 0xAB) and np.all(rest[:, offset + M:] == 0xAB)


def test_act_128x1_special_values(cuda_lib, orc):
    """Zero and -0 columns (scale 1), subnormal amax (scale off the fast
    quotient's range: IEEE division), huge amax, a column at 448, NaN
    elements (out of contract: skipped by amax, NaN codes)."""
    x = torch.randn(256, 512, generator=torch.Generator().manual_seed(66)) * 3
    x[:128, 0] = 0.0
    x[:128, 1] = -0.0
    x[128:, 2] = 1e-39
    x[130, 2] = -2e-39
    x[:, 3] = torch.linspace(-1e-3, 1e-3, 256)
    x[7, 4] = 3.0e38
    x[128:, 5] = 448.0
    x[3, 6] = float("nan")
    x[200:, 7] = float("nan")
    xb = x.to(torch.bfloat16)
    qt, st = cuda_lib.fp8_quantize_act_128x1(xb.cuda())
    qo, so = orc.quantize_act_128x1(to_oracle(xb))
    assert_scales_equal(st.cpu().numpy(), so)
    g = np_u8(qt)
    nan = np.isnan(x.numpy().T)
    assert np.all((g[nan] & 0x7F) == 0x7F)       # NaN code; its sign is not specified
    g[nan] = qo[nan]
    assert_codes_equal(g, qo)


def test_act_128x1_bf16_quotient_sweep(cuda_lib, orc):
    """Every bf16 (amax, x) mantissa pair of the quotient sweep, laid out
    down the columns: column tiles carry the sweep's amax first."""
    from _util import bf16_quotient_sweep
    cols = []
    for lst in bf16_quotient_sweep():
        amax, xs = lst[0], lst[1:]
        for i in range(0, len(xs), 127):
            col = np.zeros(128, dtype=np.uint16)
            col[0] = amax
            chunk = xs[i:i + 127]
            col[1:1 + len(chunk)] = chunk
            cols.append(col)
    while len(cols) % 128:
        cols.append(np.zeros(128, dtype=np.uint16))
    bits = np.stack(cols, axis=1)                   # [128, R]
    qt, st = cuda_lib.fp8_quantize_act_128x1(_bf16(bits).cuda())
    qo, so = orc.quantize_act_128x1(bits)
    assert_scales_equal(st.cpu().numpy(), so)
    assert_codes_equal(np_u8(qt), qo)


# ------------------------------------------------------ column-scale GEMM

def oracle_operands(orc, M, N, K, seed):
    """A = X^T and B = dY^T quantized along the contraction (K, the tokens)."""
    x = synth.normal((K, M), 1.0, seed, "cpu", torch.bfloat16)
    synth.scale_outliers(x, 1e-2, 100.0, seed + 1)
    dy = synth.normal((K, N), 1e-3, seed + 2, "cpu", torch.bfloat16)
    qa, sa = orc.quantize_act_128x1(to_oracle(x))        # [M, K], [M, K/128]
    qb, sb_cols = orc.quantize_act_128x1(to_oracle(dy))  # [N, K], [N, K/128]
    return qa, sa, qb, sb_cols


def colscale(cuda_lib, qa, sa, qb, sb_cols, out_dtype):
    return cuda_lib.fp8_blockscaled_gemm_colscale(
        cuda_u8(qa), torch.from_numpy(sa).cuda(), cuda_u8(qb),
        torch.from_numpy(np.ascontiguousarray(sb_cols.T)).cuda(), out_dtype=out_dtype)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (128, 256, 128), (127, 256, 256),
                                   (300, 384, 512), (256, 512, 2048), (1000, 768, 1024)])
def test_colscale_gemm_matches_oracle(cuda_lib, orc, M, N, K, out_dtype):
    qa, sa, qb, sbc = oracle_operands(orc, M, N, K, 7 * M + N + K)
    c = colscale(cuda_lib, qa, sa, qb, sbc, out_dtype)
    C_ref, T = orc.gemm_ref_colscale(qa, sa, qb, sbc)
    assert_gemm_within_bound(np_f32(c), C_ref, T, out_dtype)


def test_colscale_gemm_exact_small_integers(cuda_lib, orc):
    """Small-integer codes with power-of-two scales that differ per column of
    B and per chunk: every sum is exact, so C must equal the oracle bit for
    bit (a scale read for the wrong column or chunk shows)."""
    rng = np.random.default_rng(12)
    M, N, K = 384, 512, 1024
    ints = np.array([-4, -3, -2, -1, 0, 1, 2, 3, 4], dtype=np.float32)
    codes = orc.e4m3_encode(ints)
    qa = rng.choice(codes, size=(M, K)).astype(np.uint8)
    qb = rng.choice(codes, size=(N, K)).astype(np.uint8)
    sa = np.exp2(rng.integers(-3, 4, size=(M, K // 128))).astype(np.float32)
    sbc = np.exp2(rng.integers(-3, 4, size=(N, K // 128))).astype(np.float32)
    c = colscale(cuda_lib, qa, sa, qb, sbc, torch.float32)
    C_ref, _ = orc.gemm_ref_colscale(qa, sa, qb, sbc)
    assert np.array_equal(np_f32(c).astype(np.float64), C_ref)


def test_colscale_gemm_strided_and_degenerate(cuda_lib, orc):
    """Padded sb rows (sb_stride_kb > N), a strided C, and K == 0 (C = 0)."""
    M, N, K = 200, 256, 384
    qa, sa, qb, sbc = oracle_operands(orc, M, N, K, 77)
    sb_pad = torch.full((K // 128, N + 12), float("nan"), device="cuda")
    sb_pad[:, :N] = torch.from_numpy(np.ascontiguousarray(sbc.T)).cuda()
    cbuf = torch.full((M, N + 64), 7.0, dtype=torch.float32, device="cuda")
    c = cbuf[:, 32:32 + N]
    cuda_lib.fp8_blockscaled_gemm_colscale(cuda_u8(qa), torch.from_numpy(sa).cuda(), cuda_u8(qb),
                                           sb_pad[:, :N], c=c)
    C_ref, T = orc.gemm_ref_colscale(qa, sa, qb, sbc)
    assert_gemm_within_bound(np_f32(c), C_ref, T, torch.float32)
    rest = np_f32(cbuf)
    assert np.all(rest[:, :32] == 7.0) and np.all(rest[:, 32 + N:] == 7.0)
    z = torch.full((5, 128), 3.0, device="cuda")
    empty = torch.empty((5, 0), dtype=torch.uint8, device="cuda")
    cuda_lib.fp8_blockscaled_gemm_colscale(empty, torch.empty((5, 0), device="cuda"),
                                           torch.empty((128, 0), dtype=torch.uint8, device="cuda"),
                                           torch.empty((0, 128), device="cuda"), c=z)
    torch.cuda.synchronize()
    assert torch.all(z == 0)


def test_linear_weight_grad_end_to_end(cuda_lib, orc):
    """X bf16 [512x384], dY bf16 [512x256]: both quantized 128x1 on the GPU
    (bit-exact), dW = X^T dY in fp32 within the bound, and close to the
    unquantized product."""
    x = act(512, 384, 31)
    dy = synth.normal((512, 256), 1e-3, 33, "cpu", torch.bfloat16)
    dw = cuda_lib.linear_weight_grad(x.cuda(), dy.cuda())
    qa, sa = orc.quantize_act_128x1(to_oracle(x))
    qb, sbc = orc.quantize_act_128x1(to_oracle(dy))
    C_ref, T = orc.gemm_ref_colscale(qa, sa, qb, sbc)
    assert dw.shape == (384, 256)
    assert_gemm_within_bound(np_f32(dw), C_ref, T, torch.float32)
    E = x.double().numpy().T @ dy.double().numpy()
    rel = np.linalg.norm(np_f32(dw) - E) / np.linalg.norm(E)
    assert rel < 0.05


@pytest.mark.slow
def test_wgrad_full_size_sampled(cuda_lib, orc):
    """X bf16 [16384x7168] (N(0,1), 0.1% outliers x100), dY bf16
    [16384x18432] (N(0,1e-3), 0.1% outliers x100): 128x1 quantization of
    both and dW = X^T dY -> fp32 [7168x18432], as the bench runs it.
    Columns of X and dY are independent under 128x1 tiles, so the oracle
    quantizes only the sampled ones and checks their codes, scales and the
    dW entries they produce."""
    x, dy = synth.wgrad_inputs("cuda")
    qxt, sxt = cuda_lib.fp8_quantize_act_128x1(x)
    qdt, sdt = cuda_lib.fp8_quantize_act_128x1(dy, st_kb_major=True)
    dw = cuda_lib.fp8_blockscaled_gemm_colscale(qxt, sxt, qdt, sdt, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 7167], rng.integers(0, 7168, 14)]))
    cols = np.unique(np.concatenate([[0, 18431], rng.integers(0, 18432, 30)]))
    rows_t, cols_t = torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()
    qa_o, sa_o = orc.quantize_act_128x1(to_oracle(x[:, rows_t]))
    qb_o, sb_o = orc.quantize_act_128x1(to_oracle(dy[:, cols_t]))
    assert_codes_equal(np_u8(qxt[rows_t]), qa_o)
    assert_scales_equal(sxt[rows_t].cpu().numpy(), sa_o)
    assert_codes_equal(np_u8(qdt[cols_t]), qb_o)
    assert_scales_equal(sdt[:, cols_t].t().cpu().numpy(), sb_o)
    C_ref, T = orc.gemm_ref_colscale(qa_o, sa_o, qb_o, sb_o)
    got = np_f32(dw[rows_t][:, cols_t])
    assert_gemm_within_bound(got, C_ref, T, torch.float32)
    assert cuda_lib.fp8_get_device_error() == 0

"""GPU parity of the block-scaled FP8 GEMM (tcgen05) against the oracle's
fp64 reference, within |C - C_ref| <= 1e-3 T + 1e-6 (fp32 out), plus
4e-3 |C_ref| for bf16 out; bit-exact where the result is exactly
representable."""
import numpy as np
import pytest
import torch

import synth
from _util import (assert_codes_equal, assert_gemm_within_bound, assert_scales_equal, np_f32,
                   np_u8, to_oracle)

pytestmark = pytest.mark.gpu


def oracle_operands(orc, M, N, K, seed):
    x = synth.normal((M, K), 1.0, seed, "cpu", torch.float32)
    synth.scale_outliers(x, 1e-2, 100.0, seed + 1)
    w = synth.normal((K, N), 0.02, seed + 2, "cpu", torch.float32)
    qa, sa = orc.quantize_act_1x128(x.numpy())
    qb, sb = orc.quantize_weight_128x128(w.numpy(), transpose_out=True)
    return qa, sa, qb, sb


def cuda_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_tiny_end_to_end(cuda_lib, orc):
    """A fp32 [128x256], B fp32 [256x256] (N(0,1), 1% set to +-50): 1x128 act
    quant, 128x128 weight quant, block-scaled GEMM -> fp32 C [128x256]."""
    a, b = synth.tiny_inputs("cpu")
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a.cuda())
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(b.cuda(), transpose_out=True)
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.float32)
    qa_o, sa_o = orc.quantize_act_1x128(a.numpy())
    qb_o, sb_o = orc.quantize_weight_128x128(b.numpy(), transpose_out=True)
    assert_codes_equal(np_u8(qa), qa_o)
    assert_scales_equal(sa.cpu().numpy(), sa_o)
    assert_codes_equal(np_u8(qb), qb_o)
    assert_scales_equal(sb.cpu().numpy(), sb_o)
    C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o)
    assert_gemm_within_bound(np_f32(c), C_ref, T, torch.float32)
    E = orc.gemm_exact(a.numpy(), b.numpy())
    rel = np.linalg.norm(np_f32(c) - E) / np.linalg.norm(E)
    assert rel < 0.05


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (127, 256, 256), (128, 384, 128),
                                   (129, 256, 384), (300, 640, 1024), (256, 512, 2048),
                                   (1000, 768, 512)])
def test_gemm_matches_oracle(cuda_lib, orc, M, N, K, out_dtype):
    qa, sa, qb, sb = oracle_operands(orc, M, N, K, 10 * M + N + K)
    c = cuda_lib.fp8_blockscaled_gemm(cuda_u8(qa), torch.from_numpy(sa).cuda(), cuda_u8(qb),
                                      torch.from_numpy(sb).cuda(), out_dtype=out_dtype)
    C_ref, T = orc.gemm_ref(qa, sa, qb, sb)
    assert_gemm_within_bound(np_f32(c), C_ref, T, out_dtype)


def test_gemm_exact_small_integers(cuda_lib, orc):
    """Codes of small integers with power-of-two scales: every product, every
    chunk sum and every promoted sum is exact, so C must equal the oracle bit
    for bit (catches any indexing, scale or orientation error)."""
    rng = np.random.default_rng(11)
    M, N, K = 384, 512, 1024
    ints = np.array([-4, -3, -2, -1, 0, 1, 2, 3, 4], dtype=np.float32)
    codes = orc.e4m3_encode(ints)
    qa = rng.choice(codes, size=(M, K)).astype(np.uint8)
    qb = rng.choice(codes, size=(N, K)).astype(np.uint8)
    sa = np.exp2(rng.integers(-3, 4, size=(M, K // 128))).astype(np.float32)
    sb = np.exp2(rng.integers(-3, 4, size=(K // 128, N // 128))).astype(np.float32)
    c = cuda_lib.fp8_blockscaled_gemm(cuda_u8(qa), torch.from_numpy(sa).cuda(), cuda_u8(qb),
                                      torch.from_numpy(sb).cuda(), out_dtype=torch.float32)
    C_ref, _ = orc.gemm_ref(qa, sa, qb, sb, want_t=False)
    assert np.array_equal(np_f32(c).astype(np.float64), C_ref)


def test_gemm_dgrad_orientation(cuda_lib, orc):
    """dX = dY W^T: W quantized untransposed ([K_fwd, N_fwd]) is the K-major
    operand, its scales read [nb][kb]."""
    M, Kf, Nf = 256, 384, 512          # forward W [Kf, Nf]; dgrad contracts over Nf
    dy = synth.normal((M, Nf), 1e-3, 91, "cpu", torch.bfloat16)
    synth.scale_outliers(dy, 1e-3, 100.0, 92)
    w = synth.normal((Kf, Nf), 0.02, 93, "cpu", torch.bfloat16)
    qdy, sdy = cuda_lib.fp8_quantize_act_1x128(dy.cuda())
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=False)
    dx = cuda_lib.fp8_blockscaled_gemm(qdy, sdy, qw, sw, out_dtype=torch.bfloat16,
                                       sb_kb_nb=False)
    qdy_o, sdy_o = orc.quantize_act_1x128(to_oracle(dy))
    qw_o, sw_o = orc.quantize_weight_128x128(to_oracle(w), transpose_out=False)
    assert_codes_equal(np_u8(qw), qw_o)
    C_ref, T = orc.gemm_ref(qdy_o, sdy_o, qw_o, sw_o, b_kmajor=True, sb_transposed=True)
    assert_gemm_within_bound(np_f32(dx), C_ref, T, torch.bfloat16)


def test_gemm_strided_output_and_operands(cuda_lib, orc):
    M, N, K = 130, 256, 384
    qa, sa, qb, sb = oracle_operands(orc, M, N, K, 5)
    abuf = torch.zeros((M, K + 128), dtype=torch.uint8, device="cuda")
    abuf[:, 64:64 + K] = cuda_u8(qa)
    cbuf = torch.full((M, N + 64), 7.0, dtype=torch.float32, device="cuda")
    c = cbuf[:, 32:32 + N]
    cuda_lib.fp8_blockscaled_gemm(abuf[:, 64:64 + K], torch.from_numpy(sa).cuda(), cuda_u8(qb),
                                  torch.from_numpy(sb).cuda(), c=c)
    C_ref, T = orc.gemm_ref(qa, sa, qb, sb)
    assert_gemm_within_bound(np_f32(c), C_ref, T, torch.float32)
    rest = np_f32(cbuf)
    assert np.all(rest[:, :32] == 7.0) and np.all(rest[:, 32 + N:] == 7.0)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_output_store_paths_agree(cuda_lib, orc, out_dtype):
    """C with 32-byte aligned rows is written as 32-byte stores, C at a
    16-byte offset as 16-byte stores: the two outputs are bit-identical and
    within the bound, and nothing outside C is written."""
    M, N, K = 300, 512, 640
    qa, sa, qb, sb = oracle_operands(orc, M, N, K, 17)
    args = (cuda_u8(qa), torch.from_numpy(sa).cuda(), cuda_u8(qb), torch.from_numpy(sb).cuda())
    c_al = cuda_lib.fp8_blockscaled_gemm(*args, out_dtype=out_dtype)
    off = 16 // c_al.element_size()
    cbuf = torch.full((M, N + 2 * off), 3.0, dtype=out_dtype, device="cuda")
    c_un = cbuf[:, off:off + N]
    cuda_lib.fp8_blockscaled_gemm(*args, c=c_un)
    assert torch.equal(c_al, c_un)
    C_ref, T = orc.gemm_ref(qa, sa, qb, sb)
    assert_gemm_within_bound(np_f32(c_un), C_ref, T, out_dtype)
    rest = np_f32(cbuf)
    assert np.all(rest[:, :off] == 3.0) and np.all(rest[:, off + N:] == 3.0)


def test_gemm_degenerate_sizes(cuda_lib):
    dev = "cuda"
    a = torch.zeros((0, 128), dtype=torch.uint8, device=dev)
    sa = torch.zeros((0, 1), device=dev)
    b = torch.zeros((128, 128), dtype=torch.uint8, device=dev)
    sb = torch.ones((1, 1), device=dev)
    c = cuda_lib.fp8_blockscaled_gemm(a, sa, b, sb)          # M = 0: no-op
    assert c.shape == (0, 128)
    a = torch.zeros((5, 0), dtype=torch.uint8, device=dev)
    sa = torch.zeros((5, 0), device=dev)
    b = torch.zeros((128, 0), dtype=torch.uint8, device=dev)
    sb = torch.zeros((0, 1), device=dev)
    c = torch.full((5, 128), 3.0, device=dev)
    cuda_lib.fp8_blockscaled_gemm(a, sa, b, sb, c=c)        # K = 0: C = 0
    assert torch.all(c == 0)
    assert cuda_lib.fp8_get_device_error() == 0


# ---------------------------------------------------------------- full sizes

def _sampled_linear_check(cuda_lib, orc, x, w_kn, c, qx, sx, qw, sw, rows, nbs, transposed_w):
    """Compare sampled rows x sampled 128-column blocks of C (and the operand
    codes they use) with the oracle on the same inputs."""
    rows_t = torch.from_numpy(rows).cuda()
    qa_o, sa_o = orc.quantize_act_1x128(to_oracle(x[rows_t]))
    assert_codes_equal(np_u8(qx[rows_t]), qa_o)
    assert_scales_equal(sx[rows_t].cpu().numpy(), sa_o)
    worst = 0.0
    for nb in nbs:
        if transposed_w:    # forward: w is [K, N]; block column nb -> q^T rows
            blk = w_kn[:, nb * 128:(nb + 1) * 128]
            qb_o, sb_o = orc.quantize_weight_128x128(to_oracle(blk), transpose_out=True)
            assert_codes_equal(np_u8(qw[nb * 128:(nb + 1) * 128]), qb_o)
            assert_scales_equal(sw[:, nb:nb + 1].cpu().numpy(), sb_o)
            C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o)
        else:               # dgrad: w is [N_out, K]; block row nb, scales [nb][kb]
            blk = w_kn[nb * 128:(nb + 1) * 128]
            qb_o, sb_o = orc.quantize_weight_128x128(to_oracle(blk), transpose_out=False)
            assert_codes_equal(np_u8(qw[nb * 128:(nb + 1) * 128]), qb_o)
            assert_scales_equal(sw[nb:nb + 1].cpu().numpy(), sb_o)
            C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o, b_kmajor=True, sb_transposed=True)
        got = np_f32(c[rows_t, nb * 128:(nb + 1) * 128])
        worst = max(worst, assert_gemm_within_bound(got, C_ref, T, torch.bfloat16))
    return worst


@pytest.mark.slow
def test_ffn_forward_full_size_sampled(cuda_lib, orc):
    """X bf16 [4096x7168] (N(0,1), 0.1% outliers x100), W bf16 [7168x18432]
    (N(0,0.02)), online quantization of both and the block-scaled GEMM to
    bf16 [4096x18432], in the launch configuration the bench times."""
    x, w = synth.ffn_inputs("cuda")
    c = cuda_lib.linear_forward(x, w)
    qx, sx = cuda_lib.fp8_quantize_act_1x128(x)
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 4095], rng.integers(0, 4096, 30)]))
    nbs = sorted(set(rng.integers(0, 144, 3).tolist()) | {0, 143})
    _sampled_linear_check(cuda_lib, orc, x, w, c, qx, sx, qw, sw, rows, nbs, True)
    assert cuda_lib.fp8_get_device_error() == 0


@pytest.mark.slow
def test_dgrad_full_size_sampled(cuda_lib, orc):
    """dY bf16 [16384x18432] (N(0,1e-3), 0.1% outliers x100) quantized 1x128
    along the forward N; W [7168x18432] 128x128 blocks read transposed;
    dX = dY W^T -> bf16 [16384x7168]."""
    dy, w = synth.dgrad_inputs("cuda")
    qdy, sdy = cuda_lib.fp8_quantize_act_1x128(dy)
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=False)
    dx = cuda_lib.fp8_blockscaled_gemm(qdy, sdy, qw, sw, out_dtype=torch.bfloat16,
                                       sb_kb_nb=False)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 16383], rng.integers(0, 16384, 14)]))
    nbs = sorted(set(rng.integers(0, 56, 2).tolist()) | {55})
    _sampled_linear_check(cuda_lib, orc, dy, w, dx, qdy, sdy, qw, sw, rows, nbs, False)
    assert cuda_lib.fp8_get_device_error() == 0

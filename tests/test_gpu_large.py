"""Maximum sizes: inputs and outputs past 2^31 elements, so that every row,
column and byte offset the kernels form must be 64-bit.  Each large call is
compared with the same kernel on a small slice holding the same rows (whose
offsets are small), bit for bit, and sampled rows with the oracle."""
import numpy as np
import pytest
import torch

import synth
from _util import assert_codes_equal, assert_scales_equal, np_u8, to_oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BIG = 2 ** 31


def gpu_normal(shape, std, seed):
    return synth.normal(shape, std, seed, "cuda", torch.bfloat16)


def test_act_quant_past_2_31_elements(cuda_lib, orc):
    M, K = 300_032, 7168                      # 2.15e9 elements, 4.3 GB of bf16
    assert M * K > BIG
    x = gpu_normal((M, K), 1.0, 41)
    q, sa = cuda_lib.fp8_quantize_act_1x128(x)
    tail = slice(M - 1000, M)
    q_t, sa_t = cuda_lib.fp8_quantize_act_1x128(x[tail].contiguous())
    assert torch.equal(q[tail], q_t)
    assert torch.equal(sa[tail].view(torch.int32), sa_t.view(torch.int32))
    rows = torch.tensor([0, 1, M // 2, M - 2, M - 1], device="cuda")
    qo, sao = orc.quantize_act_1x128(to_oracle(x[rows].cpu()))
    assert_codes_equal(np_u8(q[rows]), qo)
    assert_scales_equal(sa[rows].cpu().numpy(), sao)
    assert cuda_lib.fp8_get_device_error() == 0


@pytest.mark.parametrize("transpose_out", [True, False])
def test_weight_quant_past_2_31_elements(cuda_lib, orc, transpose_out):
    K, N = 16384, 139_264                     # 2.28e9 elements
    assert K * N > BIG
    w = gpu_normal((K, N), 0.02, 42)
    q, sb = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=transpose_out)
    cols = slice(N - 256, N)
    q_t, sb_t = cuda_lib.fp8_quantize_weight_128x128(w[:, cols].contiguous(),
                                                      transpose_out=transpose_out)
    if transpose_out:
        assert torch.equal(q[cols], q_t)           # [N, K] codes
    else:
        assert torch.equal(q[:, cols], q_t)        # [K, N] codes
    assert torch.equal(sb[:, -2:].contiguous().view(torch.int32), sb_t.view(torch.int32))
    blk = w[K - 128:, N - 128:].cpu()
    qo, sbo = orc.quantize_weight_128x128(to_oracle(blk), transpose_out=transpose_out)
    got = q[N - 128:, K - 128:] if transpose_out else q[K - 128:, N - 128:]
    assert_codes_equal(np_u8(got), qo)
    assert_scales_equal(sb[-1:, -1:].cpu().numpy(), sbo)
    assert cuda_lib.fp8_get_device_error() == 0


def test_gemm_output_past_2_31_elements(cuda_lib):
    """C [131072 x 18432] bf16 (2.4e9 elements): the last rows equal the same
    product computed on those rows alone (each output element comes from
    one tile, with the same K order wherever the tile sits)."""
    M, N, K = 131_072, 18432, 256
    assert M * N > BIG
    a = gpu_normal((M, K), 1.0, 43)
    w = gpu_normal((K, N), 0.02, 44)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a)
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
    del a, w
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qw, sw)
    tail = slice(M - 512, M)
    c_t = cuda_lib.fp8_blockscaled_gemm(qa[tail].contiguous(), sa[tail].contiguous(), qw, sw)
    assert torch.equal(c[tail].view(torch.int16), c_t.view(torch.int16))
    head = slice(0, 512)
    c_h = cuda_lib.fp8_blockscaled_gemm(qa[head].contiguous(), sa[head].contiguous(), qw, sw)
    assert torch.equal(c[head].view(torch.int16), c_h.view(torch.int16))
    assert cuda_lib.fp8_get_device_error() == 0


def test_dequant_past_2_31_elements(cuda_lib):
    M, K = 300_032, 7168
    codes = torch.randint(0, 256, (M, K), dtype=torch.uint8, device="cuda",
                          generator=torch.Generator("cuda").manual_seed(45))
    codes[(codes & 0x7F) == 0x7F] = 0                  # no NaN codes
    s = torch.rand((M, K // 128), device="cuda", generator=torch.Generator("cuda").manual_seed(46))
    y = cuda_lib.fp8_dequantize(codes, s, 1)
    tail = slice(M - 1000, M)
    y_t = cuda_lib.fp8_dequantize(codes[tail].contiguous(), s[tail].contiguous(), 1)
    assert torch.equal(y[tail].view(torch.int16), y_t.view(torch.int16))
    ref = (codes[tail].view(torch.float8_e4m3fn).float() *
           s[tail].repeat_interleave(128, dim=1)).to(torch.bfloat16)
    assert torch.equal(y[tail].view(torch.int16), ref.view(torch.int16))


def test_grouped_gemm_output_past_2_31_elements(cuda_lib):
    """4 groups over 140000 rows, N 16384 (C 2.3e9 elements), K 4096 (the
    CTA-pair kernel plus the one-CTA remainder kernel): each group's rows equal
    the dense GEMM of those rows with that group's weights."""
    sizes = [40_000, 30_001, 0, 69_999]
    M, N, K = sum(sizes), 16384, 4096
    assert M * N > BIG
    a = gpu_normal((M, K), 1.0, 47)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a)
    del a
    G = len(sizes)
    qb = torch.empty((G, N, K), dtype=torch.uint8, device="cuda")
    sb = torch.empty((G, K // 128, N // 128), dtype=torch.float32, device="cuda")
    for g in range(G):
        w = gpu_normal((K, N), 0.02, 48 + g)
        cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True, q=qb[g], sb=sb[g])
        del w
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    c = cuda_lib.fp8_grouped_gemm(qa, sa, qb, sb, off)
    for g, (lo, hi) in enumerate(zip(off[:-1].tolist(), off[1:].tolist())):
        for r0, r1 in ((lo, min(lo + 300, hi)), (max(hi - 300, lo), hi)):
            if r1 <= r0:
                continue
            ref = cuda_lib.fp8_blockscaled_gemm(qa[r0:r1].contiguous(), sa[r0:r1].contiguous(),
                                                qb[g], sb[g])
            assert torch.equal(c[r0:r1].view(torch.int16), ref.view(torch.int16)), (g, r0, r1)
    assert cuda_lib.fp8_get_device_error() == 0

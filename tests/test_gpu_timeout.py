"""The bounded-wait timeout path, made to run out on the GPU without a fault.

Every wait in the library's kernels (on TMA data, on the tensor core's
commits, on the epilogue's release of tensor memory, on a quantizer group's
barrier) gives up after a limit, records FP8_ERR_DEVICE_TIMEOUT in the
device error word, drains its own copies and tensor-core work in flight,
frees its tensor memory and returns.  These tests shorten the limit to a
cycle (fp8_set_wait_limit) so that ordinary waits run out, check that the
error comes back through fp8_get_device_error, then restore the limit and
check that the same context still computes results equal to the oracle.
Nothing is left waiting: every wait, including the drains, is bounded.
"""
import numpy as np
import pytest
import torch

import synth
from _util import assert_codes_equal, assert_gemm_within_bound, assert_scales_equal, np_f32, \
    np_u8, to_oracle

pytestmark = pytest.mark.gpu

TIMEOUT = 9          # FP8_ERR_DEVICE_TIMEOUT


def _operands(cuda_lib, M, N, K, seed):
    x = synth.normal((M, K), 1.0, seed, "cuda", torch.bfloat16)
    w = synth.normal((K, N), 0.02, seed + 1, "cuda", torch.bfloat16)
    qx, sx = cuda_lib.fp8_quantize_act_1x128(x)
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
    return x, w, qx, sx, qw, sw


def _context_still_usable(cuda_lib, orc):
    """A normal tiny pass after the timeouts: quantizers bit-exact, GEMM
    within the bound, no error recorded."""
    a, b = synth.tiny_inputs("cpu")
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a.cuda())
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(b.cuda(), transpose_out=True)
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.float32)
    assert cuda_lib.fp8_get_device_error() == 0
    qa_o, sa_o = orc.quantize_act_1x128(a.numpy())
    qb_o, sb_o = orc.quantize_weight_128x128(b.numpy(), transpose_out=True)
    assert_codes_equal(np_u8(qa), qa_o)
    assert_scales_equal(sa.cpu().numpy(), sa_o)
    assert_codes_equal(np_u8(qb), qb_o)
    assert_scales_equal(sb.cpu().numpy(), sb_o)
    C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o)
    assert_gemm_within_bound(np_f32(c), C_ref, T, torch.float32)


def test_gemm_wait_timeout_reported_then_context_usable(cuda_lib, orc):
    """Dense CTA-pair GEMM (K = 8192: 64 chunks per tile) under a one-cycle
    wait limit: some wait runs out, the kernel aborts and reports it."""
    assert cuda_lib.fp8_get_device_error() == 0
    _, _, qx, sx, qw, sw = _operands(cuda_lib, 1024, 2048, 8192, 41)
    torch.cuda.synchronize()
    codes = []
    cuda_lib.fp8_set_wait_limit(1)
    try:
        for _ in range(3):
            cuda_lib.fp8_blockscaled_gemm(qx, sx, qw, sw)
            codes.append(cuda_lib.fp8_get_device_error())
            if codes[-1] == TIMEOUT:
                break
    finally:
        cuda_lib.fp8_set_wait_limit(0)
    assert codes[-1] == TIMEOUT, codes
    assert set(codes) <= {0, TIMEOUT}, codes
    _context_still_usable(cuda_lib, orc)


def test_quantizer_and_grouped_wait_timeouts_then_context_usable(cuda_lib, orc):
    """The streamed quantizers (row kernel for bf16 activations, box kernel
    for weights) and the one-CTA grouped GEMM (K < 4096) under a one-cycle
    limit: each run either finishes or reports a timeout, and at least one
    reports it; afterwards a normal pass is exact."""
    assert cuda_lib.fp8_get_device_error() == 0
    x = synth.normal((4096, 7168), 1.0, 51, "cuda", torch.bfloat16)
    w = synth.normal((2048, 4096), 0.02, 52, "cuda", torch.bfloat16)
    G, rows_per, N, K = 8, 256, 1024, 2048
    a = synth.normal((G * rows_per, K), 1.0, 53, "cuda", torch.bfloat16)
    wg = synth.normal((G, N, K), 0.02, 54, "cuda", torch.bfloat16)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a)
    qg = torch.empty((G, N, K), dtype=torch.uint8, device="cuda")
    sg = torch.empty((G, K // 128, N // 128), dtype=torch.float32, device="cuda")
    for g in range(G):     # [N, K] codes are the untransposed quantization of w^T
        qb, sb = cuda_lib.fp8_quantize_weight_128x128(wg[g].t().contiguous(), transpose_out=True)
        qg[g].copy_(qb)
        sg[g].copy_(sb)
    off = torch.arange(0, (G + 1) * rows_per, rows_per, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    codes = {}
    cuda_lib.fp8_set_wait_limit(1)
    try:
        cuda_lib.fp8_quantize_act_1x128(x)
        codes["act"] = cuda_lib.fp8_get_device_error()
        cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
        codes["weight"] = cuda_lib.fp8_get_device_error()
        cuda_lib.fp8_grouped_gemm(qa, sa, qg, sg, off)
        codes["grouped"] = cuda_lib.fp8_get_device_error()
    finally:
        cuda_lib.fp8_set_wait_limit(0)
    assert set(codes.values()) <= {0, TIMEOUT}, codes
    assert TIMEOUT in codes.values(), codes
    _context_still_usable(cuda_lib, orc)
    # the same calls with the default limit: no error, exact quantization
    q, s = cuda_lib.fp8_quantize_act_1x128(x[:64])
    qo, so = orc.quantize_act_1x128(to_oracle(x[:64]))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(s.cpu().numpy(), so)
    assert cuda_lib.fp8_get_device_error() == 0


def test_wait_limit_argument_errors(cuda_lib):
    with pytest.raises(cuda_lib.Fp8Error):
        cuda_lib.fp8_set_wait_limit(-1)
    cuda_lib.fp8_set_wait_limit(0)
    assert cuda_lib.fp8_get_device_error() == 0

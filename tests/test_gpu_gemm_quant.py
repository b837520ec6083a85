"""GEMM with its output quantized in the epilogue (fp8_blockscaled_gemm_quant):
bit-identical to the unfused GEMM (bf16 out) followed by the 1x128
activation quantizer, and, against the oracle's fp64 product, within the
GEMM bound plus half an E4M3 step."""
import numpy as np
import pytest
import torch

from _util import gemm_bound, np_u8

pytestmark = pytest.mark.gpu


def operands(orc, M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-3, 4, (M, 1), generator=g).float())
    w = torch.randn(K, N, generator=g) * 0.05
    return x, w


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (130, 384, 256), (256, 256, 1024),
                                   (600, 1280, 512), (1000, 512, 7168)])
@pytest.mark.parametrize("want_c", [False, True])
def test_fused_equals_unfused(cuda_lib, orc, M, N, K, want_c):
    x, w = operands(orc, M, N, K, M + N + K)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=True)
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    qc_ref, sc_ref = cuda_lib.fp8_quantize_act_1x128(c)
    res = cuda_lib.fp8_blockscaled_gemm_quant(qa, sa, qb, sb, want_c=want_c)
    assert torch.equal(res[0], qc_ref)
    assert torch.equal(res[1].view(torch.int32), sc_ref.view(torch.int32))
    if want_c:
        assert torch.equal(res[2].view(torch.int16), c.view(torch.int16))
    assert cuda_lib.fp8_get_device_error() == 0


def test_fused_output_against_oracle(cuda_lib, orc):
    M, N, K = 300, 512, 1024
    x, w = operands(orc, M, N, K, 7)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=True)
    qc, sc = cuda_lib.fp8_blockscaled_gemm_quant(qa, sa, qb, sb)
    qa_o, sa_o = orc.quantize_act_1x128(x.numpy())
    qb_o, sb_o = orc.quantize_weight_128x128(w.numpy(), transpose_out=True)
    C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o)
    # dequantize the GPU's codes here (E4M3 value x scale)
    dec = torch.from_numpy(np_u8(qc).copy()).view(torch.float8_e4m3fn).double().numpy()
    s = np.repeat(sc.cpu().double().numpy(), 128, axis=1)
    y = dec * s
    bound = gemm_bound(C_ref, T, torch.bfloat16) + np.maximum(2.0 ** -4 * np.abs(C_ref), 2.0 ** -10 * s) * 1.01
    assert np.all(np.abs(y - C_ref) <= bound)


def test_strided_outputs(cuda_lib, orc):
    M, N, K = 200, 256, 256
    x, w = operands(orc, M, N, K, 3)
    qa, sa = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=True)
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    qc_ref, sc_ref = cuda_lib.fp8_quantize_act_1x128(c)
    qbuf = torch.full((M, 384), 0xCD, dtype=torch.uint8, device="cuda")
    sc_t = torch.full((N // 128, M), -1.0, device="cuda")             # column-major scales
    cbuf = torch.zeros((M, 384), dtype=torch.bfloat16, device="cuda")
    cuda_lib.fp8_blockscaled_gemm_quant(qa, sa, qb, sb, qc=qbuf[:, 64:64 + N], sc=sc_t.t(),
                                        c=cbuf[:, 128:128 + N])
    assert torch.equal(qbuf[:, 64:64 + N], qc_ref)
    assert torch.equal(sc_t.t(), sc_ref)
    assert torch.equal(cbuf[:, 128:128 + N].view(torch.int16), c.view(torch.int16))
    assert torch.all(qbuf[:, :64] == 0xCD) and torch.all(qbuf[:, 64 + N:] == 0xCD)


@pytest.mark.slow
def test_ffn_full_size_fused_equals_unfused(cuda_lib):
    import synth
    x, w = synth.ffn_inputs("cuda")
    qa, sa = cuda_lib.fp8_quantize_act_1x128(x)
    qb, sb = cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True)
    del x, w
    c = cuda_lib.fp8_blockscaled_gemm(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    qc_ref, sc_ref = cuda_lib.fp8_quantize_act_1x128(c)
    del c
    qc, sc = cuda_lib.fp8_blockscaled_gemm_quant(qa, sa, qb, sb)
    assert torch.equal(qc, qc_ref)
    assert torch.equal(sc.view(torch.int32), sc_ref.view(torch.int32))

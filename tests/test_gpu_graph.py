"""The library's calls are stream-ordered work with no host synchronisation,
so they capture into a CUDA graph: an FFN step (two quantizations and the
GEMM) and an MoE step (scatter dispatch, grouped GEMM) replayed on new
input contents give exactly the eager results."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_ffn_step_in_a_cuda_graph(cuda_lib):
    M, K, N = 512, 1024, 768
    x = synth.normal((M, K), 1.0, 61, "cuda")
    w = synth.normal((K, N), 0.02, 62, "cuda")
    qx = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sx = torch.empty((M, K // 128), dtype=torch.float32, device="cuda")
    qw = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty((K // 128, N // 128), dtype=torch.float32, device="cuda")
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

    def step(stream):
        cuda_lib.fp8_quantize_act_1x128(x, q=qx, sa=sx, stream=stream)
        cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True, q=qw, sb=sw, stream=stream)
        cuda_lib.fp8_blockscaled_gemm(qx, sx, qw, sw, c=c, stream=stream)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(side)                      # warm-up (first-call setup) outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(torch.cuda.current_stream())
    for seed in (63, 64):
        x.copy_(synth.normal((M, K), 1.0, seed, "cuda"))
        w.copy_(synth.normal((K, N), 0.02, seed + 10, "cuda"))
        g.replay()
        torch.cuda.synchronize()
        ref = cuda_lib.linear_forward(x, w)
        assert torch.equal(c.view(torch.int16), ref.view(torch.int16))
    assert cuda_lib.fp8_get_device_error() == 0


def test_moe_step_in_a_cuda_graph(cuda_lib):
    T, E, topk, H, N = 512, 8, 2, 4096, 512     # K 4096: the two-launch grouped path
    token_of, offsets = synth.moe_routing(T, E, topk, 65, "cpu")
    dest = synth.moe_dispatch_dest(token_of, T, topk).cuda()
    off = offsets.cuda()
    R = T * topk
    x = synth.normal((T, H), 1.0, 66, "cuda")
    qb = torch.empty((E, N, H), dtype=torch.uint8, device="cuda")
    sb = torch.empty((E, H // 128, N // 128), dtype=torch.float32, device="cuda")
    for e in range(E):
        cuda_lib.fp8_quantize_weight_128x128(synth.normal((H, N), 0.02, 70 + e, "cuda"),
                                             transpose_out=True, q=qb[e], sb=sb[e])
    qx = torch.empty((R, H), dtype=torch.uint8, device="cuda")
    sx = torch.empty((R, H // 128), dtype=torch.float32, device="cuda")
    c = torch.empty((R, N), dtype=torch.bfloat16, device="cuda")

    def step(stream):
        cuda_lib.fp8_quantize_act_1x128_scatter(x, dest, R, q=qx, sa=sx, stream=stream)
        cuda_lib.fp8_grouped_gemm(qx, sx, qb, sb, off, c=c, stream=stream)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(torch.cuda.current_stream())
    x.copy_(synth.normal((T, H), 1.0, 67, "cuda"))
    g.replay()
    torch.cuda.synchronize()
    q_ref, s_ref = cuda_lib.fp8_quantize_act_1x128(x[token_of.cuda()].contiguous())
    c_ref = cuda_lib.fp8_grouped_gemm(q_ref, s_ref, qb, sb, off)
    assert torch.equal(qx, q_ref)
    assert torch.equal(c.view(torch.int16), c_ref.view(torch.int16))
    assert cuda_lib.fp8_get_device_error() == 0

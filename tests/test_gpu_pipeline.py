"""The pipelined end-to-end linear forward (host tensors in, host tensor
out, copies in both directions overlapped across calls) gives exactly the
device path's result for every call, whatever the depth and however the
host buffers are reused; and that result is the oracle's within the GEMM
bound."""
import pytest
import torch

import synth
from _util import assert_gemm_within_bound, np_f32

pytestmark = pytest.mark.gpu


def host_operands(M, K, N, seed):
    x = synth.act_input(M, K, 1.0, 1e-2, 100.0, 3, "cpu", torch.bfloat16, tensor_id=seed % 5)
    w = (synth.normal((K, N), 0.02, seed + 50, "cpu", torch.float32)).to(torch.bfloat16)
    return x.pin_memory(), w.pin_memory()


@pytest.mark.parametrize("depth", [1, 2, 3])
def test_pipeline_matches_device_path(cuda_lib, depth):
    M, K, N = 300, 384, 512
    calls = [host_operands(M, K, N, 10 * depth + i) for i in range(5)]
    outs = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in calls]
    pipe = cuda_lib.LinearForwardPipeline(M, K, N, depth=depth)
    events = [pipe.submit(x, w, o) for (x, w), o in zip(calls, outs)]
    pipe.synchronize()
    assert all(e.query() for e in events)
    for (x, w), o in zip(calls, outs):
        ref = cuda_lib.linear_forward(x.cuda(), w.cuda())
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16))
    pipe.close()
    assert cuda_lib.fp8_get_device_error() == 0


def test_pipeline_reused_host_buffers_and_join(cuda_lib, orc):
    """The bench's pattern: the same pinned buffers every call, a join on
    the caller's stream at the end; new inputs between calls after a join."""
    M, K, N = 256, 512, 256
    (x0, w0), (x1, w1) = host_operands(M, K, N, 1), host_operands(M, K, N, 2)
    hx, hw = x0.clone().pin_memory(), w0.clone().pin_memory()
    hc = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    pipe = cuda_lib.LinearForwardPipeline(M, K, N)
    for _ in range(4):
        pipe.submit(hx, hw, hc)
    stream = torch.cuda.current_stream()
    pipe.join(stream)
    stream.synchronize()
    ref0 = cuda_lib.linear_forward(x0.cuda(), w0.cuda()).cpu()
    assert torch.equal(hc.view(torch.int16), ref0.view(torch.int16))
    hx.copy_(x1)
    hw.copy_(w1)
    pipe.submit(hx, hw, hc)
    pipe.synchronize()
    ref1 = cuda_lib.linear_forward(x1.cuda(), w1.cuda()).cpu()
    assert torch.equal(hc.view(torch.int16), ref1.view(torch.int16))
    # and the device path is the oracle's within the GEMM bound
    qa, sa = orc.quantize_act_1x128(x1.float().numpy())
    qb, sb = orc.quantize_weight_128x128(w1.float().numpy(), transpose_out=True)
    C_ref, T = orc.gemm_ref(qa, sa, qb, sb)
    assert_gemm_within_bound(np_f32(hc), C_ref, T, torch.bfloat16)
    pipe.close()


def test_pipeline_rejects_wrong_shapes(cuda_lib):
    pipe = cuda_lib.LinearForwardPipeline(128, 128, 128)
    x = torch.zeros((128, 256), dtype=torch.bfloat16)
    w = torch.zeros((128, 128), dtype=torch.bfloat16)
    o = torch.zeros((128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pipe.submit(x, w, o)
    with pytest.raises(TypeError):
        pipe.submit(torch.zeros((128, 128)), w, o)
    pipe.close()

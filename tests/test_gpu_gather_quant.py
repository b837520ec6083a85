"""Fused MoE dispatch + 1x128 quantization, in row order (gather: output row
r from token rows[r]) and in token order (scatter: token t to output rows
dest[t, :]): bit-identical to the oracle's quantization of the gathered
rows x[rows]."""
import numpy as np
import pytest
import torch

import synth
from _util import assert_codes_equal, assert_scales_equal, np_u8, to_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,R,K", [(1, 1, 128), (50, 77, 384), (300, 1201, 1024), (256, 2048, 7168)])
def test_gather_quant_matches_oracle(cuda_lib, orc, T, R, K, dtype):
    x = synth.act_input(T, K, 1.0, 1e-2, 100.0, 7, "cpu", dtype, tensor_id=T % 7)
    g = torch.Generator().manual_seed(R)
    rows = torch.randint(0, T, (R,), generator=g, dtype=torch.int32)
    q, sa = cuda_lib.fp8_quantize_act_1x128_gather(x.cuda(), rows.cuda())
    qo, sao = orc.quantize_act_1x128(to_oracle(x[rows.long()]))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa.cpu().numpy(), sao)


@pytest.mark.parametrize("offset", [0, 16])
def test_gather_quant_both_bf16_paths(cuda_lib, orc, offset):
    """Codes at 32-byte and 16-byte offsets: both equal the oracle and nothing
    outside q is written."""
    T, R, K = 97, 333, 640
    x = synth.act_input(T, K, 1.0, 1e-2, 100.0, 7, "cpu", torch.bfloat16, tensor_id=4)
    rows = torch.randint(0, T, (R,), generator=torch.Generator().manual_seed(9), dtype=torch.int32)
    qbuf = torch.full((R, K + 16 + offset), 0xCD, dtype=torch.uint8, device="cuda")
    q = qbuf[:, offset:offset + K]
    _, sa = cuda_lib.fp8_quantize_act_1x128_gather(x.cuda(), rows.cuda(), q=q)
    qo, sao = orc.quantize_act_1x128(to_oracle(x[rows.long()]))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa.cpu().numpy(), sao)
    rest = np_u8(qbuf)
    assert np.all(rest[:, :offset] == 0xCD) and np.all(rest[:, offset + K:] == 0xCD)


def test_gather_quant_equals_gather_then_quantize(cuda_lib):
    d = synth.moe_inputs("cpu", tokens=1024, experts=32, with_weights=False)
    x = synth.act_input(1024, 7168, 1.0, 1e-3, 100.0, synth.MOE.config_id, "cpu").cuda()
    rows = d["token_of"].to(torch.int32).cuda()
    q1, s1 = cuda_lib.fp8_quantize_act_1x128_gather(x, rows)
    q2, s2 = cuda_lib.fp8_quantize_act_1x128(x[rows.long()].contiguous())
    assert torch.equal(q1, q2)
    assert torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_invalid_index_reported_and_row_untouched(cuda_lib):
    x = torch.randn(10, 256, generator=torch.Generator().manual_seed(10)).bfloat16().cuda()
    rows = torch.tensor([0, 3, 10, 9, -1], dtype=torch.int32).cuda()
    q = torch.full((5, 256), 0xAB, dtype=torch.uint8, device="cuda")
    sa = torch.full((5, 2), -3.0, device="cuda")
    assert cuda_lib.fp8_get_device_error() == 0
    cuda_lib.fp8_quantize_act_1x128_gather(x, rows, q=q, sa=sa)
    assert cuda_lib.fp8_get_device_error() == 2
    assert torch.all(q[2] == 0xAB) and torch.all(q[4] == 0xAB)
    assert torch.all(sa[2] == -3.0) and torch.all(sa[4] == -3.0)
    q_ok, s_ok = cuda_lib.fp8_quantize_act_1x128(x[[0, 3, 9]].contiguous())
    assert torch.equal(q[[0, 1, 3]], q_ok)
    assert torch.equal(sa[[0, 1, 3]], s_ok)


@pytest.mark.slow
def test_moe_dispatch_full_size_sampled(cuda_lib, orc):
    """8192 tokens x top-8 of 256 experts: all 65536 routed rows of both
    dispatch forms (row-order gather, token-order scatter as the MoE bench
    runs it) equal the unfused gather + quantize; sampled rows against the
    oracle."""
    d = synth.moe_inputs("cpu", with_weights=False)
    x = synth.act_input(8192, 7168, 1.0, 1e-3, 100.0, synth.MOE.config_id, "cpu")
    rows = d["token_of"].to(torch.int32)
    xc, rc = x.cuda(), rows.cuda()
    q, sa = cuda_lib.fp8_quantize_act_1x128_gather(xc, rc)
    q2, s2 = cuda_lib.fp8_quantize_act_1x128(xc[rc.long()].contiguous())
    assert torch.equal(q, q2) and torch.equal(sa, s2)
    dest = synth.moe_dispatch_dest(d["token_of"], 8192, 8).cuda()
    q3, s3 = cuda_lib.fp8_quantize_act_1x128_scatter(xc, dest, 65536)
    assert torch.equal(q3, q2) and torch.equal(s3.view(torch.int32), s2.view(torch.int32))
    pick = np.array([0, 1, 4095, 30000, 65535])
    qo, sao = orc.quantize_act_1x128(to_oracle(x[rows[pick].long()]))
    assert_codes_equal(np_u8(q[torch.from_numpy(pick).cuda()]), qo)
    assert_scales_equal(sa[torch.from_numpy(pick).cuda()].cpu().numpy(), sao)


def _routing(T, E, topk, seed):
    token_of, _ = synth.moe_routing(T, E, topk, seed)
    return token_of, synth.moe_dispatch_dest(token_of, T, topk)


@pytest.mark.parametrize("T,E,topk,K", [(1, 4, 1, 128), (33, 8, 3, 384), (300, 16, 4, 1024),
                                        (97, 64, 11, 256), (1024, 32, 8, 7168),
                                        # more boxes than the grid's warps: one tile per row
                                        # band (every box a new band), and runs of several
                                        # boxes crossing bands
                                        (40000, 64, 2, 128), (9000, 16, 2, 640),
                                        (20000, 8, 2, 1024)])
def test_scatter_quant_matches_oracle_and_gather(cuda_lib, orc, T, E, topk, K):
    """Token-order dispatch: every routed row equals the oracle's quantization
    of its token, and the whole output equals the gather form's."""
    x = synth.act_input(T, K, 1.0, 1e-2, 100.0, 7, "cpu", torch.bfloat16, tensor_id=T % 5)
    token_of, dest = _routing(T, E, topk, 1000 + T)
    R = T * topk
    q, sa = cuda_lib.fp8_quantize_act_1x128_scatter(x.cuda(), dest.cuda(), R)
    qo, sao = orc.quantize_act_1x128(to_oracle(x[token_of]))
    assert_codes_equal(np_u8(q), qo)
    assert_scales_equal(sa.cpu().numpy(), sao)
    qg, sg = cuda_lib.fp8_quantize_act_1x128_gather(x.cuda(), token_of.to(torch.int32).cuda())
    assert torch.equal(q, qg)
    assert torch.equal(sa.view(torch.int32), sg.view(torch.int32))


def test_scatter_skips_minus_one_and_reports_bad_rows(cuda_lib, orc):
    """-1 entries write nothing; entries outside [0, R) record FP8_ERR_SHAPE
    and write nothing; the valid entries are exact."""
    T, K, R = 40, 256, 64
    x = synth.act_input(T, K, 1.0, 1e-2, 100.0, 7, "cpu", torch.bfloat16, tensor_id=3)
    dest = torch.full((T, 2), -1, dtype=torch.int32)
    dest[:, 0] = torch.arange(T, dtype=torch.int32)            # token t -> row t
    dest[5, 1] = 50
    dest[7, 1] = R                                              # out of range
    dest[9, 1] = -7                                             # out of range
    q = torch.full((R, K), 0xEE, dtype=torch.uint8, device="cuda")
    sa = torch.full((R, K // 128), -5.0, device="cuda")
    assert cuda_lib.fp8_get_device_error() == 0
    cuda_lib.fp8_quantize_act_1x128_scatter(x.cuda(), dest.cuda(), R, q=q, sa=sa)
    assert cuda_lib.fp8_get_device_error() == 2
    qo, sao = orc.quantize_act_1x128(to_oracle(x))
    assert_codes_equal(np_u8(q[:T]), qo)
    assert_scales_equal(sa[:T].cpu().numpy(), sao)
    assert_codes_equal(np_u8(q[50:51]), qo[5:6])
    untouched = [r for r in range(T, R) if r != 50]
    assert torch.all(q[untouched] == 0xEE) and torch.all(sa[untouched] == -5.0)

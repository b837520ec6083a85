"""GPU parity of the MoE grouped block-scaled GEMM against the oracle."""
import numpy as np
import pytest
import torch

import synth
from _util import assert_codes_equal, assert_gemm_within_bound, assert_scales_equal, np_f32, \
    np_u8, to_oracle

pytestmark = pytest.mark.gpu


def grouped_operands(orc, sizes, N, K, seed):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    total = int(off[-1])
    x = synth.normal((max(total, 1), K), 1.0, seed, "cpu", torch.float32)[:total]
    synth.scale_outliers(x, 1e-2, 100.0, seed + 1)
    qa, sa = orc.quantize_act_1x128(np.ascontiguousarray(x.numpy()))
    qbs, sbs = [], []
    for g in range(len(sizes)):
        w = synth.normal((K, N), 0.02, seed + 100 + g, "cpu", torch.float32)
        q, s = orc.quantize_weight_128x128(w.numpy(), transpose_out=True)
        qbs.append(q)
        sbs.append(s)
    return off, qa, sa, np.stack(qbs), np.stack(sbs)


def run_grouped(cuda_lib, off, qa, sa, qb, sb, out_dtype):
    return cuda_lib.fp8_grouped_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                                     torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda(),
                                     torch.from_numpy(off).cuda(), out_dtype=out_dtype)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("sizes,N,K", [([3, 0, 130, 1, 257], 256, 384),
                                       ([0, 0, 128], 128, 128),
                                       ([200, 56, 0, 0, 311, 129, 1, 64], 384, 256),
                                       ([1000], 512, 1024),
                                       # long contraction: the CTA-pair kernel (256-row
                                       # tiles), remainders of 1-128 rows on one CTA
                                       ([300, 0, 17, 520, 256, 1], 256, 4096),
                                       ([400, 384, 129, 250, 0, 641, 128, 512, 383], 256, 4096)])
def test_grouped_matches_oracle(cuda_lib, orc, sizes, N, K, out_dtype):
    off, qa, sa, qb, sb = grouped_operands(orc, sizes, N, K, sum(sizes) + N)
    c = run_grouped(cuda_lib, off, qa, sa, qb, sb, out_dtype)
    C_ref, T = orc.grouped_gemm_ref(qa, sa, qb, sb, off)
    assert_gemm_within_bound(np_f32(c), C_ref, T, out_dtype)
    assert cuda_lib.fp8_get_device_error() == 0


def test_single_group_equals_dense(cuda_lib, orc):
    off, qa, sa, qb, sb = grouped_operands(orc, [333], 256, 512, 9)
    cg = run_grouped(cuda_lib, off, qa, sa, qb, sb, torch.float32)
    cd = cuda_lib.fp8_blockscaled_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                                       torch.from_numpy(qb[0]).cuda(),
                                       torch.from_numpy(sb[0]).cuda(), out_dtype=torch.float32)
    assert torch.equal(cg, cd)


def test_invalid_offsets_are_reported_not_faulted(cuda_lib, orc):
    """A decreasing offset pair empties that group and sets FP8_ERR_SHAPE in
    the device error word; every access stays in bounds."""
    sizes = [64, 64, 64]
    off, qa, sa, qb, sb = grouped_operands(orc, sizes, 128, 128, 3)
    bad = off.copy()
    bad[2] = 50                         # offsets 0, 64, 50, 192: group 1 is decreasing
    assert cuda_lib.fp8_get_device_error() == 0
    run_grouped(cuda_lib, bad, qa, sa, qb, sb, torch.float32)
    assert cuda_lib.fp8_get_device_error() == 2
    assert cuda_lib.fp8_get_device_error() == 0   # read clears it


@pytest.mark.slow
def test_moe_full_size_sampled(cuda_lib, orc):
    """8192 tokens x top-8 of 256 experts (uniform routing), gate+up
    [7168 -> 4096] and down [2048 -> 7168] per expert: both grouped GEMMs at
    full size, sampled experts / rows / column blocks against the oracle."""
    d = synth.moe_inputs("cuda", with_weights=False)
    off = d["offsets"]
    off_np = off.cpu().numpy()
    assert off_np[-1] == 65536 and np.all(np.diff(off_np) >= 0)
    rng = np.random.default_rng(5)
    experts = sorted(set(rng.integers(0, 256, 4).tolist()) | {0, 255})
    for which, a_bf16, K, N in (("gate_up", d["x_routed"], 7168, 4096),
                                ("down", d["h_down"], 2048, 7168)):
        qa, sa = cuda_lib.fp8_quantize_act_1x128(a_bf16)
        qb = torch.empty((256, N, K), dtype=torch.uint8, device="cuda")
        sb = torch.empty((256, K // 128, N // 128), device="cuda")
        w_of = {}
        for e in range(256):
            w = synth.moe_expert_weight(e, which, "cuda")
            cuda_lib.fp8_quantize_weight_128x128(w, transpose_out=True, q=qb[e], sb=sb[e])
            if e in experts:
                w_of[e] = w
            del w
        c = cuda_lib.fp8_grouped_gemm(qa, sa, qb, sb, off, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        for e in experts:
            r0, r1 = int(off_np[e]), int(off_np[e + 1])
            if r1 == r0:
                continue
            rows = np.unique(np.concatenate([[r0, r1 - 1], rng.integers(r0, r1, 6)]))
            rows_t = torch.from_numpy(rows).cuda()
            qa_o, sa_o = orc.quantize_act_1x128(to_oracle(a_bf16[rows_t]))
            assert_codes_equal(np_u8(qa[rows_t]), qa_o)
            for nb in sorted(set(rng.integers(0, N // 128, 1).tolist()) | {N // 128 - 1}):
                blk = w_of[e][:, nb * 128:(nb + 1) * 128]
                qb_o, sb_o = orc.quantize_weight_128x128(to_oracle(blk), transpose_out=True)
                assert_codes_equal(np_u8(qb[e, nb * 128:(nb + 1) * 128]), qb_o)
                assert_scales_equal(sb[e, :, nb:nb + 1].cpu().numpy(), sb_o)
                C_ref, T = orc.gemm_ref(qa_o, sa_o, qb_o, sb_o)
                got = np_f32(c[rows_t, nb * 128:(nb + 1) * 128])
                assert_gemm_within_bound(got, C_ref, T, torch.bfloat16)
        del qb, c
    assert cuda_lib.fp8_get_device_error() == 0


def test_max_groups_two_launch_path(cuda_lib):
    """G = 1024 (the maximum) with random 0-300-row groups at K = 4096: the
    CTA-pair and remainder launches both build 1024-group tile tables.  A
    spread of groups (empty, small, over 256 rows) equals the dense GEMM of
    the same rows with that group's weights, bit for bit."""
    G, N, K = 1024, 256, 4096
    rng = np.random.default_rng(11)
    sizes = rng.integers(0, 301, G)
    sizes[[3, 500, 1023]] = 0
    total = int(sizes.sum())
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    a = synth.normal((total, K), 1.0, 12, "cuda")
    qa, sa = cuda_lib.fp8_quantize_act_1x128(a)
    qb = torch.empty((G, N, K), dtype=torch.uint8, device="cuda")
    sb = torch.empty((G, K // 128, N // 128), dtype=torch.float32, device="cuda")
    w = synth.normal((K, G * N), 0.02, 13, "cuda")
    for g in range(G):
        cuda_lib.fp8_quantize_weight_128x128(w[:, g * N:(g + 1) * N], transpose_out=True,
                                             q=qb[g], sb=sb[g])
    c = cuda_lib.fp8_grouped_gemm(qa, sa, qb, sb, off)
    offs = off.tolist()
    checked = 0
    for g in list(range(0, G, 37)) + [3, 500, 1022, 1023]:
        lo, hi = offs[g], offs[g + 1]
        if hi == lo:
            continue
        ref = cuda_lib.fp8_blockscaled_gemm(qa[lo:hi].contiguous(), sa[lo:hi].contiguous(), qb[g], sb[g])
        assert torch.equal(c[lo:hi].view(torch.int16), ref.view(torch.int16)), g
        checked += 1
    assert checked > 20
    assert cuda_lib.fp8_get_device_error() == 0

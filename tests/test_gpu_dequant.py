"""GPU parity of fp8_dequantize against the oracle: fp32 outputs bit-identical,
bf16 outputs bit-identical to the oracle's fp32 result rounded to nearest even."""
import numpy as np
import pytest
import torch

from _util import np_u8

pytestmark = pytest.mark.gpu


def codes_and_scales(R, C, tile_rows, seed, nan=False):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (R, C)).astype(np.uint8)
    if not nan:
        q[(q & 0x7F) == 0x7F] = 0x7E                    # no NaN codes
    s = (rng.uniform(0.5, 1.0, ((R + tile_rows - 1) // tile_rows, C // 128)) *
         np.exp2(rng.integers(-30, 30, ((R + tile_rows - 1) // tile_rows, C // 128)))).astype(np.float32)
    return q, s


def check(orc, out, q, s, tile_rows, out_dtype):
    ref = orc.dequantize_fp32(q, s, tile_rows)
    got = out.detach().cpu()
    if out_dtype == torch.float32:
        g = got.numpy().view(np.uint32)
        r = ref.view(np.uint32)
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got.numpy()), nan)
        bad = np.argwhere((g != r) & ~nan)
        assert bad.size == 0, "fp32 bits differ at %s" % bad[:5].tolist()
    else:
        g = got.view(torch.int16).numpy().view(np.uint16)
        r = orc.f32_to_bf16_bits(ref)
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got.float().numpy()), nan)
        bad = np.argwhere((g != r) & ~nan)
        assert bad.size == 0, "bf16 bits differ at %s" % bad[:5].tolist()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("tile_rows,R,C", [(1, 1, 128), (1, 257, 384), (1, 1000, 7168),
                                           (128, 128, 128), (128, 300, 512), (128, 1024, 4352)])
def test_dequant_bit_exact(cuda_lib, orc, tile_rows, R, C, out_dtype):
    q, s = codes_and_scales(R, C, tile_rows, R * 7 + C)
    out = cuda_lib.fp8_dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(),
                                  tile_rows, out_dtype=out_dtype)
    check(orc, out, q, s, tile_rows, out_dtype)


def test_dequant_nan_codes_and_extremes(cuda_lib, orc):
    q, s = codes_and_scales(64, 256, 1, 5, nan=True)
    s[0, 0] = 2.0 ** -149                               # subnormal products
    s[1, 1] = 3.0e38 / 448                              # near fp32 max
    s[2, 0] = 1.0
    for dt in (torch.float32, torch.bfloat16):
        out = cuda_lib.fp8_dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), 1,
                                      out_dtype=dt)
        check(orc, out, q, s, 1, dt)


def test_dequant_strided(cuda_lib, orc):
    """ldq > C, ldo > C, column-major scales."""
    R, C = 200, 512
    q, s = codes_and_scales(R, C, 128, 11)
    qbuf = torch.zeros((R, 640), dtype=torch.uint8, device="cuda")
    qbuf[:, 64:64 + C] = torch.from_numpy(q).cuda()
    s_t = torch.from_numpy(np.ascontiguousarray(s.T)).cuda()        # [C/128, R/128]
    obuf = torch.full((R, 768), -7.0, device="cuda")
    cuda_lib.fp8_dequantize(qbuf[:, 64:64 + C], s_t.t(), 128, out=obuf[:, 128:128 + C])
    check(orc, obuf[:, 128:128 + C], q, s, 128, torch.float32)
    assert torch.all(obuf[:, :128] == -7.0) and torch.all(obuf[:, 128 + C:] == -7.0)


def test_round_trip_through_both_quantizers(cuda_lib, orc):
    """Quantize on the GPU (bit-exact to the oracle), dequantize on the GPU:
    equal to the oracle's dequantization of its own quantization."""
    import synth
    x = synth.act_input(300, 1024, 1.0, 1e-2, 100.0, 7, "cpu", torch.bfloat16, tensor_id=3)
    w = synth.weight_input(512, 768, 0.02, 7, "cpu")
    from _util import to_oracle
    qx, sx = cuda_lib.fp8_quantize_act_1x128(x.cuda())
    qw, sw = cuda_lib.fp8_quantize_weight_128x128(w.cuda(), transpose_out=False)
    yx = cuda_lib.fp8_dequantize(qx, sx, 1, out_dtype=torch.float32)
    yw = cuda_lib.fp8_dequantize(qw, sw, 128, out_dtype=torch.float32)
    qxo, sxo = orc.quantize_act_1x128(to_oracle(x))
    qwo, swo = orc.quantize_weight_128x128(to_oracle(w))
    check(orc, yx, qxo, sxo, 1, torch.float32)
    check(orc, yw, qwo, swo, 128, torch.float32)


@pytest.mark.slow
def test_dequant_weight_full_size_sampled(cuda_lib, orc):
    """The bench's dequant workload, W codes [7168 x 18432] -> bf16: sampled rows."""
    R, C = 7168, 18432
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    q = torch.randint(0, 0x7F, (R, C), dtype=torch.uint8, device="cuda", generator=g)
    s = torch.rand((R // 128, C // 128), device="cuda", generator=g) + 0.5
    out = cuda_lib.fp8_dequantize(q, s, 128, out_dtype=torch.bfloat16)
    rows = np.array([0, 1, 127, 128, 3001, 7167])
    qs = np_u8(q[torch.from_numpy(rows).cuda()])
    ss = s.cpu().numpy()[rows // 128]
    ref_all = orc.dequantize_fp32(qs, ss, 1)
    g_bits = out[torch.from_numpy(rows).cuda()].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(g_bits, orc.f32_to_bf16_bits(ref_all))

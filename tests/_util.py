"""Helpers shared by the GPU parity tests: moving inputs to the oracle's
formats and the GEMM acceptance bound."""
import numpy as np
import torch


def to_oracle(t):
    """torch tensor (any device) -> numpy input for the oracle (bf16 bits or fp32)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def np_u8(t):
    return t.detach().contiguous().cpu().numpy().view(np.uint8)


def np_f32(t):
    return t.detach().contiguous().cpu().float().numpy()


def assert_scales_equal(gpu, ref):
    g = np.ascontiguousarray(gpu, dtype=np.float32).view(np.uint32)
    r = np.ascontiguousarray(ref, dtype=np.float32).view(np.uint32)
    bad = np.argwhere(g != r)
    assert bad.size == 0, "scale bits differ at %s (gpu %r, oracle %r)" % (
        bad[:5].tolist(), gpu[tuple(bad[0])], ref[tuple(bad[0])])


def assert_codes_equal(gpu, ref):
    bad = np.argwhere(gpu != ref)
    assert bad.size == 0, "%d codes differ, first at %s: gpu 0x%02x oracle 0x%02x" % (
        len(bad), bad[0].tolist(), gpu[tuple(bad[0])], ref[tuple(bad[0])])


# GEMM acceptance: |C - C_ref| <= 1e-3 * T + 1e-6 for fp32 output, plus
# 4e-3 * |C_ref| for bf16 output (its own rounding is 2^-9 relative), where
# T = sum_k |a_k b_k| of the dequantized operands (fp64 oracle).
FP32_T_REL = 1e-3
BF16_REL = 4e-3
ABS = 1e-6


def gemm_bound(c_ref, T, out_dtype):
    bound = FP32_T_REL * T + ABS
    if out_dtype == torch.bfloat16:
        bound = bound + BF16_REL * np.abs(c_ref)
    return bound


def assert_gemm_within_bound(c_gpu, c_ref, T, out_dtype):
    c = np.asarray(c_gpu, dtype=np.float64)
    err = np.abs(c - c_ref)
    bound = gemm_bound(c_ref, T, out_dtype)
    assert np.all(np.isfinite(c)), "non-finite GEMM output"
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError("%d of %d entries outside the bound; worst at %s: gpu %r ref %r "
                             "T %r (err/bound %.3g)" % (bad.sum(), bad.size, i, c[i], c_ref[i],
                                                        T[i], (err / bound)[i]))
    return float(np.max(err / bound))


def bf16_quotient_sweep(amax_exps=(35, 36, 37, 100, 127, 160, 254), depth=20):
    """Structured bf16 inputs covering every (amax, x) mantissa pair.

    For each amax = 2^(e-127) (1 + m/128) (m = 0..127, e in amax_exps) the
    list holds amax first, then every bf16 x of either sign with exponent
    field in [e - depth, e] and |x| <= amax.  Quotients x / s reach down to
    amax 2^-(depth+1) / s, below the smallest E4M3 midpoint (2^-10).
    Returns a list of uint16 arrays (bf16 bit patterns), one per amax."""
    out = []
    mant = np.arange(128, dtype=np.uint16)
    for e in amax_exps:
        lo = max(1, e - depth)
        for m in range(128):
            amax = np.uint16((e << 7) | m)
            xs = []
            for ex in range(lo, e + 1):
                mm = mant if ex < e else mant[:m + 1]
                xs.append((np.uint16(ex) << 7) | mm)
            mag = np.concatenate(xs).astype(np.uint16)
            out.append(np.concatenate([[amax], mag, mag | np.uint16(0x8000)]).astype(np.uint16))
    return out

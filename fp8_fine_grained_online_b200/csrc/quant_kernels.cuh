// quant_kernels.cuh -- the per-element arithmetic of online fine-grained
// E4M3 quantization, shared by the streaming quantize kernels:
// scale = amax / 448 (IEEE fp32 division, 1 when zero) and
// code = E4M3_RNE_satfinite(x / scale), bit-exact to one IEEE fp32 division
// per element, evaluated as described at encode_pair (codingmall.com "Kan du
// förklara rollen för FP8 precision i träningsprocessen för DeepSeek-V3":
// "Finkornig kvantisering", "Online-kvantisering"; holysheep.ai "FP8 混精度训练
// DeepSeek 671B" (zh), 2.2).  Also the C = 0 kernel of an empty GEMM.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace fp8fg {

constexpr float kE4M3Max = 448.0f;

// max(a, b) per bf16 lane; a NaN lane yields the other operand (like fmaxf).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight consecutive input elements held as raw bits (one or two 16-byte
// words), converted to fp32 where they are used.
template <typename T>
struct Raw8;

template <>
struct Raw8<uint16_t> {  // bf16 bit patterns
    uint4 a;
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(u[i] << 16);           // exact bf16 -> fp32
            v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
        }
    }
    // The 8 elements negated, as 4 packed fp32 pairs (one IMAD / LOP3 per
    // element, like to_float).
    __device__ __forceinline__ void to_neg_pairs(uint64_t (&v)[4]) const {
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = f2_pack(__uint_as_float((u[i] << 16) ^ 0x80000000u),
                           __uint_as_float((u[i] & 0xFFFF0000u) ^ 0x80000000u));
    }
    // max |x| of the 8 elements (exact; NaN elements are skipped), on packed
    // bf16 pairs: clear the sign bits, then lane-wise maxima.
    __device__ __forceinline__ float abs_max() const {
        const uint32_t m = bf16x2_max(bf16x2_max(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                                      bf16x2_max(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu));
        return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    }
};

template <>
struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    __device__ __forceinline__ float abs_max() const {
        return fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))),
                     fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
    }
};

__device__ __forceinline__ float scale_from_amax(float amax) {
    float s = __fdiv_rn(amax, kE4M3Max);
    return s == 0.0f ? 1.0f : s;
}

// amax[j] = max |x| over tile j of the half-warp (all 16 lanes get it).
template <typename T, int kJ>
__device__ __forceinline__ void half_warp_amax(const Raw8<T> (&raw)[kJ], float (&amax)[kJ]);

// bf16: a tile maximum is an exact bf16 value, so two tiles travel in one
// register and are reduced with packed bf16 maxima.
template <int kJ>
__device__ __forceinline__ void half_warp_amax_bf16(const Raw8<uint16_t> (&raw)[kJ],
                                                    float (&amax)[kJ]) {
    static_assert(kJ % 2 == 0, "tiles are reduced in pairs");
#pragma unroll
    for (int j = 0; j < kJ; j += 2) {
        const uint32_t a0 = __float_as_uint(raw[j].abs_max()) >> 16;
        const uint32_t a1 = __float_as_uint(raw[j + 1].abs_max()) & 0xFFFF0000u;
        uint32_t m = a0 | a1;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1)
            m = bf16x2_max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        amax[j] = __uint_as_float(m << 16);
        amax[j + 1] = __uint_as_float(m & 0xFFFF0000u);
    }
}

template <int kJ>
__device__ __forceinline__ void half_warp_amax_f32(const Raw8<float> (&raw)[kJ],
                                                   float (&amax)[kJ]) {
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
        float a = raw[j].abs_max();
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        amax[j] = a;
    }
}

template <typename T, int kJ>
__device__ __forceinline__ void half_warp_amax(const Raw8<T> (&raw)[kJ], float (&amax)[kJ]) {
    if constexpr (sizeof(T) == 2)
        half_warp_amax_bf16<kJ>(raw, amax);
    else
        half_warp_amax_f32<kJ>(raw, amax);
}

// ---------------------------------------------------------------------------
// E4M3 code of the IEEE fp32 quotient x / s, without a division per element.
//
// The code must equal E(RN32(x / s)) where E is the (monotone, saturating,
// round-to-nearest-even) E4M3 conversion.  With r = RN32(1 / s) (the
// correctly rounded reciprocal, __frcp_rn), ru = RN32(r (1 + 2^-20)) and
// rd = RN32(r (1 - 2^-20)), the products u = RN32(x ru), d = RN32(x rd) carry
// three roundings of at most 2^-24 each on top of the 2^-20 offsets:
//   |u| >= |x/s| (1 + 2^-20 - 3.1 * 2^-24) > |x/s| (1 + 2^-24) >= |RN32(x/s)|,
//   |d| <= |x/s| (1 - 2^-20 + 3.1 * 2^-24) < |x/s| (1 - 2^-24) <= |RN32(x/s)|,
// all with the sign of x.  E is monotone, hence when E(u) == E(d) that
// common code is E(RN32(x/s)).  Otherwise x/s lies within ~2^-20 of an
// E4M3 rounding midpoint (~2e-5 of random fp32 inputs, but ~0.5% of bf16
// ones, many exactly on a midpoint) and the code is recomputed with IEEE
// division.  encode8_bracket is branch free (so that the multiply / convert
// chains of many elements interleave) and reports disagreeing pairs; the
// callers resolve only those pairs, one per iteration, with encode2_exact.
// The bounds need s and 1/s to be normal fp32 numbers: tiles whose scale is
// outside [2^-125, 2^125] use IEEE division throughout.  A quotient so small
// that u or d is subnormal encodes to +-0 at both ends, as RN32(x/s) does;
// zeros, NaN and the saturation at 448 carry through both ends unchanged.
// ---------------------------------------------------------------------------
constexpr float kBracketUp = 1.0f + 0x1p-20f;
constexpr float kBracketDown = 1.0f - 0x1p-20f;

__device__ __forceinline__ bool reciprocal_path_ok(float s) {
    return s >= 0x1p-125f && s <= 0x1p125f;
}

// Bracket-path codes of 8 values, branch free.  Bit k of the returned
// `amb` is set when the bracket ends disagree for elements 2k or 2k+1 (the
// quotient lies within ~2^-20 of an E4M3 rounding midpoint).  For bf16 data
// that is not rare: a quotient of two 8-bit mantissas times 448 lands
// exactly on a midpoint for ~0.5% of elements, so ambiguous pairs are
// resolved one by one (encode2_exact) rather than by recomputing tiles.
__device__ __forceinline__ uint2 encode8_bracket(const float (&v)[8], float ru, float rd,
                                                 uint32_t& amb) {
    uint32_t hi[4];
    amb = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t x2 = f2_pack(v[2 * k], v[2 * k + 1]);
        float u0, u1, d0, d1;
        f2_unpack(f2_mul(x2, f2_pack(ru, ru)), u0, u1);
        f2_unpack(f2_mul(x2, f2_pack(rd, rd)), d0, d1);
        hi[k] = cvt_e4m3x2(u0, u1);
        amb |= (hi[k] != cvt_e4m3x2(d0, d1) ? 1u : 0u) << k;
    }
    uint2 out;
    out.x = hi[0] | (hi[1] << 16);
    out.y = hi[2] | (hi[3] << 16);
    return out;
}

// ---------------------------------------------------------------------------
// bf16 inputs: a corrected quotient.  With r = RN32(1 / s) and n = -x:
//   q0 = RN32(n (-r)) = RN32(x r),
//   t  = RN32(q0 s + n) = RN32(q0 s - x)   (FMA; exact),
//   q1 = RN32(t (-r) + q0)                 (FMA),
// and the code is E(q1).  For every bf16 x with |x| <= amax and every bf16
// amax whose scale s = RN32(amax / 448) lies in [2^-100, 2^125], E(q1) equals
// E(RN32(x / s)), signs and signed zeros included: checked exhaustively over
// all such pairs (about 1e9), which is a complete proof for bf16 data
// because a tile's elements are bf16 values no larger than its amax.  (q1
// itself is not always the correctly rounded quotient, but where it
// differs the two lie on the same side of every E4M3 rounding boundary.)
// Working on n = -x keeps x = -0 at -0 through both FMAs (q0 - t r with
// q0 = -0 and t = +0 is -0), and costs nothing: the bf16 -> fp32 unpack of
// -x is as cheap as that of x.  Three packed operations and one convert per
// pair, branch free.  fp32 inputs, which the exhaustive check does not
// cover, take the bracket path below.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool corrected_path_ok(float s) {
    return s >= 0x1p-100f && s <= 0x1p125f;
}

// n: the 8 inputs negated, as 4 packed pairs; s2 = (s, s); neg_r2 = (-r, -r)
// with r = RN32(1 / s).
__device__ __forceinline__ uint2 encode8_corrected(const uint64_t (&n)[4], uint64_t s2,
                                                   uint64_t neg_r2) {
    uint32_t c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t q0 = f2_mul(n[k], neg_r2);           // x r
        const uint64_t t = f2_fma(q0, s2, n[k]);             // q0 s - x, exact
        const uint64_t q1 = f2_fma(t, neg_r2, q0);           // q0 - t r
        float lo, hi;
        f2_unpack(q1, lo, hi);
        c[k] = cvt_e4m3x2(lo, hi);
    }
    uint2 out;
    out.x = c[0] | (c[1] << 16);
    out.y = c[2] | (c[3] << 16);
    return out;
}

// As encode8_corrected with a scale per pair of values: s2[k] and neg_r2[k]
// pack the scales of values 2k and 2k+1 (per-column scales, 128x1 tiles).
__device__ __forceinline__ uint2 encode8_corrected_pairs(const uint64_t (&n)[4],
                                                         const uint64_t (&s2)[4],
                                                         const uint64_t (&neg_r2)[4]) {
    uint32_t c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t q0 = f2_mul(n[k], neg_r2[k]);
        const uint64_t t = f2_fma(q0, s2[k], n[k]);
        const uint64_t q1 = f2_fma(t, neg_r2[k], q0);
        float lo, hi;
        f2_unpack(q1, lo, hi);
        c[k] = cvt_e4m3x2(lo, hi);
    }
    uint2 out;
    out.x = c[0] | (c[1] << 16);
    out.y = c[2] | (c[3] << 16);
    return out;
}

// Codes of 2 values through IEEE fp32 division (the definition); the
// first value in the low byte.
__device__ __forceinline__ uint32_t encode2_exact(float x0, float x1, float s) {
    return cvt_e4m3x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
}

// Pair `idx` = 4 j + k (elements 2k, 2k+1 of raw[j]) as fp32, selected
// without indexing registers dynamically.
template <int kJ>
__device__ __forceinline__ void select_pair(const Raw8<uint16_t> (&raw)[kJ], int idx, float& x0,
                                            float& x1) {
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
        const uint32_t u[4] = {raw[j].a.x, raw[j].a.y, raw[j].a.z, raw[j].a.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (idx == 4 * j + k) w = u[k];
    }
    x0 = __uint_as_float(w << 16);
    x1 = __uint_as_float(w & 0xFFFF0000u);
}

template <int kJ>
__device__ __forceinline__ void select_pair(const Raw8<float> (&raw)[kJ], int idx, float& x0,
                                            float& x1) {
    x0 = 0.0f;
    x1 = 0.0f;
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
        const float u[8] = {raw[j].a.x, raw[j].a.y, raw[j].a.z, raw[j].a.w,
                            raw[j].b.x, raw[j].b.y, raw[j].b.z, raw[j].b.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (idx == 4 * j + k) {
                x0 = u[2 * k];
                x1 = u[2 * k + 1];
            }
    }
}

// Replace the 16-bit code pair k (bytes 2k, 2k+1) of an 8-code group.
__device__ __forceinline__ void patch_pair(uint2& codes, int k, uint32_t c16) {
    const uint32_t sh = (k & 1) * 16;
    const uint32_t keep = ~(0xFFFFu << sh);
    if (k < 2)
        codes.x = (codes.x & keep) | (c16 << sh);
    else
        codes.y = (codes.y & keep) | (c16 << sh);
}

// C = 0 for a GEMM with an empty contraction (K == 0).
template <typename T>
__global__ void __launch_bounds__(256)
    zero_rows_kernel(T* __restrict__ c, int64_t rows, int64_t cols, int64_t ldc) {
    const int64_t total = rows * cols;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / cols;
        c[r * ldc + (i - r * cols)] = T(0);
    }
}

}  // namespace fp8fg

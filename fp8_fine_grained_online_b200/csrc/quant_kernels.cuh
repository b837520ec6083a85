// quant_kernels.cuh -- online fine-grained E4M3 quantization kernels.
//
// Both kernels compute, per tile / block, scale = amax / 448 (IEEE fp32
// division, 1 when zero) and code = E4M3_RNE_satfinite(x / scale) with one
// IEEE fp32 division per element, evaluated as described at encode_pair
// (codingmall.com "Kan du förklara rollen
// för FP8 precision i träningsprocessen för DeepSeek-V3": "Finkornig
// kvantisering", "Online-kvantisering"; holysheep.ai "FP8 混精度训练
// DeepSeek 671B" (zh), 2.2).  They are HBM-bound: each input element is
// read once with 16-byte loads and each code written once.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace fp8fg {

constexpr float kE4M3Max = 448.0f;

// Eight consecutive input elements held as raw 16-byte loads, so that the
// next tile's loads can be issued before the current tile is converted.
template <typename T>
struct Raw8;

template <>
struct Raw8<uint16_t> {  // bf16 bit patterns
    uint4 a;
    __device__ __forceinline__ void load(const uint16_t* p) {
        a = __ldcs(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ void zero() { a = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(u[i] << 16);           // exact bf16 -> fp32
            v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
        }
    }
};

template <>
struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

__device__ __forceinline__ float scale_from_amax(float amax) {
    float s = __fdiv_rn(amax, kE4M3Max);
    return s == 0.0f ? 1.0f : s;
}

// ---------------------------------------------------------------------------
// E4M3 code of the IEEE fp32 quotient x / s, without a division per element.
//
// The code must equal E(RN32(x / s)) where E is the (monotone, saturating,
// round-to-nearest-even) E4M3 conversion.  With r = RN32(1 / s) (the
// correctly rounded reciprocal, __frcp_rn) and q = RN32(x * r):
//   |q - x/s| <= 2^-23 |x/s| (two roundings of 2^-24 each), and
//   |RN32(x/s) - x/s| <= 2^-24 |x/s|,
// so RN32(x/s) lies between q(1 - 2^-20) and q(1 + 2^-20).  E is monotone,
// hence when E(q(1 - 2^-20)) == E(q(1 + 2^-20)) that common code is
// E(RN32(x/s)).  Otherwise (x/s within ~2^-20 of an E4M3 rounding midpoint,
// a fraction ~2e-5 of inputs) the pair is recomputed with IEEE division.
// The bounds need s and 1/s to be normal fp32 numbers: tiles whose scale is
// outside [2^-125, 2^125] use IEEE division throughout.  Signs, zeros, NaN
// and the saturation at 448 carry through both ends unchanged.
// ---------------------------------------------------------------------------
constexpr float kBracketUp = 1.0f + 0x1p-20f;
constexpr float kBracketDown = 1.0f - 0x1p-20f;

__device__ __forceinline__ bool reciprocal_path_ok(float s) {
    return s >= 0x1p-125f && s <= 0x1p125f;
}

__device__ __forceinline__ uint32_t encode_pair(float x0, float x1, float s, float r) {
    const float q0 = x0 * r;
    const float q1 = x1 * r;
    const uint32_t hi = cvt_e4m3x2(q0 * kBracketUp, q1 * kBracketUp);
    const uint32_t lo = cvt_e4m3x2(q0 * kBracketDown, q1 * kBracketDown);
    if (hi == lo) return hi;
    return cvt_e4m3x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
}

// 8 values / scale -> 8 E4M3 codes packed little-endian in a uint2.
// `fast` selects the reciprocal path (reciprocal_path_ok(s)); r = 1/s.
__device__ __forceinline__ uint2 encode8(const float (&v)[8], float s, float r, bool fast) {
    uint2 out;
    if (fast) {
        out.x = encode_pair(v[0], v[1], s, r) | (encode_pair(v[2], v[3], s, r) << 16);
        out.y = encode_pair(v[4], v[5], s, r) | (encode_pair(v[6], v[7], s, r) << 16);
    } else {
        float d[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = __fdiv_rn(v[i], s);
        out.x = cvt_e4m3x2(d[0], d[1]) | (cvt_e4m3x2(d[2], d[3]) << 16);
        out.y = cvt_e4m3x2(d[4], d[5]) | (cvt_e4m3x2(d[6], d[7]) << 16);
    }
    return out;
}

// floor(n / d) for 0 <= n < 2^31 and a fixed d >= 1, by multiplication:
// with l = ceil(log2 d) and m = ceil(2^(31+l) / d), 2^(31+l) <= m d <=
// 2^(31+l) + 2^l, so floor(n / d) = (n m) >> (31 + l) (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994,
// round-up method).  m <= 2^32 keeps n m below 2^63.
struct FastDivU31 {
    uint64_t m;
    int shift;
    __host__ static FastDivU31 make(uint32_t d) {  // d < 2^31
        int l = 0;
        while ((static_cast<uint64_t>(1) << l) < d) ++l;
        FastDivU31 f;
        const uint64_t num = static_cast<uint64_t>(1) << (31 + l);  // l <= 31
        f.m = (num + d - 1) / d;
        f.shift = 31 + l;
        return f;
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        return static_cast<uint32_t>((static_cast<uint64_t>(n) * m) >> shift);
    }
};

// ---------------------------------------------------------------------------
// 1x128 activation tiles.  A half-warp owns one tile: lane l of the half
// loads elements [8l, 8l+8) of it, the tile amax is a 16-lane shuffle
// reduction, and each lane stores 8 codes.  A block of 256 threads handles
// 16 * kActUnroll consecutive tiles per step; the raw loads of the block's
// next step are issued before the current step is converted, so every lane
// keeps up to 2 * kActUnroll 16-byte loads in flight.
// ---------------------------------------------------------------------------
constexpr int kActThreads = 256;
// Tiles per half-warp per step: 4 for bf16 input, 2 for fp32 (same bytes).
template <typename T>
__host__ __device__ constexpr int act_unroll() { return sizeof(T) == 2 ? 4 : 2; }

// kSmall: M * nkb + step < 2^31, tile index -> (row, kb) by FastDivU31;
// otherwise 64-bit division.
template <typename T, bool kSmall>
__global__ void __launch_bounds__(kActThreads, 3)
    quant_act_1x128_kernel(const T* __restrict__ x, int64_t M, int64_t nkb, FastDivU31 fd,
                           int64_t ldx, uint8_t* __restrict__ q, int64_t ldq,
                           float* __restrict__ sa, int64_t sa_sm, int64_t sa_skb) {
    const int hl = threadIdx.x & 15;          // lane within the half-warp
    const int hw = threadIdx.x >> 4;          // half-warp within the block (0..15)
    constexpr int kActUnroll = act_unroll<T>();
    const int64_t total = M * nkb;
    const int64_t step = static_cast<int64_t>(gridDim.x) * (16 * kActUnroll);

    auto row_of = [&](int64_t t) -> int64_t {
        if (kSmall) return static_cast<int64_t>(fd.div(static_cast<uint32_t>(t)));
        return t / nkb;
    };
    auto load_step = [&](int64_t base, Raw8<T> (&raw)[kActUnroll]) {
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            const int64_t t = base + u * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                raw[u].load(x + row * ldx + (t - row * nkb) * 128 + hl * 8);
            } else {
                raw[u].zero();
            }
        }
    };

    Raw8<T> cur[kActUnroll], nxt[kActUnroll];
    int64_t base = static_cast<int64_t>(blockIdx.x) * (16 * kActUnroll);
    load_step(base, cur);
    for (; base < total; base += step) {
        load_step(base + step, nxt);
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            float v[8];
            cur[u].to_float(v);
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));  // NaN skipped
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
            const float s = scale_from_amax(amax);
            const float r = __frcp_rn(s);
            const int64_t t = base + u * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                const int64_t kb = t - row * nkb;
                const uint2 codes = encode8(v, s, r, reciprocal_path_ok(s));
                __stcs(reinterpret_cast<uint2*>(q + row * ldq + kb * 128 + hl * 8), codes);
                if (hl == 0) sa[row * sa_sm + kb * sa_skb] = s;
            }
        }
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) cur[u] = nxt[u];
    }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks.  One block of 256 threads owns one 128x128 block:
// thread (kq = tid/16, c = tid%16) holds rows {4kq..4kq+3, 64+4kq..64+4kq+3}
// and columns [8c, 8c+8).  The block amax is reduced through shared memory,
// then codes are written either directly ([K, N]) or through a shared
// transpose buffer ([N, K]).
// ---------------------------------------------------------------------------
constexpr int kWThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kWThreads, sizeof(T) == 2 ? 2 : 1)
    quant_weight_128x128_kernel(const T* __restrict__ w, int64_t nkb, int64_t nnb, int64_t ldw,
                                uint8_t* __restrict__ q, int transpose_out, int64_t ldq,
                                float* __restrict__ sb, int64_t sb_skb, int64_t sb_snb) {
    __shared__ float red[kWThreads / 32];
    __shared__ uint32_t tbuf[128][33];  // [n][k/4] words, one padding word per row

    const int tid = threadIdx.x;
    const int c = tid & 15;
    const int kq = tid >> 4;
    const int64_t nblocks = nkb * nnb;
    // Row of slot r (0..7) of this thread within a 128-row block.
    auto row_in_block = [&](int r) { return (r >> 2) * 64 + kq * 4 + (r & 3); };
    auto load_block = [&](int64_t blk, Raw8<T> (&raw)[8]) {
        const int64_t kb = blk / nnb;
        const int64_t nb = blk - kb * nnb;
        const T* src = w + (kb * 128) * ldw + nb * 128 + c * 8;
#pragma unroll
        for (int r = 0; r < 8; ++r) raw[r].load(src + row_in_block(r) * ldw);
    };

    Raw8<T> cur[8], nxt[8];
    int64_t blk = blockIdx.x;
    if (blk < nblocks) load_block(blk, cur);
    for (; blk < nblocks; blk += gridDim.x) {
        const int64_t kb = blk / nnb;
        const int64_t nb = blk - kb * nnb;
        if (blk + gridDim.x < nblocks) load_block(blk + gridDim.x, nxt);

        float amax = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float v[8];
            cur[r].to_float(v);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int i = 1; i < kWThreads / 32; ++i) amax = fmaxf(amax, red[i]);
        const float s = scale_from_amax(amax);
        const float rcp = __frcp_rn(s);
        const bool fast = reciprocal_path_ok(s);
        if (tid == 0) sb[kb * sb_skb + nb * sb_snb] = s;

        uint2 codes[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float v[8];
            cur[r].to_float(v);
            codes[r] = encode8(v, s, rcp, fast);
        }

        if (!transpose_out) {
            uint8_t* dst = q + (kb * 128) * ldq + nb * 128 + c * 8;
#pragma unroll
            for (int r = 0; r < 8; ++r)
                __stcs(reinterpret_cast<uint2*>(dst + row_in_block(r) * ldq), codes[r]);
        } else {
            // Gather, per column n, the 4 codes of rows 4kq..4kq+3 (and the
            // +64 group) into one word: tbuf[n][k/4].
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint32_t word = 0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint2 cj = codes[h * 4 + j];
                        const uint32_t half = (i < 4) ? cj.x : cj.y;
                        word |= ((half >> ((i & 3) * 8)) & 0xFFu) << (8 * j);
                    }
                    tbuf[c * 8 + i][h * 16 + kq] = word;
                }
            }
            __syncthreads();
            // Thread (n = tid/2, part = tid%2) writes 64 codes of row n of q^T.
            const int n = tid >> 1;
            const int part = tid & 1;
            uint8_t* dst = q + (nb * 128 + n) * ldq + kb * 128 + part * 64;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 o;
                o.x = tbuf[n][part * 16 + j * 4 + 0];
                o.y = tbuf[n][part * 16 + j * 4 + 1];
                o.z = tbuf[n][part * 16 + j * 4 + 2];
                o.w = tbuf[n][part * 16 + j * 4 + 3];
                __stcs(reinterpret_cast<uint4*>(dst) + j, o);
            }
        }
        __syncthreads();  // red[] and tbuf[] are reused by the next block
#pragma unroll
        for (int r = 0; r < 8; ++r) cur[r] = nxt[r];
    }
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

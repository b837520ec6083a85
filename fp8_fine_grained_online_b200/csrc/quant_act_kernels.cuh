// quant_act_kernels.cuh -- online 1x128 activation quantization
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"): every 1x128 tile of x [M, K] gets
// scale = amax / 448 and E4M3 codes of x / scale (see quant_kernels.cuh).
//
// HBM-bound; straight from registers.  A half-warp owns a tile (lane l of
// the half holds elements [8l, 8l+8) as one 16-byte load).  A block of 256
// threads takes kActTilesPerStep consecutive tiles per step: half-warp h
// gets tiles h, h+16, ..., so each lane issues kActTilesPerLane independent
// 16-byte loads before it needs any of them; latency is hidden by those and
// by occupancy (kActMinBlocks blocks per SM).  For its j-th tile the
// half-warp reduces amax with shuffles, the lanes l = j (mod
// kActTilesPerLane) compute the scale and reciprocal once, and the
// half-warp takes them by shuffle, so no lane divides per element.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "quant_kernels.cuh"

namespace fp8fg {

constexpr int kActThreads = 256;
constexpr int kActTilesPerLane = 4;                       // tiles a half-warp holds per step
constexpr int kActMinBlocks = 4;                          // resident blocks per SM
constexpr int kActTilesPerStep = 16 * kActTilesPerLane;   // 16 half-warps per block

template <typename T>
__device__ __forceinline__ void load_raw_global(const T* p, Raw8<T>& r);

template <>
__device__ __forceinline__ void load_raw_global<uint16_t>(const uint16_t* p, Raw8<uint16_t>& r) {
    r.a = __ldcs(reinterpret_cast<const uint4*>(p));
}

template <>
__device__ __forceinline__ void load_raw_global<float>(const float* p, Raw8<float>& r) {
    r.a = __ldcs(reinterpret_cast<const float4*>(p));
    r.b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
}

template <typename T>
__device__ __forceinline__ void zero_raw(Raw8<T>& r);
template <>
__device__ __forceinline__ void zero_raw<uint16_t>(Raw8<uint16_t>& r) { r.a = make_uint4(0u, 0u, 0u, 0u); }
template <>
__device__ __forceinline__ void zero_raw<float>(Raw8<float>& r) {
    r.a = r.b = make_float4(0.f, 0.f, 0.f, 0.f);
}

// kSmall: M * nkb + step < 2^31 (tile index -> row by FastDivU31).
template <typename T, bool kSmall>
__global__ void __launch_bounds__(kActThreads, kActMinBlocks)
    quant_act_1x128_kernel(const T* __restrict__ x, int64_t M, int64_t nkb, FastDivU31 fd,
                           int64_t ldx, uint8_t* __restrict__ q, int64_t ldq,
                           float* __restrict__ sa, int64_t sa_sm, int64_t sa_skb) {
    const int lane = threadIdx.x & 31;
    const int hl = threadIdx.x & 15;          // lane within the half-warp
    const int hw = threadIdx.x >> 4;          // half-warp within the block (0..15)
    const int half_base = lane & 16;
    const int64_t total = M * nkb;
    const int64_t step = static_cast<int64_t>(gridDim.x) * kActTilesPerStep;

    auto row_of = [&](int64_t t) -> int64_t {
        if (kSmall) return static_cast<int64_t>(fd.div(static_cast<uint32_t>(t)));
        return t / nkb;
    };
    auto load_step = [&](int64_t base, Raw8<T> (&raw)[kActTilesPerLane]) {
#pragma unroll
        for (int j = 0; j < kActTilesPerLane; ++j) {
            const int64_t t = base + j * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                load_raw_global<T>(x + row * ldx + (t - row * nkb) * 128 + hl * 8, raw[j]);
            } else {
                zero_raw<T>(raw[j]);
            }
        }
    };

    Raw8<T> cur[kActTilesPerLane];
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kActTilesPerStep; base < total;
         base += step) {
        load_step(base, cur);

        float amax[kActTilesPerLane];
        half_warp_amax<T, kActTilesPerLane>(cur, amax);
        float my_amax = amax[0];
#pragma unroll
        for (int j = 1; j < kActTilesPerLane; ++j)
            if (hl % kActTilesPerLane == j) my_amax = amax[j];
        const float my_s = scale_from_amax(my_amax);
        const float my_r = __frcp_rn(my_s);

        // Codes are stored tile by tile.  bf16 input takes the corrected
        // quotient; fp32 input the bracket, whose ambiguous pairs (bit
        // 4j + k: pair k of tile j) are then recomputed with IEEE division
        // and their two bytes overwritten.  Tiles with a scale off the fast
        // paths go through the same loop, all pairs.
        float sj[kActTilesPerLane];
        uint32_t amb = 0;
#pragma unroll
        for (int j = 0; j < kActTilesPerLane; ++j) {
            sj[j] = __shfl_sync(0xFFFFFFFFu, my_s, half_base + j);
            uint32_t amb4;
            uint2 codes;
            if constexpr (sizeof(T) == 2) {
                const float neg_r = __shfl_sync(0xFFFFFFFFu, -my_r, half_base + j);
                float n[8];
                cur[j].to_neg_float(n);
                codes = encode8_corrected(n, sj[j], neg_r);
                amb4 = corrected_path_ok(sj[j]) ? 0u : 0xFu;
            } else {
                const float ru = __shfl_sync(0xFFFFFFFFu, my_r * kBracketUp, half_base + j);
                const float rd = __shfl_sync(0xFFFFFFFFu, my_r * kBracketDown, half_base + j);
                float v[8];
                cur[j].to_float(v);
                codes = encode8_bracket(v, ru, rd, amb4);
                if (!reciprocal_path_ok(sj[j])) amb4 = 0xFu;
            }
            const int64_t t = base + j * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                const int64_t kb = t - row * nkb;
                __stcs(reinterpret_cast<uint2*>(q + row * ldq + kb * 128 + hl * 8), codes);
                if (hl == j) sa[row * sa_sm + kb * sa_skb] = sj[j];
                amb |= amb4 << (4 * j);
            }
        }
        while (amb != 0) {
            const int idx = __ffs(amb) - 1;
            amb &= amb - 1;
            const int j = idx >> 2;
            float x0, x1, s = sj[0];
            select_pair<kActTilesPerLane>(cur, idx, x0, x1);
#pragma unroll
            for (int jj = 1; jj < kActTilesPerLane; ++jj)
                if (j == jj) s = sj[jj];
            const int64_t t = base + j * 16 + hw;
            const int64_t row = row_of(t);
            const int64_t kb = t - row * nkb;
            *reinterpret_cast<uint16_t*>(q + row * ldq + kb * 128 + hl * 8 + 2 * (idx & 3)) =
                static_cast<uint16_t>(encode2_exact(x0, x1, s));
        }
    }
}

}  // namespace fp8fg

// quant_act_kernels.cuh -- online 1x128 activation quantization
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"): every 1x128 tile of x [M, K] gets
// scale = amax / 448 and E4M3 codes of x / scale (see quant_kernels.cuh).
//
// HBM-bound; straight from registers.  A half-warp owns a tile (lane l of
// the half holds elements [8l, 8l+8) as one 16-byte load).  A block of 256
// threads takes 128 consecutive tiles per step: half-warp h gets tiles
// h, h+16, ..., h+112, so each lane issues 8 independent 16-byte loads
// before it needs any of them; latency is hidden by those and by occupancy
// (two blocks, 16 warps per SM).  For its j-th tile the half-warp reduces
// amax with shuffles, lanes j and j+8 compute the scale and reciprocal once,
// and the half-warp takes them by shuffle, so no lane divides per element.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "quant_kernels.cuh"
#include "quant_stream_kernels.cuh"   // row_amax8

namespace fp8fg {

constexpr int kActThreads = 256;
constexpr int kActTilesPerStep = 128;

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
__global__ void __launch_bounds__(kActThreads, 2)
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
    auto load_step = [&](int64_t base, Raw8<T> (&raw)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t t = base + j * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                load_raw_global<T>(x + row * ldx + (t - row * nkb) * 128 + hl * 8, raw[j]);
            } else {
                zero_raw<T>(raw[j]);
            }
        }
    };

    Raw8<T> cur[8];
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kActTilesPerStep; base < total;
         base += step) {
        load_step(base, cur);

        float amax[8];
        row_amax8<T>(cur, amax);
        float my_amax = amax[0];
#pragma unroll
        for (int j = 1; j < 8; ++j)
            if ((hl & 7) == j) my_amax = amax[j];
        const float my_s = scale_from_amax(my_amax);
        const float my_r = __frcp_rn(my_s);
        const float my_ru = my_r * kBracketUp;
        const float my_rd = my_r * kBracketDown;

        float sj[8];
        uint32_t bad = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sj[j] = __shfl_sync(0xFFFFFFFFu, my_s, half_base + j);
            const float ru = __shfl_sync(0xFFFFFFFFu, my_ru, half_base + j);
            const float rd = __shfl_sync(0xFFFFFFFFu, my_rd, half_base + j);
            bad |= reciprocal_path_ok(sj[j]) ? 0u : 1u;
            float v[8];
            cur[j].to_float(v);
            const uint2 codes = encode8_bracket(v, ru, rd, bad);
            const int64_t t = base + j * 16 + hw;
            if (t < total) {
                const int64_t row = row_of(t);
                const int64_t kb = t - row * nkb;
                __stcs(reinterpret_cast<uint2*>(q + row * ldq + kb * 128 + hl * 8), codes);
                if (hl == j) sa[row * sa_sm + kb * sa_skb] = sj[j];
            }
        }
        if (bad != 0) {    // rare: recompute this thread's tiles with IEEE division
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t t = base + j * 16 + hw;
                if (t < total) {
                    float v[8];
                    cur[j].to_float(v);
                    const int64_t row = row_of(t);
                    __stcs(reinterpret_cast<uint2*>(q + row * ldq + (t - row * nkb) * 128 + hl * 8),
                           encode8_exact(v, sj[j]));
                }
            }
        }
    }
}

}  // namespace fp8fg

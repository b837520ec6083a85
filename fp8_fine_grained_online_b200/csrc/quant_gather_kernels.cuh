// quant_gather_kernels.cuh -- 1x128 activation quantization fused with the
// row gather that sorts MoE tokens by expert: output row r is the
// quantization of input row rows[r] (codingmall.com "Kan du förklara rollen
// för FP8 precision i träningsprocessen för DeepSeek-V3", "Finkornig
// kvantisering", "Online-kvantisering"; the permutation is the routing's),
// so the expert-sorted bf16 copy of the activations is never written.
// Codes and scales are bit-identical to gathering the rows and then calling
// the 1x128 quantizer.
//
// HBM/L2-bound, straight from registers: a half-warp owns one output row at
// a time and walks its 1x128 tiles kGqTilesPerLane at a time (lane l of the
// half holds elements [8l, 8l+8) of each tile: one 16-byte load per tile,
// all issued before the first is used).  Per tile the half-warp reduces
// amax with shuffles, lanes l = j (mod kGqTilesPerLane) compute tile j's
// scale and reciprocal once and share them by shuffle; bf16 input is
// encoded through the corrected quotient, fp32 through the bracket with
// ambiguous pairs recomputed by IEEE division (quant_kernels.cuh).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "gemm_kernels.cuh"   // record_device_error, kDevErrShape
#include "quant_kernels.cuh"

namespace fp8fg {

constexpr int kGqThreads = 256;
constexpr int kGqTilesPerLane = 4;     // tiles of one row in flight per half-warp
constexpr int kGqMinBlocks = 4;        // resident blocks per SM

template <typename T>
__device__ __forceinline__ void load_raw_global(const T* p, Raw8<T>& r);

template <>
__device__ __forceinline__ void load_raw_global<uint16_t>(const uint16_t* p, Raw8<uint16_t>& r) {
    r.a = __ldg(reinterpret_cast<const uint4*>(p));
}

template <>
__device__ __forceinline__ void load_raw_global<float>(const float* p, Raw8<float>& r) {
    r.a = __ldg(reinterpret_cast<const float4*>(p));
    r.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
}

template <typename T>
__device__ __forceinline__ void zero_raw(Raw8<T>& r);
template <>
__device__ __forceinline__ void zero_raw<uint16_t>(Raw8<uint16_t>& r) {
    r.a = make_uint4(0u, 0u, 0u, 0u);
}
template <>
__device__ __forceinline__ void zero_raw<float>(Raw8<float>& r) {
    r.a = r.b = make_float4(0.f, 0.f, 0.f, 0.f);
}

template <typename T>
__global__ void __launch_bounds__(kGqThreads, kGqMinBlocks)
    quant_gather_kernel(const T* __restrict__ x, int64_t src_rows, int64_t ldx,
                        const int32_t* __restrict__ rows, int64_t R, int64_t nkb,
                        uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sa,
                        int64_t sa_sm, int64_t sa_skb) {
    constexpr int J = kGqTilesPerLane;
    const int lane = threadIdx.x & 31;
    const int hl = threadIdx.x & 15;                     // lane within the half-warp
    const int half_base = lane & 16;
    // A warp takes output rows (r2, r2 + 1), one per half-warp, so that both
    // halves run the same loop trips (the shuffles need the whole warp); a
    // half with no row, or an invalid index, works on zeros and stores nothing.
    const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * kGqThreads + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kGqThreads) >> 5;

    for (int64_t r2 = 2 * warp_id; r2 < R; r2 += 2 * n_warps) {
        const int64_t r = r2 + (half_base >> 4);
        bool valid = r < R;
        int64_t src = 0;
        if (valid) {
            src = __ldg(rows + r);
            if (src < 0 || src >= src_rows) {
                if (hl == 0) record_device_error(kDevErrShape);
                valid = false;
                src = 0;
            }
        }
        const T* xrow = x + src * ldx + hl * 8;
        uint8_t* qrow = q + (valid ? r : 0) * ldq + hl * 8;
        float* srow = sa + (valid ? r : 0) * sa_sm;
        for (int64_t kb0 = 0; kb0 < nkb; kb0 += J) {
            Raw8<T> cur[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                if (valid && kb0 + j < nkb)
                    load_raw_global<T>(xrow + (kb0 + j) * 128, cur[j]);
                else
                    zero_raw<T>(cur[j]);
            }
            float amax[J];
            half_warp_amax<T, J>(cur, amax);
            float my_amax = amax[0];
#pragma unroll
            for (int j = 1; j < J; ++j)
                if (hl % J == j) my_amax = amax[j];
            const float my_s = scale_from_amax(my_amax);
            const float my_r = __frcp_rn(my_s);

            float sj[J];
            uint32_t amb = 0;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                sj[j] = __shfl_sync(0xFFFFFFFFu, my_s, half_base + j);
                uint32_t amb4;
                uint2 codes;
                if constexpr (sizeof(T) == 2) {
                    const float neg_r = __shfl_sync(0xFFFFFFFFu, -my_r, half_base + j);
                    uint64_t n[4];
                    cur[j].to_neg_pairs(n);
                    codes = encode8_corrected(n, f2_pack(sj[j], sj[j]), f2_pack(neg_r, neg_r));
                    amb4 = corrected_path_ok(sj[j]) ? 0u : 0xFu;
                } else {
                    const float ru = __shfl_sync(0xFFFFFFFFu, my_r * kBracketUp, half_base + j);
                    const float rd = __shfl_sync(0xFFFFFFFFu, my_r * kBracketDown, half_base + j);
                    float v[8];
                    cur[j].to_float(v);
                    codes = encode8_bracket(v, ru, rd, amb4);
                    if (!reciprocal_path_ok(sj[j])) amb4 = 0xFu;
                }
                if (valid && kb0 + j < nkb) {
                    __stcs(reinterpret_cast<uint2*>(qrow + (kb0 + j) * 128), codes);
                    if (hl == j) srow[(kb0 + j) * sa_skb] = sj[j];
                    amb |= amb4 << (4 * j);
                }
            }
            while (amb != 0) {     // pairs the fast paths leave open: IEEE division
                const int idx = __ffs(amb) - 1;
                amb &= amb - 1;
                const int j = idx >> 2;
                float x0, x1, sv = sj[0];
                select_pair<J>(cur, idx, x0, x1);
#pragma unroll
                for (int jj = 1; jj < J; ++jj)
                    if (j == jj) sv = sj[jj];
                *reinterpret_cast<uint16_t*>(qrow + (kb0 + j) * 128 + 2 * (idx & 3)) =
                    static_cast<uint16_t>(encode2_exact(x0, x1, sv));
            }
        }
    }
}

}  // namespace fp8fg

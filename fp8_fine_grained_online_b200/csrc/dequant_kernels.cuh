// dequant_kernels.cuh -- E4M3 codes back to real values: each code's E4M3
// value times its tile's scale (holysheep.ai "FP8 混精度训练 DeepSeek 671B"
// (zh), 2.2: dequantize = code value x scale), in one IEEE fp32 multiply,
// written as fp32 or rounded to bf16 (nearest even).  Tiles are 1x128
// (activation scales sa[m, kb]) or 128x128 (weight scales sb[kb, nb]).
//
// HBM-bound: 1 byte read and 2 or 4 bytes written per element.  A thread
// takes 8 consecutive codes of a row (an 8-byte load; a warp reads 256
// contiguous bytes and, for bf16, stores 512 as whole 32-byte sectors) and
// kDqRowsInFlight rows at a time, all loads issued before the first is
// used, so that enough bytes are in flight per SM to cover HBM latency.
// Block (x, y): 2048 codes of the rows y, y + gridDim.y, ...  The scale row
// of code row r is r >> tile_shift (tile_shift = log2 of the tile height:
// 0 for 1x128 tiles, 7 for 128x128 blocks).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fp8fg {

constexpr int kDqThreads = 256;
constexpr int kDqCodesPerThread = 8;
constexpr int kDqCodesPerBlock = kDqThreads * kDqCodesPerThread;
constexpr int kDqRowsInFlight = 8;
constexpr int kDqBlocksPerSm = 4;   // 32 warps, 64 KB of loads in flight per SM

// Two E4M3 codes (low byte first) -> two fp32 values, exactly (every E4M3
// value is an f16 value; NaN codes give NaN).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    float lo, hi;
    asm("{\n\t.reg .f16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\t"
        "cvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return make_float2(lo, hi);
}

template <bool kOutBf16>
__device__ __forceinline__ void dequant_store8(uint2 codes, float sc, void* out, int64_t off) {
    const uint32_t w[2] = {codes.x, codes.y};
    float v[8];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float2 a = e4m3x2_to_float2(static_cast<uint16_t>(w[i] & 0xFFFFu));
        const float2 b = e4m3x2_to_float2(static_cast<uint16_t>(w[i] >> 16));
        v[4 * i + 0] = __fmul_rn(a.x, sc);
        v[4 * i + 1] = __fmul_rn(a.y, sc);
        v[4 * i + 2] = __fmul_rn(b.x, sc);
        v[4 * i + 3] = __fmul_rn(b.y, sc);
    }
    if (kOutBf16) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            o[i] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        __stcs(reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + off),
               make_uint4(o[0], o[1], o[2], o[3]));
    } else {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
        __stcs(dst, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(dst + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
}

template <bool kOutBf16>
__global__ void __launch_bounds__(kDqThreads, kDqBlocksPerSm)
    dequant_kernel(const uint8_t* __restrict__ q, int64_t rows, int64_t cols, int64_t ldq,
                   const float* __restrict__ s, int64_t s_stride_r, int64_t s_stride_c,
                   int tile_shift, void* __restrict__ out, int64_t ldo) {
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kDqCodesPerBlock +
                       threadIdx.x * kDqCodesPerThread;
    if (c0 >= cols) return;
    const float* s_col = s + (c0 >> 7) * s_stride_c;
    const int64_t step = gridDim.y;
    for (int64_t r0 = blockIdx.y; r0 < rows; r0 += step * kDqRowsInFlight) {
        uint2 codes[kDqRowsInFlight];
        float sc[kDqRowsInFlight];
#pragma unroll
        for (int i = 0; i < kDqRowsInFlight; ++i) {
            const int64_t r = r0 + i * step;
            if (r < rows) {
                codes[i] = __ldcs(reinterpret_cast<const uint2*>(q + r * ldq + c0));
                sc[i] = __ldg(s_col + (r >> tile_shift) * s_stride_r);
            }
        }
#pragma unroll
        for (int i = 0; i < kDqRowsInFlight; ++i) {
            const int64_t r = r0 + i * step;
            if (r < rows) dequant_store8<kOutBf16>(codes[i], sc[i], out, r * ldo + c0);
        }
    }
}

}  // namespace fp8fg

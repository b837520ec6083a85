// quant_stream_kernels.cuh -- online fine-grained E4M3 quantization streamed
// through shared memory by TMA.
//
// Activations: every 1x128 tile of x [M, K] gets scale = amax / 448;
// weights: every 128x128 block of w [K, N] gets scale = amax / 448
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"; holysheep.ai "FP8 混精度训练 DeepSeek 671B" (zh),
// 2.2).  Codes are E4M3_RNE_satfinite(x / scale), bit-exact to IEEE fp32
// division (see encode_pair).
//
// Both are HBM-bound.  One persistent CTA per SM with two groups of 8
// warps.  Group g takes the CTA's boxes g, g+2, ... of 128x128 input
// elements; each group owns two shared-memory slots (one for fp32 input)
// that its first thread fills by TMA.  For every box the group copies its
// slot to registers, meets at a group barrier, and the slot is refilled with
// the group's box two ahead while the group computes the scales, encodes and
// writes codes and scales; so HBM reads overlap the arithmetic of both
// groups.
//
// Consumer thread (kq = t / 16, c = t % 16) of its group holds rows
// {4kq .. 4kq+3, 64+4kq .. 64+4kq+3} of the box, columns [8c, 8c+8).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_kernels.cuh"   // bounded_wait, drain_wait, record_device_error
#include "quant_kernels.cuh"  // Raw8, encode8, scale_from_amax, reciprocal_path_ok

namespace fp8fg {

enum QuantMode { kQuantAct = 0, kQuantWeight = 1, kQuantWeightT = 2 };

constexpr int kQsGroups = 2;                 // consumer groups of 8 warps
constexpr int kQsThreads = kQsGroups * 256;

template <typename T>
struct QsCfg {
    static constexpr int kSlots = sizeof(T) == 2 ? 2 : 1;   // ring slots per group
    static constexpr int kStages = kQsGroups * kSlots;
    static constexpr int kBoxBytes = 128 * 128 * static_cast<int>(sizeof(T));
    static constexpr int kRowBytes = 128 * static_cast<int>(sizeof(T));
};

struct QsSmemTail {
    uint64_t full[4];                  // slot filled (TMA bytes)
    uint64_t gbar[kQsGroups];          // per-group barrier (8 warp arrivals)
    float red[kQsGroups][2][8];        // [group][block parity][warp]
    uint32_t tbuf[kQsGroups][128][33]; // [group][n][k/4], transposed codes
    int abort_flag;
};

template <typename T>
constexpr size_t quant_stream_smem_bytes() {
    return 1024 + QsCfg<T>::kStages * QsCfg<T>::kBoxBytes + sizeof(QsSmemTail);
}

struct QsParams {
    int64_t rows, cols;        // input [rows, cols]; act: [M, K], weight: [K, N]
    int64_t nbr, nbc;          // boxes along rows / cols
    uint8_t* q;
    int64_t ldq;
    float* s;
    int64_t s_stride_r, s_stride_c;   // act: (m, kb); weight: (kb, nb)
};

// Barrier of one consumer group (its 8 warps) through an mbarrier, so that
// the wait is bounded like every other wait of the kernel.  `uses` counts
// this thread's passes (the phase parity).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& uses, int lane,
                                           volatile int* abort_flag) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
    const bool ok = bounded_wait(bar, uses & 1u, abort_flag);
    ++uses;
    return ok;
}

// 16-byte shared-memory load (input elements staged by TMA).
__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

template <typename T>
__device__ __forceinline__ void load_raw_smem(const uint8_t* row_base, int c, Raw8<T>& r);

template <>
__device__ __forceinline__ void load_raw_smem<uint16_t>(const uint8_t* row_base, int c,
                                                        Raw8<uint16_t>& r) {
    r.a = lds128(row_base + c * 16);
}

template <>
__device__ __forceinline__ void load_raw_smem<float>(const uint8_t* row_base, int c,
                                                     Raw8<float>& r) {
    const uint4 a = lds128(row_base + c * 32);
    const uint4 b = lds128(row_base + c * 32 + 16);
    r.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z),
                      __uint_as_float(a.w));
    r.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z),
                      __uint_as_float(b.w));
}

// 4x4 byte transpose: w[e] = byte e of r0 | byte e of r1 << 8 | ... (PRMT).
__device__ __forceinline__ void transpose4x4_bytes(uint32_t r0, uint32_t r1, uint32_t r2,
                                                   uint32_t r3, uint32_t (&w)[4]) {
    const uint32_t t0 = __byte_perm(r0, r1, 0x5140);   // r0.b0 r1.b0 r0.b1 r1.b1
    const uint32_t t1 = __byte_perm(r0, r1, 0x7362);   // r0.b2 r1.b2 r0.b3 r1.b3
    const uint32_t t2 = __byte_perm(r2, r3, 0x5140);
    const uint32_t t3 = __byte_perm(r2, r3, 0x7362);
    w[0] = __byte_perm(t0, t2, 0x5410);
    w[1] = __byte_perm(t0, t2, 0x7632);
    w[2] = __byte_perm(t1, t3, 0x5410);
    w[3] = __byte_perm(t1, t3, 0x7632);
}

// Per-row amax of 8 rows held by a half-warp (16 lanes x 8 elements per
// row): every lane gets all eight row maxima.
template <typename T>
__device__ __forceinline__ void row_amax8(const Raw8<T> (&raw)[8], float (&amax)[8]);

// bf16: a row maximum is an exact bf16 value, so two rows travel in one
// register and are reduced with packed bf16 maxima.
template <>
__device__ __forceinline__ void row_amax8<uint16_t>(const Raw8<uint16_t> (&raw)[8],
                                                    float (&amax)[8]) {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const uint32_t a0 = __float_as_uint(raw[j].abs_max()) >> 16;        // bf16 bits
        const uint32_t a1 = __float_as_uint(raw[j + 1].abs_max()) & 0xFFFF0000u;
        uint32_t m = a0 | a1;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1)
            m = bf16x2_max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        amax[j] = __uint_as_float(m << 16);
        amax[j + 1] = __uint_as_float(m & 0xFFFF0000u);
    }
}

template <>
__device__ __forceinline__ void row_amax8<float>(const Raw8<float> (&raw)[8], float (&amax)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a = raw[j].abs_max();
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        amax[j] = a;
    }
}

template <typename T, int kMode>
__global__ void __launch_bounds__(kQsThreads, 1)
    quant_stream_kernel(const __grid_constant__ CUtensorMap tm_in, const QsParams p) {
    constexpr int kSlots = QsCfg<T>::kSlots;
    constexpr int kStages = QsCfg<T>::kStages;
    constexpr int kBoxBytes = QsCfg<T>::kBoxBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    QsSmemTail* tail = reinterpret_cast<QsSmemTail*>(smem + kStages * kBoxBytes);
    volatile int* abort_flag = &tail->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nboxes = p.nbr * p.nbc;
    // This CTA's boxes: blockIdx.x + i * gridDim.x, i = 0 .. count-1.
    const int64_t count = nboxes > blockIdx.x ? (nboxes - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&tail->full[s], 1);
        for (int gi = 0; gi < kQsGroups; ++gi) mbar_init(&tail->gbar[gi], 8);
        tail->abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_in);
    }
    __syncthreads();

    const int g = warp >> 3;                 // group
    const int t = threadIdx.x & 255;         // thread within the group
    const int wg = t >> 5;                   // warp within the group
    const int kq = t >> 4;
    const int c = t & 15;
    auto row_in_box = [&](int j) { return (j >> 2) * 64 + kq * 4 + (j & 3); };
    uint32_t gbar_uses = 0;

    // Group g owns the CTA's boxes i = g + kQsGroups * k (k = 0, 1, ...) and
    // ring slots g * kSlots .. g * kSlots + kSlots - 1: its k-th box lands in
    // slot g * kSlots + k % kSlots.  Thread 0 of the group issues the loads;
    // a slot is refilled once the whole group has read it.
    auto box_of = [&](int64_t k) { return g + kQsGroups * k; };
    auto slot_of = [&](int64_t k) { return g * kSlots + static_cast<int>(k % kSlots); };
    auto issue = [&](int64_t k) {
        const int64_t box = blockIdx.x + box_of(k) * gridDim.x;
        const int64_t br = box / p.nbc;
        const int64_t bc = box - br * p.nbc;
        const int slot = slot_of(k);
        mbar_arrive_expect_tx(&tail->full[slot], kBoxBytes);
        tma_load_2d(smem + slot * kBoxBytes, &tm_in, &tail->full[slot],
                    static_cast<int32_t>(bc * 128), static_cast<int32_t>(br * 128));
    };
    if (t == 0)
        for (int64_t k = 0; k < kSlots && box_of(k) < count; ++k) issue(k);

    for (int64_t k = 0; box_of(k) < count; ++k) {
        const int64_t i = box_of(k);
        const int stage = slot_of(k);
        const uint32_t phase = static_cast<uint32_t>((k / kSlots) & 1);
        if (!bounded_wait(&tail->full[stage], phase, abort_flag)) break;
        const uint8_t* box_smem = smem + stage * kBoxBytes;
        auto row_ptr = [&](int j) { return box_smem + row_in_box(j) * QsCfg<T>::kRowBytes; };
        // The group has finished reading the slot: refill it with the
        // group's box k + kSlots.
        auto release_stage = [&]() -> bool {
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) return false;
            if (t == 0 && box_of(k + kSlots) < count) issue(k + kSlots);
            return true;
        };
        const int64_t box = blockIdx.x + i * gridDim.x;
        const int64_t br = box / p.nbc;
        const int64_t bc = box - br * p.nbc;

        if (kMode == kQuantAct) {
            // One 1x128 tile per row: the 16 lanes of a half-warp share a row.
            // Lane c computes the scale of row slot (c & 7) once; the half-
            // warp shares the eight scales by shuffle.
            const int half_base = lane & 16;
            Raw8<T> raw[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) load_raw_smem<T>(row_ptr(j), c, raw[j]);
            if (!release_stage()) break;
            float amax[8];
            row_amax8<T>(raw, amax);
            float my_amax = amax[0];
#pragma unroll
            for (int j = 1; j < 8; ++j)
                if ((c & 7) == j) my_amax = amax[j];
            const float my_s = scale_from_amax(my_amax);
            const float my_r = __frcp_rn(my_s);
            const float my_ru = my_r * kBracketUp;
            const float my_rd = my_r * kBracketDown;
            // Codes are stored row by row; in the rare case of a bracket
            // disagreement (or a scale off the reciprocal path) the thread
            // recomputes its rows with IEEE division and overwrites them.
            float sj[8];
            uint32_t bad = 0;
            uint8_t* qrow0 = p.q + (br * 128) * p.ldq + bc * 128 + c * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sj[j] = __shfl_sync(0xFFFFFFFFu, my_s, half_base + j);
                const float ru = __shfl_sync(0xFFFFFFFFu, my_ru, half_base + j);
                const float rd = __shfl_sync(0xFFFFFFFFu, my_rd, half_base + j);
                bad |= reciprocal_path_ok(sj[j]) ? 0u : 1u;
                float v[8];
                raw[j].to_float(v);
                const uint2 codes = encode8_bracket(v, ru, rd, bad);
                const int r = row_in_box(j);
                if (br * 128 + r < p.rows) {
                    __stcs(reinterpret_cast<uint2*>(qrow0 + r * p.ldq), codes);
                    if (c == j) p.s[(br * 128 + r) * p.s_stride_r + bc * p.s_stride_c] = sj[j];
                }
            }
            if (bad != 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v[8];
                    raw[j].to_float(v);
                    const int r = row_in_box(j);
                    if (br * 128 + r < p.rows)
                        __stcs(reinterpret_cast<uint2*>(qrow0 + r * p.ldq), encode8_exact(v, sj[j]));
                }
            }
        } else {
            // One scale for the whole 128x128 box: an amax pass over the box
            // in shared memory, a block reduction, then an encode pass.
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                Raw8<T> r;
                load_raw_smem<T>(row_ptr(j), c, r);
                a = fmaxf(a, r.abs_max());
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            const int par = static_cast<int>((i / kQsGroups) & 1);
            if (lane == 0) tail->red[g][par][wg] = a;
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
            a = tail->red[g][par][0];
#pragma unroll
            for (int w = 1; w < 8; ++w) a = fmaxf(a, tail->red[g][par][w]);
            const float s = scale_from_amax(a);
            const float rcp = __frcp_rn(s);
            const float ru = rcp * kBracketUp;
            const float rd = rcp * kBracketDown;
            const uint32_t off_path = reciprocal_path_ok(s) ? 0u : 1u;
            if (t == 0) p.s[br * p.s_stride_r + bc * p.s_stride_c] = s;
            uint32_t(*tb)[33] = tail->tbuf[g];
#pragma unroll
            for (int h4 = 0; h4 < 2; ++h4) {
                Raw8<T> raw[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) load_raw_smem<T>(row_ptr(h4 * 4 + jj), c, raw[jj]);
                if (h4 == 1 && !release_stage()) break;
                uint2 codes[4];
                uint32_t bad = off_path;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    float v[8];
                    raw[jj].to_float(v);
                    codes[jj] = encode8_bracket(v, ru, rd, bad);
                }
                if (bad != 0) {    // rare: recompute these rows exactly
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float v[8];
                        raw[jj].to_float(v);
                        codes[jj] = encode8_exact(v, s);
                    }
                }
                if (kMode == kQuantWeight) {
                    uint8_t* dst = p.q + (br * 128) * p.ldq + bc * 128 + c * 8;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        __stcs(reinterpret_cast<uint2*>(dst + row_in_box(h4 * 4 + jj) * p.ldq),
                               codes[jj]);
                } else {
                    // Transposed output [N, K]: per column n, the codes of rows
                    // 4kq..4kq+3 (+64 h4) form one word of tbuf[n][k/4]; a 4x4
                    // byte transpose of each half of the four rows' codes.
                    uint32_t wx[4], wy[4];
                    transpose4x4_bytes(codes[0].x, codes[1].x, codes[2].x, codes[3].x, wx);
                    transpose4x4_bytes(codes[0].y, codes[1].y, codes[2].y, codes[3].y, wy);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        tb[c * 8 + e][h4 * 16 + kq] = wx[e];
                        tb[c * 8 + 4 + e][h4 * 16 + kq] = wy[e];
                    }
                }
            }
            if (*abort_flag) break;
            if (kMode == kQuantWeightT) {
                if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
                const int n = t >> 1;
                const int part = t & 1;
                uint8_t* dst = p.q + (bc * 128 + n) * p.ldq + br * 128 + part * 64;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 o;
                    o.x = tb[n][part * 16 + j * 4 + 0];
                    o.y = tb[n][part * 16 + j * 4 + 1];
                    o.z = tb[n][part * 16 + j * 4 + 2];
                    o.w = tb[n][part * 16 + j * 4 + 3];
                    __stcs(reinterpret_cast<uint4*>(dst) + j, o);
                }
                // tbuf is rewritten for the next box
                if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
            }
        }
    }
    // After an abandoned wait a refill may still be in flight: let it land
    // before the CTA leaves (every fill is consumed on the normal path).
    if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 22)) {
        }
    }
}

}  // namespace fp8fg

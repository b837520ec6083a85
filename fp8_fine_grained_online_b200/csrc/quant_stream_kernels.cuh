// quant_stream_kernels.cuh -- online fine-grained E4M3 quantization streamed
// through shared memory by TMA, in four modes:
//   activations: every 1x128 tile of x [M, K] gets its own scale;
//   weights:     every 128x128 block of w [K, N] gets its own scale, codes
//                written [K, N] as given, or transposed to [N, K] (K
//                contiguous, the GEMM's B operand layout);
//   activations along M (bf16): every 128x1 tile of x [M, K] (128 rows of
//                one column) gets its own scale, codes written transposed
//                to [K, M]: the 1x128 tiles of x^T that the weight gradient
//                x^T dY contracts over.
// scale = amax / 448 and codes E4M3_RNE_satfinite(x / scale), bit-exact to
// IEEE fp32 division (see encode8_corrected, encode8_bracket)
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"; holysheep.ai "FP8 混精度训练 DeepSeek 671B" (zh),
// 2.2).
//
// HBM-bound.  One persistent CTA per SM with two groups of 8 warps.  Group
// g takes the CTA's boxes g, g+2, ... of 128x128 input elements; each group
// owns two shared-memory slots (one for fp32 input) that its first thread
// fills by TMA; the slot is refilled with the group's box two ahead as soon
// as the group has taken the box into registers (weights: its second half,
// after the amax pass), so HBM reads overlap the arithmetic of both groups.
//
// Consumer thread (kq = t / 16, c = t % 16) of its group holds rows
// {4kq .. 4kq+3, 64+4kq .. 64+4kq+3} of the box, columns [8c, 8c+8): for
// activations a half-warp holds 8 whole rows (8 tiles).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_kernels.cuh"   // bounded_wait, drain_wait, record_device_error
#include "quant_kernels.cuh"  // Raw8, encode8, scale_from_amax, reciprocal_path_ok

namespace fp8fg {

// kQuantActT: 128x1 activation tiles (128 consecutive rows of one column,
// the contraction of the weight-gradient product), codes written transposed
// [K, M] and one scale per (column, 128 rows); bf16 input only.
enum QuantMode { kQuantAct = 0, kQuantWeight = 1, kQuantWeightT = 2, kQuantActT = 3 };

constexpr int kQsGroups = 2;                 // consumer groups of 8 warps
constexpr int kQsThreads = kQsGroups * 256;

constexpr int kQsMaxStages = 4;

// Ring per group: two 32 KB bf16 boxes or one 64 KB fp32 box.  (Three bf16
// boxes per group measured no faster for activations and slower for [K,N]
// weights.)
template <typename T, int kMode>
struct QsCfg {
    static constexpr bool kTransposed = kMode == kQuantWeightT || kMode == kQuantActT;
    static constexpr int kSlots = sizeof(T) == 2 ? 2 : 1;
    static constexpr int kStages = kQsGroups * kSlots;
    static constexpr int kBoxBytes = 128 * 128 * static_cast<int>(sizeof(T));
    static constexpr int kRowBytes = 128 * static_cast<int>(sizeof(T));
    static_assert(kStages <= kQsMaxStages, "ring too long");
};

// 16-byte multiple, so that the transpose buffer after it is 16-byte aligned
// (its column maxima are read and written as uint4).
struct alignas(16) QsSmemTail {
    uint64_t full[kQsMaxStages];       // slot filled (TMA bytes)
    uint64_t gbar[kQsGroups];          // per-group barrier (8 warp arrivals)
    float red[kQsGroups][2][8];        // [group][block parity][warp]
    WaitCtl wait;
};

// Transposed output only: [group][box parity][n][k/4 swizzled], transposed
// codes; 128x1 tiles: per-warp column maxima [group][parity][warp][c][word].
struct alignas(16) QsTransposeBuf {
    uint32_t tbuf[kQsGroups][2][128][33];
    uint32_t colmax[kQsGroups][2][8][16][4];
};
static_assert(sizeof(QsSmemTail) % 16 == 0 && offsetof(QsTransposeBuf, colmax) % 16 == 0,
              "uint4 access to the column maxima");

template <typename T, int kMode>
constexpr size_t quant_stream_smem_bytes() {
    return 1024 + QsCfg<T, kMode>::kStages * QsCfg<T, kMode>::kBoxBytes + sizeof(QsSmemTail) +
           (QsCfg<T, kMode>::kTransposed ? sizeof(QsTransposeBuf) : 0);
}

struct QsParams {
    int64_t rows, cols;        // input [rows, cols]; act: [M, K], weight: [K, N]
    int64_t nbr, nbc;          // boxes along rows / cols
    uint8_t* q;
    int64_t ldq;
    float* s;
    int64_t s_stride_r, s_stride_c;   // act: (m, kb); weight: (kb, nb)
    // A group's consecutive boxes are kQsGroups * gridDim.x apart: that
    // step as (box rows, box columns) with step_c < nbc, set by the host.
    int64_t step_r, step_c;
};

// (box row, box column) of a group's box sequence, advanced without dividing.
struct BoxCursor {
    int64_t br, bc;
    __device__ __forceinline__ void init(int64_t box, int64_t nbc) {
        br = box / nbc;
        bc = box - br * nbc;
    }
    __device__ __forceinline__ void advance(const QsParams& p) {
        bc += p.step_c;
        br += p.step_r;
        if (bc >= p.nbc) {
            bc -= p.nbc;
            ++br;
        }
    }
};

// Barrier of one consumer group (its 8 warps) through an mbarrier, so that
// the wait is bounded like every other wait of the kernel.  `uses` counts
// this thread's passes (the phase parity).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& uses, int lane,
                                           volatile int* abort_flag) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
    const bool ok = bounded_wait_warp(bar, uses & 1u, abort_flag);
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

template <typename T, int kMode>
__global__ void __launch_bounds__(kQsThreads, 1)
    quant_stream_kernel(const __grid_constant__ CUtensorMap tm_in, const QsParams p) {
    using Cfg = QsCfg<T, kMode>;
    constexpr int kSlots = Cfg::kSlots;
    constexpr int kStages = Cfg::kStages;
    constexpr int kBoxBytes = Cfg::kBoxBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    QsSmemTail* tail = reinterpret_cast<QsSmemTail*>(smem + kStages * kBoxBytes);
    QsTransposeBuf* tx = reinterpret_cast<QsTransposeBuf*>(tail + 1);   // [N, K] output only
    volatile int* abort_flag = &tail->wait.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nboxes = p.nbr * p.nbc;
    // This CTA's boxes: blockIdx.x + i * gridDim.x, i = 0 .. count-1.
    const int64_t count = nboxes > blockIdx.x ? (nboxes - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&tail->full[s], 1);
        for (int gi = 0; gi < kQsGroups; ++gi) mbar_init(&tail->gbar[gi], 8);
        init_wait_ctl(&tail->wait);
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
    // Boxes are issued in order k = 0, 1, ... (by the group's thread 0) and
    // consumed in the same order: one cursor each.
    BoxCursor issue_at, box_at;
    issue_at.init(blockIdx.x + static_cast<int64_t>(g) * gridDim.x, p.nbc);
    box_at = issue_at;
    auto issue = [&](int64_t k) {
        const int slot = slot_of(k);
        mbar_arrive_expect_tx(&tail->full[slot], kBoxBytes);
        tma_load_2d(smem + slot * kBoxBytes, &tm_in, &tail->full[slot],
                    static_cast<int32_t>(issue_at.bc * 128), static_cast<int32_t>(issue_at.br * 128));
        issue_at.advance(p);
    };
    if (t == 0)
        for (int64_t k = 0; k < kSlots && box_of(k) < count; ++k) issue(k);

    for (int64_t k = 0; box_of(k) < count; ++k) {
        const int64_t i = box_of(k);
        const int stage = slot_of(k);
        const uint32_t phase = static_cast<uint32_t>((k / kSlots) & 1);
        if (!bounded_wait_warp(&tail->full[stage], phase, abort_flag)) break;
        const uint8_t* box_smem = smem + stage * kBoxBytes;
        auto row_ptr = [&](int j) { return box_smem + row_in_box(j) * Cfg::kRowBytes; };
        // The group has finished reading the slot: refill it with the
        // group's box k + kSlots.
        auto release_stage = [&]() -> bool {
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) return false;
            if (t == 0 && box_of(k + kSlots) < count) issue(k + kSlots);
            return true;
        };
        const int64_t br = box_at.br;
        const int64_t bc = box_at.bc;
        box_at.advance(p);

        if constexpr (kMode == kQuantAct) {
            // One 1x128 tile per row: the 16 lanes of a half-warp share 8
            // rows.  Lane c computes the scale of row slot (c & 7) once and
            // the half-warp shares the eight scales by shuffle.
            const int half_base = lane & 16;
            Raw8<T> raw[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) load_raw_smem<T>(row_ptr(j), c, raw[j]);
            if (!release_stage()) break;
            float amax[8];
            half_warp_amax<T, 8>(raw, amax);
            float my_amax = amax[0];
#pragma unroll
            for (int j = 1; j < 8; ++j)
                if ((c & 7) == j) my_amax = amax[j];
            const float my_s = scale_from_amax(my_amax);
            const float my_r = __frcp_rn(my_s);
            // bf16: corrected quotient; fp32: bracket, with its ambiguous
            // pairs (bit 4j + k) recomputed by IEEE division afterwards, as
            // are all pairs of a row whose scale is off the fast path.
            float sj[8];
            uint32_t amb = 0;
            uint8_t* qrow0 = p.q + (br * 128) * p.ldq + bc * 128 + c * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sj[j] = __shfl_sync(0xFFFFFFFFu, my_s, half_base + j);
                uint32_t amb4;
                uint2 codes;
                if constexpr (sizeof(T) == 2) {
                    const float neg_r = __shfl_sync(0xFFFFFFFFu, -my_r, half_base + j);
                    uint64_t n[4];
                    raw[j].to_neg_pairs(n);
                    codes = encode8_corrected(n, f2_pack(sj[j], sj[j]), f2_pack(neg_r, neg_r));
                    amb4 = corrected_path_ok(sj[j]) ? 0u : 0xFu;
                } else {
                    const float ru = __shfl_sync(0xFFFFFFFFu, my_r * kBracketUp, half_base + j);
                    const float rd = __shfl_sync(0xFFFFFFFFu, my_r * kBracketDown, half_base + j);
                    float v[8];
                    raw[j].to_float(v);
                    codes = encode8_bracket(v, ru, rd, amb4);
                    if (!reciprocal_path_ok(sj[j])) amb4 = 0xFu;
                }
                const int r = row_in_box(j);
                if (br * 128 + r < p.rows) {
                    __stcs(reinterpret_cast<uint2*>(qrow0 + r * p.ldq), codes);
                    if (c == j) p.s[(br * 128 + r) * p.s_stride_r + bc * p.s_stride_c] = sj[j];
                    amb |= amb4 << (4 * j);
                }
            }
            while (amb != 0) {
                const int idx = __ffs(amb) - 1;
                amb &= amb - 1;
                const int j = idx >> 2;
                float x0, x1, sv = sj[0];
                select_pair<8>(raw, idx, x0, x1);
#pragma unroll
                for (int jj = 1; jj < 8; ++jj)
                    if (j == jj) sv = sj[jj];
                *reinterpret_cast<uint16_t*>(qrow0 + row_in_box(j) * p.ldq + 2 * (idx & 3)) =
                    static_cast<uint16_t>(encode2_exact(x0, x1, sv));
            }
            continue;
        } else {
        constexpr bool kColScales = kMode == kQuantActT;
        const int par = static_cast<int>((i / kQsGroups) & 1);
        // 128x1 tiles: one scale per column of the box, from a per-column
        // amax (bf16 column pairs, packed maxima; NaN skipped) over the
        // thread's 8 rows, its lane partner (the other kq of the warp) and
        // the group's 8 warps.
        uint64_t cs2[4], cnr2[4];     // column-pair scales (kColScales)
        float cs[8];
        bool col_off = false;
        if constexpr (kColScales) {
            uint32_t cm[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                Raw8<T> r;
                load_raw_smem<T>(row_ptr(j), c, r);
                cm[0] = bf16x2_max(cm[0], r.a.x & 0x7FFF7FFFu);
                cm[1] = bf16x2_max(cm[1], r.a.y & 0x7FFF7FFFu);
                cm[2] = bf16x2_max(cm[2], r.a.z & 0x7FFF7FFFu);
                cm[3] = bf16x2_max(cm[3], r.a.w & 0x7FFF7FFFu);
            }
#pragma unroll
            for (int w = 0; w < 4; ++w) cm[w] = bf16x2_max(cm[w], __shfl_xor_sync(0xFFFFFFFFu, cm[w], 16));
            if (lane < 16)
                *reinterpret_cast<uint4*>(tx->colmax[g][par][wg][c]) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
#pragma unroll
            for (int w8 = 0; w8 < 8; ++w8) {
                const uint4 o = *reinterpret_cast<const uint4*>(tx->colmax[g][par][w8][c]);
                cm[0] = bf16x2_max(cm[0], o.x);
                cm[1] = bf16x2_max(cm[1], o.y);
                cm[2] = bf16x2_max(cm[2], o.z);
                cm[3] = bf16x2_max(cm[3], o.w);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                cs[2 * k] = scale_from_amax(__uint_as_float(cm[k] << 16));
                cs[2 * k + 1] = scale_from_amax(__uint_as_float(cm[k] & 0xFFFF0000u));
                const float r0 = __frcp_rn(cs[2 * k]), r1 = __frcp_rn(cs[2 * k + 1]);
                cs2[k] = f2_pack(cs[2 * k], cs[2 * k + 1]);
                cnr2[k] = f2_pack(-r0, -r1);
                col_off |= !corrected_path_ok(cs[2 * k]) || !corrected_path_ok(cs[2 * k + 1]);
            }
            if (kq == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    p.s[(bc * 128 + c * 8 + e) * p.s_stride_r + br * p.s_stride_c] = cs[e];
            }
        }
        // Otherwise one scale for the whole 128x128 box: an amax pass over
        // the box in shared memory, a block reduction, then an encode pass.
        float a = 0.0f;
        if constexpr (!kColScales) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                Raw8<T> r;
                load_raw_smem<T>(row_ptr(j), c, r);
                a = fmaxf(a, r.abs_max());
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            if (lane == 0) tail->red[g][par][wg] = a;
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
            a = tail->red[g][par][0];
#pragma unroll
            for (int w = 1; w < 8; ++w) a = fmaxf(a, tail->red[g][par][w]);
        }
        const float s = scale_from_amax(a);
        const float rcp = __frcp_rn(s);
        const float ru = rcp * kBracketUp;
        const float rd = rcp * kBracketDown;
        const bool off_path = kColScales ? col_off
                                         : (sizeof(T) == 2 ? !corrected_path_ok(s) : !reciprocal_path_ok(s));
        const uint64_t s2 = f2_pack(s, s);
        const uint64_t neg_r2 = f2_pack(-rcp, -rcp);
        if (!kColScales && t == 0) p.s[br * p.s_stride_r + bc * p.s_stride_c] = s;
        uint32_t(*tb)[33] = tx->tbuf[g][par];
        // Word w of row n sits at column (w + 2 (n / 8)) mod 32 of a 33-word
        // row: the stores below (n = 8c + e, w = 16 h4 + kq) hit 32 distinct
        // banks, the loads (16 consecutive n, two w) at most two per bank.
        // tbuf word w holds the codes of k = 4w .. 4w+3.
        auto tcol = [](int n, int w) { return (w + 2 * (n >> 3)) & 31; };
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
            Raw8<T> raw[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) load_raw_smem<T>(row_ptr(h4 * 4 + jj), c, raw[jj]);
            if (h4 == 1 && !release_stage()) break;
            // bf16: corrected quotient.  fp32: bracket; pairs whose ends
            // disagree (bit 4 jj + k) are recomputed with IEEE division, one
            // per iteration, as are all pairs of a block whose scale is off
            // the fast path.
            uint2 codes[4];
            uint32_t amb = 0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if constexpr (kColScales) {
                    uint64_t n[4];
                    raw[jj].to_neg_pairs(n);
                    codes[jj] = encode8_corrected_pairs(n, cs2, cnr2);
                } else if constexpr (sizeof(T) == 2) {
                    uint64_t n[4];
                    raw[jj].to_neg_pairs(n);
                    codes[jj] = encode8_corrected(n, s2, neg_r2);
                } else {
                    float v[8];
                    raw[jj].to_float(v);
                    uint32_t amb4;
                    codes[jj] = encode8_bracket(v, ru, rd, amb4);
                    amb |= amb4 << (4 * jj);
                }
            }
            if (off_path) amb = 0xFFFFu;
            while (amb != 0) {
                const int idx = __ffs(amb) - 1;
                amb &= amb - 1;
                float x0, x1;
                select_pair<4>(raw, idx, x0, x1);
                uint32_t c16;
                if constexpr (kColScales) {   // the pair's two column scales
                    float s0 = cs[0], s1 = cs[1];
#pragma unroll
                    for (int k = 1; k < 4; ++k)
                        if ((idx & 3) == k) {
                            s0 = cs[2 * k];
                            s1 = cs[2 * k + 1];
                        }
                    c16 = cvt_e4m3x2(__fdiv_rn(x0, s0), __fdiv_rn(x1, s1));
                } else {
                    c16 = encode2_exact(x0, x1, s);
                }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if ((idx >> 2) == jj) patch_pair(codes[jj], idx & 3, c16);
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
                    tb[c * 8 + e][tcol(c * 8 + e, h4 * 16 + kq)] = wx[e];
                    tb[c * 8 + 4 + e][tcol(c * 8 + 4 + e, h4 * 16 + kq)] = wy[e];
                }
            }
        }
        if (*abort_flag) break;
        if (kMode == kQuantWeightT || kMode == kQuantActT) {
            if (!group_sync(&tail->gbar[g], gbar_uses, lane, abort_flag)) break;
            const int n = t >> 1;
            const int part = t & 1;
            // Row n of the output block: 128 codes, written as 16-byte
            // pieces 32 j + 16 part, so that the two lanes of a row fill
            // whole 32-byte sectors in each store.
            uint8_t* dst = p.q + (bc * 128 + n) * p.ldq + br * 128 + part * 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 o;
                o.x = tb[n][tcol(n, j * 8 + part * 4 + 0)];
                o.y = tb[n][tcol(n, j * 8 + part * 4 + 1)];
                o.z = tb[n][tcol(n, j * 8 + part * 4 + 2)];
                o.w = tb[n][tcol(n, j * 8 + part * 4 + 3)];
                __stcs(reinterpret_cast<uint4*>(dst + j * 32), o);
            }
            // No barrier here: this parity of tbuf is written again two boxes
            // on, after group barriers that every thread reaches only once
            // its loads above are done.
        }
        }  // weight modes
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

// quant_weight_kernels.cuh -- online 128x128 weight quantization of bf16
// weights, one block row per thread:
//   sb[kb, nb] = amax over the 128x128 block (kb, nb) of |w| / 448  (1 when 0)
//   q          = E4M3_RNE_satfinite(w / sb)   written [K, N] or [N, K]
// computed on every call, bit-exact to one IEEE fp32 division per element
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"; holysheep.ai "FP8 混精度训练 DeepSeek 671B" (zh),
// 2.2).
//
// HBM-bound streaming.  One persistent CTA per SM holds kQwGroups groups of
// 4 warps; a group walks its own sequence of 128x128 blocks through a ring of
// kQwSlots shared-memory slots (32 KB each):
//   * the group's first thread fills a slot with two TMA loads of 128 rows x
//     64 bf16 (128-byte swizzle: 16-byte chunk c of row r sits at chunk
//     c ^ (r % 8));
//   * each thread takes its share of the block into registers, reduces it
//     with packed |max|, and the warp and then the group (through shared
//     memory and a bounded group barrier) combine the block's amax; the slot
//     is refilled with the group's block kQwSlots ahead right after that
//     barrier (every value is in registers by then);
//   * every thread computes the block's scale and reciprocal and encodes its
//     values with the FMA-corrected quotient (exact for bf16).
// [K, N] output: thread t holds block row t (16 x 16-byte loads: 8 lanes
// read chunk c of 8 consecutive rows, 8 distinct bank groups) and writes its
// 128 codes as four 32-byte stores.
// [N, K] output: thread t holds the column pair 2cp, 2cp+1 (cp = t % 64) over
// block rows 64 kh .. 64 kh + 63 (kh = t / 64): 64 four-byte loads, a warp
// reading one whole 128-byte row per load (no bank conflict).  The low and
// high halves of its words are two rows of the transposed output; each gets
// 64 codes, two 32-byte stores.  No transpose buffer, one barrier per block.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_kernels.cuh"        // bounded_wait_warp, record_device_error
#include "quant_act_kernels.cuh"   // bf16x2_absmax, stg256_cs, lds128_addr
#include "quant_kernels.cuh"       // Raw8, encode8_corrected, scale_from_amax

namespace fp8fg {

constexpr int kQwGroups = 2;                      // groups of 4 warps per CTA
constexpr int kQwSlots = 3;
constexpr int kQwHalfBytes = 128 * 128;           // 128 rows x 64 bf16
constexpr int kQwBlockBytes = 2 * kQwHalfBytes;   // 32 KB: a 128x128 bf16 block
constexpr int kQwThreads = kQwGroups * 128;

// Modes: 128x128 blocks with [K, N] or transposed [N, K] codes; or 128x1
// tiles (128 rows of one column: the weight gradient's 1x128 tiles along
// the tokens), codes transposed, one scale per column of each 128-row band.
enum QwMode { kQwBlockRows = 0, kQwBlockCols = 1, kQwColTiles = 2 };

struct QwSmemTail {
    uint64_t full[kQwGroups][kQwSlots];   // slot filled (TMA bytes)
    uint64_t gbar[kQwGroups];             // group barrier: 4 warp arrivals
    uint32_t red[kQwGroups][2][4];        // per warp packed |max|, by block parity
    uint32_t colred[kQwGroups][2][2][64]; // 128x1: per column pair packed |max|, [parity][kh][cp]
    WaitCtl wait;
};

constexpr size_t kQwSmemBytes =
    1024 /* alignment slack */ + kQwGroups * kQwSlots * kQwBlockBytes + sizeof(QwSmemTail);
static_assert(kQwSmemBytes <= 227 * 1024, "shared memory per CTA");

struct QwParams {
    int64_t nbr, nbc;          // blocks along K (rows of w) and N (columns)
    int64_t nblocks;           // nbr * nbc
    uint8_t* q;
    int64_t ldq;
    float* s;
    // blocks: s[kb * s_stride_kb + nb * s_stride_nb]; 128x1 tiles:
    // s[column * s_stride_nb + band * s_stride_kb]
    int64_t s_stride_kb, s_stride_nb;
};

// Barrier of the 4 warps of a group (an mbarrier, so that the wait is
// bounded); `uses` counts this thread's passes (the phase parity).
__device__ __forceinline__ bool qw_group_sync(uint64_t* bar, uint32_t& uses, int lane,
                                              volatile int* abort_flag) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
    const bool ok = bounded_wait_warp(bar, uses & 1u, abort_flag);
    ++uses;
    return ok;
}

template <int kMode>
__global__ void __launch_bounds__(kQwThreads, 1)
    quant_weight_rows_kernel(const __grid_constant__ CUtensorMap tm_in, const QwParams p) {
    constexpr bool kTransposed = kMode != kQwBlockRows;
    constexpr bool kColScales = kMode == kQwColTiles;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    QwSmemTail* tail =
        reinterpret_cast<QwSmemTail*>(smem + kQwGroups * kQwSlots * kQwBlockBytes);
    volatile int* abort_flag = &tail->wait.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = warp >> 2;              // group
    const int wg = warp & 3;              // warp within the group
    const int t = threadIdx.x & 127;      // thread within the group = block row
    if (threadIdx.x == 0) {
        for (int gi = 0; gi < kQwGroups; ++gi) {
            for (int s = 0; s < kQwSlots; ++s) mbar_init(&tail->full[gi][s], 1);
            mbar_init(&tail->gbar[gi], 4);
        }
        init_wait_ctl(&tail->wait);
        fence_mbar_init();
        tma_prefetch_desc(&tm_in);
    }
    __syncthreads();

    // Group-major numbering across the grid, so that surplus blocks land on
    // different SMs.
    const int64_t gg = static_cast<int64_t>(g) * gridDim.x + blockIdx.x;
    const int64_t ng = static_cast<int64_t>(kQwGroups) * gridDim.x;
    const int64_t count = p.nblocks > gg ? (p.nblocks - 1 - gg) / ng + 1 : 0;
    uint8_t* ring = smem + g * kQwSlots * kQwBlockBytes;
    uint64_t* full = tail->full[g];
    uint32_t uses = 0;

    // Block b = gg + k ng is (b / nbc, b % nbc); cursors advance by ng.
    const int64_t step_r = ng / p.nbc;
    const int64_t step_c = ng - step_r * p.nbc;
    auto advance = [&](int64_t& br, int64_t& bc) {
        br += step_r;
        bc += step_c;
        if (bc >= p.nbc) {
            bc -= p.nbc;
            ++br;
        }
    };
    int64_t i_br = gg / p.nbc, i_bc = gg - (gg / p.nbc) * p.nbc;   // next block to issue
    int64_t c_br = i_br, c_bc = i_bc;                               // next block to consume

    auto issue = [&](int64_t k) {   // thread 0 of the group: block k into slot k % kQwSlots
        const int slot = static_cast<int>(k % kQwSlots);
        uint8_t* dst = ring + slot * kQwBlockBytes;
        mbar_arrive_expect_tx(&full[slot], kQwBlockBytes);
        const int32_t x = static_cast<int32_t>(i_bc * 128);
        const int32_t y = static_cast<int32_t>(i_br * 128);
        tma_load_2d(dst, &tm_in, &full[slot], x, y);
        tma_load_2d(dst + kQwHalfBytes, &tm_in, &full[slot], x + 64, y);
        advance(i_br, i_bc);
    };
    if (t == 0)
        for (int64_t k = 0; k < kQwSlots && k < count; ++k) issue(k);

    const uint32_t swz = static_cast<uint32_t>(t & 7);
    // [N, K] output: thread t holds the column pair cp = t % 64 (columns 2cp,
    // 2cp + 1 of the block) over the block rows kh * 64 .. kh * 64 + 63.
    const uint32_t cp = static_cast<uint32_t>(t) & 63u;
    const uint32_t kh = static_cast<uint32_t>(t) >> 6;
    for (int64_t k = 0; k < count; ++k) {
        const int slot = static_cast<int>(k % kQwSlots);
        if (!bounded_wait_warp(&full[slot], static_cast<uint32_t>((k / kQwSlots) & 1), abort_flag))
            break;
        const uint32_t slot_addr = smem_u32(ring + slot * kQwBlockBytes);
        // kTransposed: w2[i] = (w[k][2cp], w[k][2cp+1]) for k = 64 kh + i, a
        // 4-byte load from the swizzled box (the 32 lanes of a warp read one
        // whole 128-byte row of a half: no bank conflict).  Otherwise raw[c]
        // = row t, columns 8c .. 8c+7.
        Raw8<uint16_t> raw[16];
        uint32_t w2[64];
        uint32_t m[16];
        if constexpr (kTransposed) {
            const uint32_t base = slot_addr + (cp >> 5) * kQwHalfBytes + ((cp & 3u) << 2);
            const uint32_t chunk = (cp & 31u) >> 2;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const uint32_t kr = kh * 64u + static_cast<uint32_t>(i);
                asm volatile("ld.shared.u32 %0, [%1];"
                             : "=r"(w2[i])
                             : "r"(base + kr * 128u + ((chunk ^ (kr & 7u)) << 4)));
            }
#pragma unroll
            for (int c = 0; c < 16; ++c)
                m[c] = bf16x2_absmax(bf16x2_absmax(w2[4 * c], w2[4 * c + 1]),
                                     bf16x2_absmax(w2[4 * c + 2], w2[4 * c + 3]));
        } else {
            const uint32_t row_addr = slot_addr + t * 128;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                raw[c].a = lds128_addr(row_addr + (c >> 3) * kQwHalfBytes +
                                       (((static_cast<uint32_t>(c) & 7u) ^ swz) << 4));
#pragma unroll
            for (int c = 0; c < 16; ++c)
                m[c] = bf16x2_absmax(bf16x2_absmax(raw[c].a.x, raw[c].a.y),
                                     bf16x2_absmax(raw[c].a.z, raw[c].a.w));
        }
#pragma unroll
        for (int w = 8; w > 0; w >>= 1)
#pragma unroll
            for (int c = 0; c < w; ++c) m[c] = bf16x2_absmax(m[c], m[c + w]);
        const int par = static_cast<int>(k & 1);
        // The block's amax (one scale), or the column pair's maxima over the
        // band's 128 rows (two scales): this thread's half and the half of
        // thread t ^ 64, through shared memory.
        float sj[2], rj[2];
        if constexpr (kColScales) {
            tail->colred[g][par][kh][cp] = m[0];
            if (!qw_group_sync(&tail->gbar[g], uses, lane, abort_flag)) break;
            uint32_t cm = bf16x2_absmax(m[0], tail->colred[g][par][kh ^ 1u][cp]) & 0x7FFF7FFFu;
            sj[0] = scale_from_amax(__uint_as_float(cm << 16));
            sj[1] = scale_from_amax(__uint_as_float(cm & 0xFFFF0000u));
        } else {
            uint32_t wm = m[0];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                wm = bf16x2_absmax(wm, __shfl_xor_sync(0xFFFFFFFFu, wm, off));
            if (lane == 0) tail->red[g][par][wg] = wm;
            // After this barrier every thread's values are in registers and
            // the four warp maxima are visible.
            if (!qw_group_sync(&tail->gbar[g], uses, lane, abort_flag)) break;
            uint32_t bm = bf16x2_absmax(bf16x2_absmax(tail->red[g][par][0], tail->red[g][par][1]),
                                        bf16x2_absmax(tail->red[g][par][2], tail->red[g][par][3]));
            bm &= 0x7FFF7FFFu;
            sj[0] = sj[1] = scale_from_amax(
                fmaxf(__uint_as_float(bm << 16), __uint_as_float(bm & 0xFFFF0000u)));
        }
        // The slot just read takes the block kQwSlots ahead.
        if (t == 0 && k + kQwSlots < count) issue(k + kQwSlots);

        const int64_t br = c_br, bc = c_bc;
        advance(c_br, c_bc);
        rj[0] = __frcp_rn(sj[0]);
        rj[1] = kColScales ? __frcp_rn(sj[1]) : rj[0];
        const float s = sj[0];
        if constexpr (kColScales) {
            if (kh == 0) {
                p.s[(bc * 128 + 2 * cp) * p.s_stride_nb + br * p.s_stride_kb] = sj[0];
                p.s[(bc * 128 + 2 * cp + 1) * p.s_stride_nb + br * p.s_stride_kb] = sj[1];
            }
        } else if (t == 0) {
            p.s[br * p.s_stride_kb + bc * p.s_stride_nb] = s;
        }
        const bool fast = corrected_path_ok(s);
        const uint64_t s2 = f2_pack(s, s);
        const uint64_t neg_r2 = f2_pack(-rj[0], -rj[0]);

        if constexpr (!kTransposed) {
            uint32_t codes[32];
            if (fast) {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint64_t n[4];
                    raw[c].to_neg_pairs(n);
                    const uint2 cc = encode8_corrected(n, s2, neg_r2);
                    codes[2 * c] = cc.x;
                    codes[2 * c + 1] = cc.y;
                }
            } else {
                // Scale off the corrected quotient's proven range: IEEE division.
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    float v[8];
                    raw[c].to_float(v);
                    codes[2 * c] =
                        encode2_exact(v[0], v[1], s) | (encode2_exact(v[2], v[3], s) << 16);
                    codes[2 * c + 1] =
                        encode2_exact(v[4], v[5], s) | (encode2_exact(v[6], v[7], s) << 16);
                }
            }
            uint8_t* dst = p.q + (br * 128 + t) * p.ldq + bc * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint32_t w[8] = {codes[8 * q4], codes[8 * q4 + 1], codes[8 * q4 + 2],
                                       codes[8 * q4 + 3], codes[8 * q4 + 4], codes[8 * q4 + 5],
                                       codes[8 * q4 + 6], codes[8 * q4 + 7]};
                stg256_cs(dst + 32 * q4, w);
            }
        } else {
            // Output rows n = 2cp + j (j = 0: low bf16 of each word, 1: high),
            // codes of block rows 64 kh .. 64 kh + 63: 8 codes per 8 rows.
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                // this output row's scale: the block's, or its column's
                const float sc = sj[j];
                const bool fast_j = corrected_path_ok(sc);
                const uint64_t s2j = f2_pack(sc, sc);
                const uint64_t neg_r2j = f2_pack(-rj[j], -rj[j]);
                uint32_t codes[16];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (fast_j) {
                        uint64_t n[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t a = w2[8 * c + 2 * q], b = w2[8 * c + 2 * q + 1];
                            const uint32_t xa = j == 0 ? a << 16 : a & 0xFFFF0000u;
                            const uint32_t xb = j == 0 ? b << 16 : b & 0xFFFF0000u;
                            n[q] = f2_pack(__uint_as_float(xa ^ 0x80000000u),
                                           __uint_as_float(xb ^ 0x80000000u));
                        }
                        const uint2 cc = encode8_corrected(n, s2j, neg_r2j);
                        codes[2 * c] = cc.x;
                        codes[2 * c + 1] = cc.y;
                    } else {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t a = w2[8 * c + e];
                            v[e] = __uint_as_float(j == 0 ? a << 16 : a & 0xFFFF0000u);
                        }
                        codes[2 * c] =
                            encode2_exact(v[0], v[1], sc) | (encode2_exact(v[2], v[3], sc) << 16);
                        codes[2 * c + 1] =
                            encode2_exact(v[4], v[5], sc) | (encode2_exact(v[6], v[7], sc) << 16);
                    }
                }
                uint8_t* dst = p.q + (bc * 128 + 2 * cp + j) * p.ldq + br * 128 + kh * 64;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const uint32_t w[8] = {codes[8 * q2], codes[8 * q2 + 1], codes[8 * q2 + 2],
                                           codes[8 * q2 + 3], codes[8 * q2 + 4], codes[8 * q2 + 5],
                                           codes[8 * q2 + 6], codes[8 * q2 + 7]};
                    stg256_cs(dst + 32 * q2, w);
                }
            }
        }
    }
    // After an abandoned wait a fill may still be in flight: let it land
    // before the CTA leaves (every fill is consumed on the normal path).
    if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 22)) {
        }
    }
}

}  // namespace fp8fg

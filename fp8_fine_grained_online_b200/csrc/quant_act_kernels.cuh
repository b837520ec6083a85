// quant_act_kernels.cuh -- online 1x128 activation quantization of bf16
// rows, one row per thread:
//   scale[m, kb] = amax_{k in tile kb} |x[m, k]| / 448   (1 when zero)
//   q[m, k]      = E4M3_RNE_satfinite(x[m, k] / scale[m, k / 128])
// computed on every call, bit-exact to one IEEE fp32 division per element
// (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Finkornig kvantisering",
// "Online-kvantisering"; holysheep.ai "FP8 混精度训练 DeepSeek 671B" (zh),
// 2.2).
//
// HBM-bound streaming.  One persistent CTA per SM of kQaWarps independent
// warps; each warp owns a ring of kQaSlots shared-memory slots and walks
// its own sequence of boxes of 32 rows x 128 columns (one 1x128 tile per
// row):
//   * lane 0 fills a slot with two TMA loads of 32 rows x 64 bf16 (128-byte
//     rows, 128-byte swizzle: 16-byte chunk c of row r lands at chunk
//     c ^ (r % 8), so that the 32 lanes, reading chunk c of 32 consecutive
//     rows, hit every bank group once per 8 lanes);
//   * lane r takes row r into 64 registers (16 shared loads), reduces the
//     tile's amax with packed |max| on bf16 pairs, computes the scale and
//     its reciprocal once, and encodes the 128 values with the
//     FMA-corrected quotient (exact for bf16, see encode8_corrected);
//   * the slot is refilled with the warp's box kQaSlots ahead as soon as
//     every lane has its row in registers (after the amax, which consumes
//     all of them);
//   * codes leave as four 32-byte stores per row (whole sectors), the scale
//     as one 4-byte store.
// No cross-warp synchronization: a warp's only waits are on its own slots,
// each bounded like every other wait of the library.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_kernels.cuh"   // bounded_wait_warp, record_device_error
#include "quant_kernels.cuh"  // Raw8, encode8_corrected, scale_from_amax

namespace fp8fg {

constexpr int kQaWarps = 8;
constexpr int kQaSlots = 3;
constexpr int kQaRows = 32;                        // rows of a box (one per lane)
constexpr int kQaHalfBytes = kQaRows * 128;        // 32 rows x 64 bf16
constexpr int kQaBoxBytes = 2 * kQaHalfBytes;      // 8 KB: 32 rows x 128 bf16
constexpr int kQaThreads = 32 * kQaWarps;

// What a box's rows are and where they go.
enum QaMode {
    kRowsPlain = 0,    // input row m -> output row m
    kRowsScatter = 1,  // input row t (a token) -> output rows dest[t, :]
};

struct QaSmemTail {
    uint64_t full[kQaWarps][kQaSlots];
    WaitCtl wait;
};

constexpr int kQaRingBytes = kQaWarps * kQaSlots * kQaBoxBytes;
constexpr size_t kQaSmemBytes = 1024 /* alignment slack */ + kQaRingBytes + sizeof(QaSmemTail);
static_assert(kQaSmemBytes <= 227 * 1024, "shared memory per CTA");

struct QaParams {
    int64_t rows;              // M (the input rows: tokens for the scatter form)
    int64_t nkb;               // K / 128
    int64_t nboxes;            // ceil(M / 32) * nkb
    uint8_t* q;
    int64_t ldq;
    float* s;
    int64_t s_stride_m, s_stride_kb;
    // Scatter form (MoE dispatch): input row t is written to the output rows
    // dest[t * topk + j] (j < topk) that are not -1; out_rows bounds them.
    const int32_t* dest;
    int64_t topk;
    int64_t out_rows;
};

// max(|a|, |b|) per bf16 lane (sign bits are the XOR of the inputs' and are
// cleared by the caller); a NaN lane yields the other operand.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ void stg256_cs(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                 "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ uint4 lds128_addr(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// One row's 128 codes (32 words) and its scale to output row `row`.
__device__ __forceinline__ void store_row_tile(const QaParams& p, int64_t row, int64_t kb,
                                               const uint32_t (&codes)[32], float s) {
    uint8_t* dst = p.q + row * p.ldq + kb * 128;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t w[8] = {codes[8 * g], codes[8 * g + 1], codes[8 * g + 2], codes[8 * g + 3],
                               codes[8 * g + 4], codes[8 * g + 5], codes[8 * g + 6],
                               codes[8 * g + 7]};
        stg256_cs(dst + 32 * g, w);
    }
    p.s[row * p.s_stride_m + kb * p.s_stride_kb] = s;
}

// kMode (QaMode): plain rows, or the MoE dispatch fused in, in token order
// (scatter: each token row is read and quantized once, and its codes and
// scale are written to each of its up to topk destination rows).
template <int kMode>
__global__ void __launch_bounds__(kQaThreads, 1)
    quant_act_rows_kernel(const __grid_constant__ CUtensorMap tm_in, const QaParams p) {
    constexpr bool kScatter = kMode == kRowsScatter;
    constexpr int kSlotBytes = kQaBoxBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    QaSmemTail* tail = reinterpret_cast<QaSmemTail*>(smem + kQaRingBytes);
    volatile int* abort_flag = &tail->wait.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int w = 0; w < kQaWarps; ++w)
            for (int s = 0; s < kQaSlots; ++s) mbar_init(&tail->full[w][s], 1);
        init_wait_ctl(&tail->wait);
        fence_mbar_init();
        tma_prefetch_desc(&tm_in);
    }
    __syncthreads();

    // Plain rows: warp-major numbering across the grid (warp w of CTA b is
    // w * grid + b, its boxes gw, gw + nw, ...), so that when the boxes do
    // not divide evenly the surplus lands on different SMs.  Scatter: each
    // warp takes a contiguous run of boxes (the grid's share split evenly,
    // tiles of one row band in order), so that a band's destination rows
    // are read once per warp and prefetched a whole band ahead.
    const int64_t gw = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x;
    const int64_t nw = static_cast<int64_t>(kQaWarps) * gridDim.x;
    int64_t first, count, step_mb, step_kb;
    if constexpr (kScatter) {
        first = p.nboxes * gw / nw;
        count = p.nboxes * (gw + 1) / nw - first;
        step_mb = p.nkb == 1 ? 1 : 0;
        step_kb = p.nkb == 1 ? 0 : 1;
    } else {
        first = gw;
        count = p.nboxes > gw ? (p.nboxes - 1 - gw) / nw + 1 : 0;
        step_mb = nw / p.nkb;
        step_kb = nw - step_mb * p.nkb;
    }
    uint8_t* ring = smem + warp * kQaSlots * kSlotBytes;
    uint64_t* full = tail->full[warp];

    // Box b is (row band b / nkb, tile b % nkb); both cursors (issue,
    // consume) advance by the warp's stride without dividing.
    auto advance = [&](int64_t& mb, int64_t& kb) {
        mb += step_mb;
        kb += step_kb;
        if (kb >= p.nkb) {
            kb -= p.nkb;
            ++mb;
        }
    };
    int64_t i_mb = first / p.nkb, i_kb = first - (first / p.nkb) * p.nkb;   // next box to issue
    int64_t c_mb = i_mb, c_kb = i_kb;                                       // next box to consume

    auto issue = [&](int64_t k) {   // lane 0: box k of this warp into slot k % kQaSlots
        const int slot = static_cast<int>(k % kQaSlots);
        uint8_t* dst = ring + slot * kQaBoxBytes;
        mbar_arrive_expect_tx(&full[slot], kQaBoxBytes);
        const int32_t x = static_cast<int32_t>(i_kb * 128);
        const int32_t y = static_cast<int32_t>(i_mb * kQaRows);
        tma_load_2d(dst, &tm_in, &full[slot], x, y);
        tma_load_2d(dst + kQaHalfBytes, &tm_in, &full[slot], x + 64, y);
        advance(i_mb, i_kb);
    };
    if (lane == 0)
        for (int64_t k = 0; k < kQaSlots && k < count; ++k) issue(k);

    // Scatter form: the first kDestBatch destinations of each of the 32
    // tokens of the band being processed (dst_cur, band dst_band) and of the
    // band after it (dst_next), loaded when the warp enters a band.
    constexpr int kDestBatch = 8;
    int32_t dst_cur[kDestBatch], dst_next[kDestBatch];
    int64_t dst_band = -1;
    auto load_dest = [&](int64_t mb, int32_t (&d)[kDestBatch]) {
        const int64_t row = mb * kQaRows + lane;
#pragma unroll
        for (int j = 0; j < kDestBatch; ++j)
            d[j] = (row < p.rows && j < p.topk) ? __ldg(p.dest + row * p.topk + j) : -1;
    };
    if constexpr (kScatter) {
        if (count > 0) {
            load_dest(c_mb, dst_cur);
            load_dest(c_mb + 1, dst_next);
            dst_band = c_mb;
        }
    }

    const uint32_t swz = static_cast<uint32_t>(lane & 7);
    for (int64_t k = 0; k < count; ++k) {
        const int slot = static_cast<int>(k % kQaSlots);
        if (!bounded_wait_warp(&full[slot], static_cast<uint32_t>((k / kQaSlots) & 1), abort_flag))
            break;
        Raw8<uint16_t> raw[16];
        const uint32_t row_addr = smem_u32(ring + slot * kSlotBytes) + lane * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c)
            raw[c].a = lds128_addr(row_addr + (c >> 3) * kQaHalfBytes +
                                   (((static_cast<uint32_t>(c) & 7u) ^ swz) << 4));
        // amax of the row's 128 values: packed |max| over the 64 pairs.
        uint32_t m[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
            m[c] = bf16x2_absmax(bf16x2_absmax(raw[c].a.x, raw[c].a.y),
                                 bf16x2_absmax(raw[c].a.z, raw[c].a.w));
#pragma unroll
        for (int w = 8; w > 0; w >>= 1)
#pragma unroll
            for (int c = 0; c < w; ++c) m[c] = bf16x2_absmax(m[c], m[c + w]);
        const uint32_t mm = m[0] & 0x7FFF7FFFu;
        const float amax = fmaxf(__uint_as_float(mm << 16), __uint_as_float(mm & 0xFFFF0000u));
        // Every lane's row is in registers: the slot takes the box kQaSlots on.
        __syncwarp();
        if (lane == 0 && k + kQaSlots < count) issue(k + kQaSlots);

        const int64_t kb = c_kb;
        const int64_t row = c_mb * kQaRows + lane;
        const int64_t mb = c_mb;
        advance(c_mb, c_kb);
        const float s = scale_from_amax(amax);
        const float r = __frcp_rn(s);
        uint32_t codes[32];
        if (corrected_path_ok(s)) {
            const uint64_t s2 = f2_pack(s, s);
            const uint64_t neg_r2 = f2_pack(-r, -r);
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
                codes[2 * c] = encode2_exact(v[0], v[1], s) | (encode2_exact(v[2], v[3], s) << 16);
                codes[2 * c + 1] =
                    encode2_exact(v[4], v[5], s) | (encode2_exact(v[6], v[7], s) << 16);
            }
        }
        if constexpr (kScatter) {
            if (mb != dst_band) {   // runs advance one tile at a time: the next band
                if (mb == dst_band + 1) {
#pragma unroll
                    for (int j = 0; j < kDestBatch; ++j) dst_cur[j] = dst_next[j];
                } else {
                    load_dest(mb, dst_cur);
                }
                dst_band = mb;
                load_dest(mb + 1, dst_next);
            }
            for (int64_t j0 = 0; j0 < p.topk; j0 += kDestBatch) {
                int32_t dst_rows[kDestBatch];
#pragma unroll
                for (int j = 0; j < kDestBatch; ++j)
                    dst_rows[j] = j0 == 0 ? dst_cur[j]
                                  : (row < p.rows && j0 + j < p.topk)
                                      ? __ldg(p.dest + row * p.topk + j0 + j)
                                      : -1;
#pragma unroll
                for (int j = 0; j < kDestBatch; ++j) {
                    const int32_t d = dst_rows[j];
                    if (d == -1) continue;
                    if (d < -1 || d >= p.out_rows) {   // reported once per tile, never written
                        if (kb == 0) record_device_error(kDevErrShape);
                        continue;
                    }
                    store_row_tile(p, d, kb, codes, s);
                }
            }
        } else if (row < p.rows) {
            store_row_tile(p, row, kb, codes, s);
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

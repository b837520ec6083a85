// gemm_kernels.cuh -- block-scaled FP8 GEMM on sm_100a tensor cores
// (tcgen05 UMMA, TMEM accumulators, TMA operand loads), dense and MoE-grouped.
//
//   C[m, n] = sum_kb sa[m, kb] * sb[kb, n/128] * P_kb[m, n]
//   P_kb    = the tensor-core product of one 128-wide K chunk of E4M3 codes
//
// The promotion interval is one 128-wide chunk, the scaling unit of both
// operands (codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Ökad ackumuleringsprecision": the
// tensor-core partial sums are promoted to FP32 registers at fixed
// intervals; "Finkornig kvantisering" for the 1x128 / 128x128 scales).
//
// Structure of the one-CTA kernel (one persistent CTA per SM, 384 threads;
// the CTA-pair kernel in gemm_pair_kernels.cuh has the same roles):
//   warps 0-7   epilogue: warp w reads TMEM lanes 32*(w%4).. and columns
//               128*(w/4).., scales the chunk partial by sa*sb and adds it
//               to 128 FP32 accumulators per thread (one output row, 128
//               columns); at tile end converts and stores the row.
//   warp 8      TMA producer: A tile 128x128 B and B tile 256x128 B per chunk
//               into a 4-stage shared-memory ring (128-byte swizzle).
//   warp 9      TMEM owner and MMA issuer: per chunk, 4 x UMMA
//               (M=128, N=256, K=32) into one of two TMEM partial buffers
//               (2 x 256 columns), then commits to the ring's "empty"
//               barrier and the buffer's "full" barrier.
//   warp 10     grouped: builds the tile table at start; warp 11 idle.
// Double-buffered TMEM lets the MMA of chunk kb+1 run while the epilogue
// promotes chunk kb.
//
// Every mbarrier wait is bounded (kWaitLimitCycles); on timeout the kernel
// records FP8_ERR_DEVICE_TIMEOUT in the device error word, all roles stop,
// in-flight copies and MMAs are waited for (bounded), TMEM is released and
// the kernel returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "quant_kernels.cuh"  // fused 1x128 quantization of the output
#include "sm100_ptx.cuh"

namespace fp8fg {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;  // one scale chunk = 128 bytes of E4M3 per row
constexpr int kStages = 4;
// 12 warps = 3 warpgroups.  Warps 0-7 (warpgroups 0-1) are the epilogue;
// warpgroup 2 holds the TMA producer (warp 8), the MMA issuer / TMEM owner
// (warp 9) and two idle warps.  Registers at launch: 384 x 168; warpgroup 2
// drops to kCtrlRegs and warpgroups 0-1 rise to kEpiRegs:
// 128 x 40 + 256 x 232 = 64512 = 384 x 168.
constexpr int kGemmThreads = 384;
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMmaWarp2 = 10;   // second MMA issuer of the CTA-pair kernel
constexpr int kSchedWarp = 10;  // grouped kernel: builds the tile table
constexpr int kCtrlRegs = 40;
constexpr int kEpiRegs = 232;
static_assert(128 * kCtrlRegs + 256 * kEpiRegs <= kGemmThreads * 168, "register split");
constexpr int kABytes = kBM * kBK;  // 16 KB
constexpr int kBBytes = kBN * kBK;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;      // 2 partial buffers x 256 FP32 columns
constexpr int kMaxGroups = 1024;

// Grouped GEMM row split.  kGrpAll: a launch covers every row of each group
// in tiles of its own height.  The split form covers a group's rows with
// CTA-pair tiles of kPairRows rows except a remainder of 1 to kBM rows,
// which a second launch of the one-CTA kernel covers with one kBM-row tile,
// so that no group pads its last tile by more than kBM - 1 rows of MMA work
// (a 256-row tile for a 257-row group would pad it by 255):
//   kGrpPairPart: whole kPairRows blocks, and a remainder of more than kBM rows;
//   kGrpTailPart: a remainder of 1 to kBM rows.
constexpr int kGrpAll = 0;
constexpr int kGrpPairPart = 1;
constexpr int kGrpTailPart = 2;
constexpr int64_t kPairRows = 256;

// Status codes recorded in the device error word (values of fp8_status_t).
constexpr unsigned kDevErrShape = 2;
constexpr unsigned kDevErrTimeout = 9;

// Device error word; read and cleared by fp8_get_device_error().
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_device_error(unsigned code) {
    atomicCAS(&g_device_error, 0u, code);
}

// The limit of the waits that can abort (bounded_wait) is a device variable,
// kWaitLimitCycles unless fp8_set_wait_limit() changed it.  Each CTA copies it
// into shared memory at start (WaitCtl, next to its abort flag), so that no
// wait depends on a global load.  A limit below kShortWaitLimit is a test of
// the timeout path: the waits then check the clock after every poll instead
// of every kPollsPerClockCheck polls, so that a real wait runs out.  The
// drains below always keep kWaitLimitCycles.
constexpr long long kWaitLimitCycles = 1ll << 31;
constexpr long long kShortWaitLimit = 1ll << 20;
constexpr int kPollsPerClockCheck = 64;

__device__ long long g_wait_limit_cycles = kWaitLimitCycles;

// A CTA's abort flag and its copy of the wait limit.  The flag is the first
// member: the waits receive a pointer to it.
struct WaitCtl {
    int abort_flag;
    int polls_per_check;
    long long limit;
};

__device__ __forceinline__ void init_wait_ctl(WaitCtl* w) {
    const long long limit = *static_cast<volatile long long*>(&g_wait_limit_cycles);
    w->abort_flag = 0;
    w->limit = limit;
    w->polls_per_check = limit < kShortWaitLimit ? 1 : kPollsPerClockCheck;
}

struct GemmParams {
    const float* sa;
    int64_t sa_sm, sa_skb;
    const float* sb;
    int64_t sb_sg, sb_skb, sb_snb;
    void* c;
    int64_t ldc;
    int64_t M;       // dense: rows; grouped: total rows
    int64_t N;
    int nkb;         // K / 128
    int num_nt;      // ceil(N / kBN)
    int num_mt;      // dense only: ceil(M / kBM)
    int band_m;      // dense raster: m-tiles per band (band_n == 0)
    int band_n;      // dense raster: n-tiles per band, or 0 for bands of m-tiles
    const int32_t* offsets;  // grouped only: [G + 1]
    int G;
    // Quantized output (fp8_blockscaled_gemm_quant): codes [M, ldqc] and
    // scales sc[m * sc_sm + (n / 128) * sc_snb]; c (bf16) may then be null.
    uint8_t* qc;
    int64_t ldqc;
    float* sc;
    int64_t sc_sm, sc_snb;
    int c_v8;        // C rows may be written as 32-byte stores (c and ldc 32-byte aligned)
    int qc_v8;       // code rows may be written as 32-byte stores (qc and ldqc 32-byte aligned)
    // Grouped: which rows of each group this launch covers (kGrpAll, or one
    // part of a split between the CTA-pair and the one-CTA kernel).
    int grp_split;
};

// One 32-byte store of 8 words (the address 32-byte aligned).
__device__ __forceinline__ void stg256(void* p, const uint32_t* w) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

// Grouped GEMM: the persistent tile schedule, built in shared memory from
// the device-side offsets at kernel start.
struct GroupTables {
    int grp_prefix[kMaxGroups + 1];  // tiles before group g
    int grp_lo[kMaxGroups];          // first row of group g
    int grp_hi[kMaxGroups];          // one past its last row (clamped to M)
};

// Shared-memory layout after the 1024-aligned operand ring.
struct GemmSmemTail {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int total_tiles;
    WaitCtl wait;
    GroupTables grp;
};

constexpr size_t kGemmSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes +
                                  sizeof(GemmSmemTail);

struct TileCoord {
    int64_t m0;       // first row of the tile (global row index)
    int64_t row_end;  // rows >= row_end are not part of this tile's problem
    int64_t n0;       // first column
    int g;            // group (0 for dense)
};

// Wait for phase `parity` of `bar` to complete; false if this CTA aborted or
// the wait ran past kWaitLimitCycles (which aborts the CTA).
// The limit is counted in SM clock cycles (clock64 is a cheap local
// counter; the device-wide %globaltimer is slow to read and would delay the
// reaction to a completed barrier).  2^31 cycles is about one second at the
// B200's 1.9 GHz and a few seconds at its lowest clocks.
// The normal form polls kPollsPerClockCheck times (unrolled) between checks
// of the abort flag and the clock: measured, any extra work in the polling
// loop (a loop counter, a clock read per poll) slows the GEMM by 6-20%,
// because spinning warps share issue slots with the epilogue.  The test form
// (a limit below kShortWaitLimit) checks after every poll.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag) {
    const uint32_t a = smem_u32(bar);
    const volatile WaitCtl* ctl = reinterpret_cast<const volatile WaitCtl*>(abort_flag);
    const bool every_poll = ctl->polls_per_check == 1;   // read before the first poll
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    if (!every_poll) {
        while (true) {
#pragma unroll
            for (int i = 0; i < kPollsPerClockCheck; ++i)
                if (mbar_try_wait(a, parity)) return true;
            if (*abort_flag) return false;
            if (clock64() - t0 > ctl->limit) break;
        }
    } else {
        while (true) {
            if (mbar_try_wait(a, parity)) return true;
            if (*abort_flag) return false;
            if (clock64() - t0 > ctl->limit) break;
        }
    }
    *abort_flag = 1;
    record_device_error(kDevErrTimeout);
    return false;
}

// bounded_wait by every lane of a converged warp, decided for the warp as a
// whole: true only if every lane saw the phase complete, so that all lanes
// leave a loop on an abandoned wait together.
__device__ __forceinline__ bool bounded_wait_warp(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag) {
    const bool ok = bounded_wait(bar, parity, abort_flag);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Same, ignoring the abort flag: used to drain copies, MMAs and arrivals
// this CTA is owed, so that no async write outlives the CTA.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const long long t0 = clock64();
    while (true) {
        for (int i = 0; i < kPollsPerClockCheck; ++i)
            if (mbar_try_wait(a, parity)) return;
        if (clock64() - t0 > kWaitLimitCycles) {
            record_device_error(kDevErrTimeout);
            return;
        }
    }
}

// One warp builds the grouped tile table from the device offsets: group g
// covers the rows [grp_lo, grp_hi) this launch takes (all of them, or its
// part of the pair / one-CTA split, kGrp*) in ceil(rows / kTileM) m-tiles
// times num_nt n-tiles.  Invalid offsets (negative, or decreasing) give an
// empty group and record FP8_ERR_SHAPE.
template <int kTileM>
__device__ __forceinline__ void build_group_tables(const GemmParams& p, GroupTables* gt, int lane,
                                                   int* total_tiles) {
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
        const int g = base + lane;
        int tiles = 0;
        if (g < p.G) {
            int64_t lo = p.offsets[g];
            int64_t hi = p.offsets[g + 1];
            if (lo < 0 || hi < lo) {
                record_device_error(kDevErrShape);
                lo = hi = 0;
            }
            lo = lo < p.M ? lo : p.M;
            hi = hi < p.M ? hi : p.M;
            if (p.grp_split != kGrpAll) {
                const int64_t full = (hi - lo) / kPairRows;
                const int64_t rem = (hi - lo) - full * kPairRows;
                if (p.grp_split == kGrpPairPart) {
                    if (rem > 0 && rem <= kBM) hi = lo + full * kPairRows;
                } else {   // kGrpTailPart
                    lo += full * kPairRows;
                    if (rem > kBM) hi = lo;
                }
            }
            gt->grp_lo[g] = static_cast<int>(lo);
            gt->grp_hi[g] = static_cast<int>(hi);
            tiles = static_cast<int>((hi - lo + kTileM - 1) / kTileM) * p.num_nt;
        }
        int incl = tiles;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        if (g < p.G) gt->grp_prefix[g + 1] = carry + incl;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
        gt->grp_prefix[0] = 0;
        *total_tiles = carry;
    }
}

// Tile t of the persistent schedule: kTileM rows (of one group, for the
// grouped form) by kBN columns.
template <bool kGrouped, int kTileM = kBM>
__device__ __forceinline__ TileCoord decode_tile(int t, const GemmParams& p,
                                                 const GroupTables* gt) {
    TileCoord tc;
    if (!kGrouped) {
        // Bands of band_m m-tiles (the A rows of a band stay in L2 while B
        // streams past them), m fastest inside a band; or bands of band_n
        // n-tiles (the B rows stay, A streams), n fastest.  Either way the
        // CTAs of one wave share both A rows and B rows through L2.
        int mt, nt;
        if (p.band_n == 0) {
            const int per_band = p.band_m * p.num_nt;
            const int band = t / per_band;
            const int within = t - band * per_band;
            const int bm0 = band * p.band_m;
            const int bm = min(p.band_m, p.num_mt - bm0);
            nt = within / bm;
            mt = bm0 + (within - nt * bm);
        } else {
            const int per_band = p.band_n * p.num_mt;
            const int band = t / per_band;
            const int within = t - band * per_band;
            const int bn0 = band * p.band_n;
            const int bn = min(p.band_n, p.num_nt - bn0);
            mt = within / bn;
            nt = bn0 + (within - mt * bn);
        }
        tc.m0 = static_cast<int64_t>(mt) * kTileM;
        tc.row_end = p.M;
        tc.n0 = static_cast<int64_t>(nt) * kBN;
        tc.g = 0;
    } else {
        // Group g owns tiles [grp_prefix[g], grp_prefix[g+1]).
        int lo = 0, hi = p.G;  // find the last g with grp_prefix[g] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (gt->grp_prefix[mid] <= t) lo = mid; else hi = mid;
        }
        const int g = lo;
        const int local = t - gt->grp_prefix[g];
        const int rows = gt->grp_hi[g] - gt->grp_lo[g];
        const int nmt = (rows + kTileM - 1) / kTileM;
        const int nt = local / nmt;
        const int mt = local - nt * nmt;  // m fastest: neighbours share B tiles
        tc.m0 = gt->grp_lo[g] + static_cast<int64_t>(mt) * kTileM;
        tc.row_end = gt->grp_hi[g];
        tc.n0 = static_cast<int64_t>(nt) * kBN;
        tc.g = g;
    }
    return tc;
}

// acc[kOff .. kOff+32) += s * P (32 FP32 partials from TMEM), packed FMAs.
// Per-column B scales: acc[i] += (sa * sb[i]) * P[i] for 32 columns, sb[]
// read from shared memory (the same four values for every lane: broadcast).
template <int kOff>
__device__ __forceinline__ void promote32_cols(float (&acc)[128], const uint32_t (&part)[32],
                                               uint64_t sa2, const float* sbk) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const float4 b = lds_f4(sbk + kOff + i);
        const uint64_t s01 = f2_mul(sa2, f2_pack(b.x, b.y));
        const uint64_t s23 = f2_mul(sa2, f2_pack(b.z, b.w));
        const uint64_t d01 = f2_fma(f2_pack(__uint_as_float(part[i]), __uint_as_float(part[i + 1])),
                                    s01, f2_pack(acc[kOff + i], acc[kOff + i + 1]));
        const uint64_t d23 = f2_fma(f2_pack(__uint_as_float(part[i + 2]), __uint_as_float(part[i + 3])),
                                    s23, f2_pack(acc[kOff + i + 2], acc[kOff + i + 3]));
        f2_unpack(d01, acc[kOff + i], acc[kOff + i + 1]);
        f2_unpack(d23, acc[kOff + i + 2], acc[kOff + i + 3]);
    }
}

template <int kOff>
__device__ __forceinline__ void promote32(float (&acc)[128], const uint32_t (&part)[32], float s) {
#pragma unroll
    for (int i = 0; i < 32; i += 2)
        ffma2_scalar(acc[kOff + i], acc[kOff + i + 1], s, __uint_as_float(part[i]),
                     __uint_as_float(part[i + 1]));
}

// One tile of the epilogue, for one thread: promotes every 128-wide K chunk
// of its row slice (128 columns of the 256-wide tile) from TMEM into FP32
// registers, acc += sa[row, kb] * sb[kb, nb] * P_kb, then converts and stores
// the row slice.  `release(buf)` (called by lane 0 after the warp has read
// its slice of a chunk) hands TMEM buffer `buf` back to the MMA issuer.
// Returns false if a wait was abandoned because the CTA is aborting.
// The row's 128 accumulators as the next layer's input: rounded to bf16
// (stored as C when p.c is set), then quantized as one 1x128 activation tile
// exactly as fp8_quantize_act_1x128 quantizes that bf16 row: NaN-skipping
// amax, scale = amax / 448 (1 if 0), codes of the corrected quotient (exact
// for bf16), IEEE division when the scale is off that path.
__device__ __forceinline__ void store_row_quantized(const GemmParams& p, const float (&acc)[128],
                                                    int64_t row, int64_t col0) {
    uint32_t hb[64];
#pragma unroll
    for (int j = 0; j < 64; ++j) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
        hb[j] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    uint32_t m = hb[0] & 0x7FFF7FFFu;
#pragma unroll
    for (int j = 1; j < 64; ++j) m = bf16x2_max(m, hb[j] & 0x7FFF7FFFu);
    const float amax = fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    if (p.c != nullptr) {
        __nv_bfloat16* crow = reinterpret_cast<__nv_bfloat16*>(p.c) + row * p.ldc + col0;
        if (p.c_v8) {
#pragma unroll
            for (int j = 0; j < 8; ++j) stg256(crow + 16 * j, hb + 8 * j);
        } else {
            uint4* out = reinterpret_cast<uint4*>(crow);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                out[j] = make_uint4(hb[4 * j], hb[4 * j + 1], hb[4 * j + 2], hb[4 * j + 3]);
        }
    }
    const float s = scale_from_amax(amax);
    const float r = __frcp_rn(s);
    const uint64_t s2 = f2_pack(s, s);
    const uint64_t neg_r2 = f2_pack(-r, -r);
    const bool fast = corrected_path_ok(s);
    uint8_t* qbase = p.qc + row * p.ldqc + col0;
    uint4* qrow = reinterpret_cast<uint4*>(qbase);
    uint32_t pending[4];   // the previous 16 codes, when rows take 32-byte stores
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint2 codes[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            Raw8<uint16_t> raw;
            raw.a = make_uint4(hb[8 * j + 4 * h], hb[8 * j + 4 * h + 1], hb[8 * j + 4 * h + 2],
                               hb[8 * j + 4 * h + 3]);
            if (fast) {
                uint64_t n[4];
                raw.to_neg_pairs(n);
                codes[h] = encode8_corrected(n, s2, neg_r2);
            } else {
                float v[8];
                raw.to_float(v);
                codes[h].x = encode2_exact(v[0], v[1], s) | (encode2_exact(v[2], v[3], s) << 16);
                codes[h].y = encode2_exact(v[4], v[5], s) | (encode2_exact(v[6], v[7], s) << 16);
            }
        }
        if (p.qc_v8) {
            if (j & 1) {
                const uint32_t w[8] = {pending[0], pending[1], pending[2], pending[3],
                                       codes[0].x, codes[0].y, codes[1].x, codes[1].y};
                stg256(qbase + 16 * (j - 1), w);
            } else {
                pending[0] = codes[0].x;
                pending[1] = codes[0].y;
                pending[2] = codes[1].x;
                pending[3] = codes[1].y;
            }
        } else {
            qrow[j] = make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
        }
    }
    p.sc[row * p.sc_sm + (col0 / 128) * p.sc_snb] = s;
}

//
// kColScaleB: B carries one scale per row n of B (column of C) and K chunk,
// sb[kb * sb_skb + n] (n contiguous): acc += sa[row, kb] * sb[kb, n] * P_kb.
// The warp stages the 128 sb values of its columns for chunk kb + 1 in
// `sb_stage` ([2][128] floats of this warp) by cp.async while it promotes
// chunk kb.
template <bool kOutBf16, bool kQuantOut = false, bool kColScaleB = false, typename Release>
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, uint64_t* tfull,
                                              volatile int* abort_flag, uint32_t tmem_base,
                                              uint32_t t_lane, int h, int lane, int64_t row,
                                              bool row_ok, int64_t col0, bool col_ok, int g,
                                              uint32_t& chunk, Release release,
                                              float* sb_stage = nullptr) {
    const int nkb = p.nkb;
    const float* sa_row = p.sa + (row_ok ? row : 0) * p.sa_sm;
    const float* sb_col = kColScaleB ? p.sb + (col_ok ? col0 : 0) + 4 * lane
                                     : p.sb + g * p.sb_sg + (col_ok ? col0 / 128 : 0) * p.sb_snb;
    if constexpr (kColScaleB) {
        // The previous tile's lanes are done with both staging buffers.
        __syncwarp();
        if (col_ok && nkb > 0) cp_async_16(sb_stage + 4 * lane, sb_col);
        cp_async_commit();
    }

    float acc[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
    float sa_next = (row_ok && nkb > 0) ? __ldg(sa_row) : 0.0f;
    float sb_next = (!kColScaleB && col_ok && nkb > 0) ? __ldg(sb_col) : 0.0f;

    // Scales two chunks ahead (the loads are L2 round trips).
    float sa1 = (row_ok && nkb > 1) ? __ldg(sa_row + p.sa_skb) : 0.0f;
    float sb1 = (!kColScaleB && col_ok && nkb > 1) ? __ldg(sb_col + p.sb_skb) : 0.0f;

    // Per chunk: two round trips of 64 columns through 64 staging registers;
    // the second pair of loads is issued while the first is promoted, and the
    // TMEM buffer is handed back to the MMA issuer as soon as the last load
    // has landed, before the second half is promoted.
    uint32_t pa[32], pb[32];
    for (int kb = 0; kb < nkb; ++kb) {
        const float scale = sa_next * sb_next;
        const uint64_t sa2p = f2_pack(sa_next, sa_next);
        float sa2 = 0.0f, sb2 = 0.0f;
        if (kb + 2 < nkb) {
            sa2 = row_ok ? __ldg(sa_row + (kb + 2) * p.sa_skb) : 0.0f;
            sb2 = (!kColScaleB && col_ok) ? __ldg(sb_col + (kb + 2) * p.sb_skb) : 0.0f;
        }
        sa_next = sa1;
        sb_next = sb1;
        sa1 = sa2;
        sb1 = sb2;
        const float* sbk = sb_stage + (kb & 1) * 128;
        if constexpr (kColScaleB) {
            // Chunk kb's column scales have landed (for every lane after the
            // warp barrier); the other buffer, read during chunk kb - 1, takes
            // chunk kb + 1's.
            cp_async_wait_all();
            __syncwarp();
            if (col_ok && kb + 1 < nkb)
                cp_async_16(sb_stage + ((kb + 1) & 1) * 128 + 4 * lane, sb_col + (kb + 1) * p.sb_skb);
            cp_async_commit();
        }

        const uint32_t buf = chunk & 1u;
        if (!bounded_wait_warp(&tfull[buf], (chunk >> 1) & 1u, abort_flag)) {
            if constexpr (kColScaleB) cp_async_wait_all();
            return false;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + t_lane + buf * kBN + h * 128;
        tmem_ld_32x32b_x32(taddr, pa);
        tmem_ld_32x32b_x32(taddr + 32, pb);
        tmem_wait_ld_dep(pa);
        tmem_wait_ld_dep(pb);
        if constexpr (kColScaleB) promote32_cols<0>(acc, pa, sa2p, sbk);
        else promote32<0>(acc, pa, scale);
        tmem_ld_32x32b_x32(taddr + 64, pa);
        if constexpr (kColScaleB) promote32_cols<32>(acc, pb, sa2p, sbk);
        else promote32<32>(acc, pb, scale);
        tmem_ld_32x32b_x32(taddr + 96, pb);
        tmem_wait_ld_dep(pa);
        tmem_wait_ld_dep(pb);
        // This warp's slice of the chunk is in registers: hand the TMEM
        // buffer back to the MMA issuer.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release(buf);
        ++chunk;
        if constexpr (kColScaleB) {
            promote32_cols<64>(acc, pa, sa2p, sbk);
            promote32_cols<96>(acc, pb, sa2p, sbk);
        } else {
            promote32<64>(acc, pa, scale);
            promote32<96>(acc, pb, scale);
        }
    }
    if (row_ok && col_ok) {
        if (kQuantOut) {
            store_row_quantized(p, acc, row, col0);
        } else if (kOutBf16) {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.c) + row * p.ldc + col0;
            uint32_t w[64];
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            if (p.c_v8) {   // whole 32-byte sectors per lane
#pragma unroll
                for (int j = 0; j < 8; ++j) stg256(out + 16 * j, w + 8 * j);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    reinterpret_cast<uint4*>(out)[j] =
                        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            }
        } else {
            float* out = reinterpret_cast<float*>(p.c) + row * p.ldc + col0;
            if (p.c_v8) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(acc[8 * j + e]);
                    stg256(out + 8 * j, w);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    reinterpret_cast<float4*>(out)[j] =
                        make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            }
        }
    }
    return true;
}

template <bool kGrouped, bool kOutBf16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    blockscaled_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint8_t* sA = smem;                         // kStages x 16 KB
    uint8_t* sB = smem + kStages * kABytes;     // kStages x 32 KB
    GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &tail->wait.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == kProducerWarp && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tail->tfull[b], 1);
            mbar_init(&tail->tempty[b], kEpiWarps);
        }
        init_wait_ctl(&tail->wait);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tail->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (kGrouped && warp == kSchedWarp) {
        build_group_tables<kBM>(p, &tail->grp, lane, &tail->total_tiles);
    } else if (!kGrouped && warp == kSchedWarp && lane == 0) {
        tail->total_tiles = p.num_mt * p.num_nt;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->total_tiles;
    const int nkb = p.nkb;

    if (warp >= kEpiWarps) {
        // Control warpgroup (producer, MMA, two idle warps): few registers.
        setmaxnreg_dec<kCtrlRegs>();
        if (warp == kProducerWarp && lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, last_parity = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileCoord tc = decode_tile<kGrouped>(t, p, &tail->grp);
                const int32_t a_row = static_cast<int32_t>(tc.m0);
                const int32_t b_row = static_cast<int32_t>(tc.g * p.N + tc.n0);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!bounded_wait(&tail->empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&tail->full[stage], kStageBytes);
                    tma_load_2d(sA + stage * kABytes, &tmA, &tail->full[stage], kb * kBK, a_row);
                    tma_load_2d(sB + stage * kBBytes, &tmB, &tail->full[stage], kb * kBK, b_row);
                    issued_mask |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < kStages; ++s)
                    if (issued_mask & (1u << s)) drain_wait(&tail->full[s], (last_parity >> s) & 1u);
            }
        } else if (warp == kMmaWarp && lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_e4m3_f32(kBM, kBN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t chunk = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const uint32_t buf = chunk & 1u;
                    const uint32_t use = chunk >> 1;
                    // Operands first (usually long ready), then the TMEM
                    // buffer: the epilogue's release is the critical path.
                    if (!bounded_wait(&tail->full[stage], phase, abort_flag) ||
                        !bounded_wait(&tail->tempty[buf], (use & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * kABytes));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + stage * kBBytes));
                    const uint32_t d = tmem_base + buf * kBN;
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k)  // 32 bytes of K per MMA = +2 in addr>>4
                        umma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
                    umma_commit(&tail->empty[stage]);
                    umma_commit(&tail->tfull[buf]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    ++chunk;
                }
            }
            if (!ok && chunk > 0) {
                const uint32_t last = chunk - 1;
                drain_wait(&tail->tfull[last & 1u], (last >> 1) & 1u);
            }
        }
    } else {
        // ------------------------------------------------ epilogue warps 0-7
        setmaxnreg_inc<kEpiRegs>();
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int h = warp >> 2;           // column half of the 256-wide tile
        const int r = q * 32 + lane;       // row within the tile
        const uint32_t t_lane = static_cast<uint32_t>(q * 32) << 16;
        uint32_t chunk = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            const TileCoord tc = decode_tile<kGrouped>(t, p, &tail->grp);
            const int64_t row = tc.m0 + r;
            const bool row_ok = row < tc.row_end;
            const int64_t col0 = tc.n0 + h * 128;
            const bool col_ok = col0 < p.N;
            ok = epilogue_tile<kOutBf16>(p, tail->tfull, abort_flag, tmem_base, t_lane, h, lane, row,
                                         row_ok, col0, col_ok, tc.g, chunk,
                                         [&](uint32_t buf) { mbar_arrive(&tail->tempty[buf]); });
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace fp8fg

// gemm_pair_kernels.cuh -- block-scaled FP8 GEMM on a CTA pair (tcgen05
// cta_group::2): one 256 x 256 output tile per pair of SMs.  Dense, or
// grouped (MoE experts: tiles of 256 rows of one group, B and sb per group).
//
// Same arithmetic as blockscaled_gemm_kernel (each 128-wide K chunk's
// tensor-core partial is scaled by sa * sb and added into FP32 registers;
// codingmall.com "Kan du förklara rollen för FP8 precision i
// träningsprocessen för DeepSeek-V3", "Ökad ackumuleringsprecision"), with
// the MMA spread over two SMs so that each SM streams half as much of B:
//
//   * cluster of 2 CTAs; CTA r holds rows [m0 + 128 r, +128) of A and rows
//     [n0 + 128 r, +128) of B (N-major rows, K contiguous) in its own
//     shared memory, 6-stage ring of 16 KB + 16 KB per 128-wide K chunk;
//   * each CTA's TMA loads count their bytes on the even CTA's "full"
//     barrier (cta_group::2 completion, no multicast);
//   * one thread of the even CTA issues UMMA M=256 N=256 K=32 (cta_group::2):
//     A and B from both CTAs' shared memory, D rows 0-127 into the even
//     CTA's TMEM and rows 128-255 into the odd CTA's, two partial buffers of
//     256 columns; its commits arrive on the "empty" / "full" barriers of
//     both CTAs (tcgen05.commit multicast);
//   * each CTA's 8 epilogue warps promote their 128 rows exactly as in the
//     single-CTA kernel and release a TMEM buffer on the even CTA's
//     "tmem empty" barrier (16 arrivals: 8 warps x 2 CTAs).
//
// Per SM and chunk this moves 32 KB from L2 instead of 48 KB for a
// 128 x 256 single-CTA tile of the same MMA time.
//
// kColScaleB (dense): B has one scale per row and K chunk (1x128 tiles
// along K, the weight-gradient product's second operand) instead of one
// per 128 x 128 block.
#pragma once

#include "gemm_kernels.cuh"

namespace fp8fg {

constexpr int kPairBM = 256;          // rows of a pair tile
static_assert(kPairBM == kPairRows, "grouped row split assumes pair tiles of kPairRows rows");
constexpr int kPairStages = 6;
constexpr int kPairHalfBytes = 128 * kBK;                // 16 KB: 128 rows x 128 B
constexpr int kPairStageBytes = 2 * kPairHalfBytes;       // A half + B half
constexpr uint64_t kDrainGraceNs = 2000000ull;            // abort path: let copies land

struct GemmPairSmemTail {
    uint64_t full[kPairStages];    // even CTA: TMA bytes of both CTAs
    uint64_t empty[kPairStages];   // both CTAs: MMA commit (multicast)
    uint64_t tfull[2];             // both CTAs: MMA commit (multicast)
    uint64_t tempty[2];            // even CTA: 16 epilogue-warp arrivals
    uint32_t tmem_base;
    int total_tiles;
    WaitCtl wait;
    uint64_t pad;                  // 16-byte multiple
};

constexpr size_t kGemmPairSmemBytes =
    1024 /* alignment slack */ + kPairStages * kPairStageBytes + sizeof(GemmPairSmemTail);
// The grouped form adds its tile table (GroupTables) after the tail.
constexpr size_t kGemmPairGroupedSmemBytes = kGemmPairSmemBytes + sizeof(GroupTables);
// Per-column B scales: each epilogue warp's two staging rows of 128 sb
// values after the tail (16-byte cp.async destinations).
constexpr size_t kGemmPairColScaleSmemBytes =
    kGemmPairSmemBytes + kEpiWarps * 2 * 128 * sizeof(float);
static_assert(sizeof(GemmPairSmemTail) % 16 == 0, "staging rows must be 16-byte aligned");

__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < ns) {
    }
}

template <bool kGrouped, bool kOutBf16, bool kQuantOut = false, bool kColScaleB = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    blockscaled_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                                 const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
    static_assert(!(kColScaleB && (kGrouped || kQuantOut)), "per-column B scales: dense, C only");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    GemmPairSmemTail* tail =
        reinterpret_cast<GemmPairSmemTail*>(smem + kPairStages * kPairStageBytes);
    GroupTables* gt = reinterpret_cast<GroupTables*>(tail + 1);   // grouped only
    float* sb_stages = reinterpret_cast<float*>(tail + 1);         // per-column sb only
    volatile int* abort_flag = &tail->wait.abort_flag;
    auto stage_a = [&](int s) { return smem + s * kPairStageBytes; };
    auto stage_b = [&](int s) { return smem + s * kPairStageBytes + kPairHalfBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();    // 0: even CTA (issues the MMAs)
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;

    if (warp == kProducerWarp && lane == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tail->tfull[b], 1);
            mbar_init(&tail->tempty[b], 2 * kEpiWarps);
        }
        init_wait_ctl(&tail->wait);
        if (!kGrouped) tail->total_tiles = p.num_mt * p.num_nt;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == kMmaWarp) {
        tmem_alloc_pair(&tail->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    if (kGrouped && warp == kSchedWarp)   // both CTAs build the same table
        build_group_tables<kPairBM>(p, gt, lane, &tail->total_tiles);
    tc_fence_before();
    cluster_sync();
    tc_fence_after();

    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->total_tiles;
    const int nkb = p.nkb;
    bool aborted = false;

    if (warp >= kEpiWarps) {
        setmaxnreg_dec<kCtrlRegs>();
        if (warp == kProducerWarp && lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t used_mask = 0, last_parity = 0;
            bool ok = true;
            for (int t = pair; t < total_tiles && ok; t += num_pairs) {
                const TileCoord tc = decode_tile<kGrouped, kPairBM>(t, p, gt);
                const int32_t a_row = static_cast<int32_t>(tc.m0) + 128 * static_cast<int32_t>(rank);
                // grouped: expert g's weights are rows [g N, g N + N) of B
                const int32_t b_row = static_cast<int32_t>(static_cast<int64_t>(tc.g) * p.N + tc.n0) +
                                      128 * static_cast<int32_t>(rank);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!bounded_wait(&tail->empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(smem_u32(&tail->full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&tail->full[stage], 2 * kPairStageBytes);
                    tma_load_2d_pair(stage_a(stage), &tmA, full_leader, kb * kBK, a_row);
                    tma_load_2d_pair(stage_b(stage), &tmB, full_leader, kb * kBK, b_row);
                    used_mask |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (ok) {
                // Every stage filled was consumed: wait for the last commit on
                // each of this CTA's "empty" barriers to have landed.
                for (int s = 0; s < kPairStages; ++s)
                    if (used_mask & (1u << s)) drain_wait(&tail->empty[s], (last_parity >> s) & 1u);
            } else {
                aborted = true;
            }
        } else if ((warp == kMmaWarp || warp == kMmaWarp2) && lane == 0 && leader) {
            // ------------------------------------------------ MMA issuers (even CTA)
            // Warp 9 issues the even chunks (TMEM buffer 0, ring stages 0, 2,
            // 4), warp 10 the odd ones (buffer 1, stages 1, 3, 5).  A chunk
            // accumulates only into its own buffer and each issuer commits
            // only its own chunks, so the two instruction streams are
            // independent.  One thread would spend ~800 cycles per chunk on
            // two barrier waits, four UMMAs and two commits, against 512
            // cycles of tensor work; two threads keep the tensor pipe fed.
            const uint32_t par = warp == kMmaWarp ? 0u : 1u;
            constexpr uint32_t idesc = idesc_e4m3_f32(kPairBM, kBN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t chunk = 0;
            uint32_t last_issued = 0;
            bool issued_any = false;
            bool ok = true;
            for (int t = pair; t < total_tiles && ok; t += num_pairs) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if ((chunk & 1u) == par) {
                        const uint32_t use = chunk >> 1;
                        // Operands first (usually long ready), then the TMEM
                        // buffer: the epilogue's release is the critical path.
                        if (!bounded_wait(&tail->full[stage], phase, abort_flag) ||
                            !bounded_wait(&tail->tempty[par], (use & 1u) ^ 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(stage_a(stage)));
                        const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(stage_b(stage)));
                        const uint32_t d = tmem_base + par * kBN;
#pragma unroll
                        for (int k = 0; k < kBK / 32; ++k)
                            umma_f8f6f4_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc,
                                             k > 0 ? 1u : 0u);
                        umma_commit_pair_mc(&tail->empty[stage], 0x3);
                        umma_commit_pair_mc(&tail->tfull[par], 0x3);
                        last_issued = chunk;
                        issued_any = true;
                    }
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    ++chunk;
                }
            }
            if (ok) {
                // Both CTAs' epilogues release every buffer they used: wait for
                // the last release of this issuer's buffer so that no remote
                // arrival is in flight when the pair exits.
                if (issued_any) drain_wait(&tail->tempty[par], (last_issued >> 1) & 1u);
            } else {
                aborted = true;
                if (issued_any) drain_wait(&tail->tfull[par], (last_issued >> 1) & 1u);
            }
        }
    } else {
        // ------------------------------------------------ epilogue warps 0-7 (both CTAs)
        setmaxnreg_inc<kEpiRegs>();
        const int q = warp & 3;
        const int h = warp >> 2;
        const int r = 128 * static_cast<int>(rank) + q * 32 + lane;   // row within the pair tile
        const uint32_t t_lane = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tail->tempty[0]), 0),
                                           mapa_shared(smem_u32(&tail->tempty[1]), 0)};
        uint32_t chunk = 0;
        bool ok = true;
        for (int t = pair; t < total_tiles && ok; t += num_pairs) {
            const TileCoord tc = decode_tile<kGrouped, kPairBM>(t, p, gt);
            const int64_t row = tc.m0 + r;
            const bool row_ok = row < tc.row_end;
            const int64_t col0 = tc.n0 + h * 128;
            const bool col_ok = col0 < p.N;
            ok = epilogue_tile<kOutBf16, kQuantOut, kColScaleB>(
                p, tail->tfull, abort_flag, tmem_base, t_lane, h, lane, row, row_ok, col0, col_ok,
                tc.g, chunk, [&](uint32_t buf) { mbar_arrive_cluster(tempty_leader[buf]); },
                sb_stages + warp * 2 * 128);
        }
        if (!ok) aborted = true;
    }

    // An abandoned wait leaves copies or arrivals of the peer possibly in
    // flight: give them time to land before the pair leaves.
    if (aborted || *abort_flag) spin_ns(kDrainGraceNs);
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace fp8fg

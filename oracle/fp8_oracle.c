/*
 * fp8_oracle.c -- plain, slow CPU oracle for fine-grained online FP8
 * quantization and the block-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the
 * bench's CPU-baseline leg do.  It shares no code, header, table or
 * constant generator with the CUDA library; it is written from the method's
 * description alone:
 *
 *   [KB]  codingmall.com knowledge base, "Kan du förklara rollen för FP8
 *         precision i träningsprocessen för DeepSeek-V3" -- sections
 *         "Finkornig kvantisering" (1x128 activation tiles, 128x128 weight
 *         blocks, each scaled on its own), "Online-kvantisering" (scale
 *         computed from the current values on every call), "Ökad
 *         ackumuleringsprecision" (partial sums promoted to FP32 at fixed
 *         intervals) and "Unified E4M3 Format" (E4M3 for every operand).
 *   [HS]  holysheep.ai, "FP8 混精度训练 DeepSeek 671B" (Chinese edition),
 *         section "2.2 细粒度量化实现" -- the quantizer divides each value by
 *         scale = amax / 448 (448 being the E4M3 maximum) and casts to
 *         float8_e4m3fn; dequantization is code value times scale.
 *
 * Readings where the pages leave a step open (each one is also listed in
 * the design notes of the repository):
 *   - E4M3 is the OCP "e4m3fn" encoding: bias 7, no infinities, NaN =
 *     S.1111.111, largest finite value 448, smallest subnormal 2^-9.
 *   - Rounding into E4M3 is round-to-nearest, ties to even significand,
 *     saturating: any |v| >= 448 (infinity included) becomes +-448.
 *   - x / scale is one IEEE fp32 division (round to nearest), as is
 *     amax / 448.
 *   - scale is replaced by 1 when amax / 448 is zero.  This is the stated
 *     "scale = 1 when amax = 0" rule; it also covers fp32 inputs whose
 *     amax is so small that amax / 448 underflows to zero.
 *   - amax ignores NaN elements (a NaN element itself encodes to NaN).
 *   - A partial tile or block (K or N not a multiple of 128) takes its amax
 *     over the elements that exist.
 *   - The promotion interval is one 128-wide K chunk: the chunk is also the
 *     scaling unit, so the GEMM is  C = sum_kb (sa*sb) * P_kb  where P_kb is
 *     the chunk's product of decoded codes.  The oracle evaluates it in
 *     fp64 as the sum over k of the dequantized products, which is the
 *     same value up to the order of rounding.
 *
 * Floating-point discipline: compile with -O2 -fno-fast-math
 * -ffp-contract=off on x86-64 (SSE2 scalar float arithmetic is IEEE
 * single precision, no FMA contraction).  OpenMP, when enabled, only
 * splits independent output rows across threads; each row is computed by
 * exactly the loops written below.
 */
#include "fp8_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_TILE 128
#define ORC_E4M3_MAX 448.0

/* ------------------------------------------------------------------ */
/* E4M3 codec, from the format definition                               */
/* ------------------------------------------------------------------ */

/* Value of an E4M3 code: sign s, 4 exponent bits e (bias 7), 3 mantissa
 * bits m.  e == 0 is subnormal (m * 2^-9); S.1111.111 is NaN. */
double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double mag;
    if ((c & 0x7F) == 0x7F)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest E4M3 code to v.  The search runs over the 127 non-negative
 * finite codes 0x00..0x7E (monotone in value) in fp64, which holds every
 * code and every midpoint exactly; an exact tie goes to the code whose
 * mantissa LSB is 0.  |v| >= 448 saturates to 448.  The sign bit is
 * copied from v, so -0 and tiny negatives give 0x80. */
uint8_t orc_e4m3_encode(float v)
{
    uint8_t sign;
    double a, bestd;
    int c, best;
    if (isnan(v))
        return 0x7F;
    sign = signbit(v) ? 0x80 : 0x00;
    a = fabs((double)v);
    if (a >= ORC_E4M3_MAX)
        return (uint8_t)(sign | 0x7E);
    best = 0;
    bestd = a;                       /* distance to code 0x00 (= 0.0) */
    for (c = 1; c <= 0x7E; c++) {
        double d = fabs(a - orc_e4m3_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

void orc_e4m3_decode_array(const uint8_t* c, int64_t n, double* out)
{
    int64_t i;
    for (i = 0; i < n; i++)
        out[i] = orc_e4m3_decode(c[i]);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; i++)
        out[i] = orc_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------ */
/* Inputs: bf16 (raw 16-bit patterns) or fp32.  bf16 -> fp32 is exact.  */
/* ------------------------------------------------------------------ */

static float load_in(const void* x, int in_type, int64_t idx)
{
    if (in_type == ORC_IN_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t*)x)[idx] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return f;
    }
    return ((const float*)x)[idx];
}

/* scale = amax / 448 in fp32 (IEEE division), 1 when that is zero. */
static float scale_from_amax(float amax)
{
    float s = amax / 448.0f;
    if (s == 0.0f)
        s = 1.0f;
    return s;
}

/* ------------------------------------------------------------------ */
/* Online 1x128 activation quantization  ([KB] "Finkornig kvantisering", */
/* "Online-kvantisering"; [HS] 2.2 FP8BlockQuantizer.quantize)          */
/* ------------------------------------------------------------------ */

void orc_quantize_act_1x128(const void* x, int in_type, int64_t M, int64_t K,
                            int64_t ldx, uint8_t* q, int64_t ldq, float* sa,
                            int64_t sa_stride_m, int64_t sa_stride_kb)
{
    int64_t m;
    int64_t nkb = (K + ORC_TILE - 1) / ORC_TILE;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; m++) {
        int64_t kb, k;
        for (kb = 0; kb < nkb; kb++) {
            int64_t k0 = kb * ORC_TILE;
            int64_t k1 = k0 + ORC_TILE < K ? k0 + ORC_TILE : K;
            float amax = 0.0f, s;
            for (k = k0; k < k1; k++) {
                float a = fabsf(load_in(x, in_type, m * ldx + k));
                if (a > amax)        /* false for NaN: NaN is skipped */
                    amax = a;
            }
            s = scale_from_amax(amax);
            sa[m * sa_stride_m + kb * sa_stride_kb] = s;
            for (k = k0; k < k1; k++)
                q[m * ldq + k] = orc_e4m3_encode(load_in(x, in_type, m * ldx + k) / s);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Online 128x128 weight quantization ([KB] "Finkornig kvantisering")    */
/* w is [K][N] row-major (ldw).  q is [K][N] (transpose_out == 0) or     */
/* [N][K] (transpose_out == 1) with row stride ldq; sb[kb][nb].          */
/* ------------------------------------------------------------------ */

void orc_quantize_weight_128x128(const void* w, int in_type, int64_t K, int64_t N,
                                 int64_t ldw, uint8_t* q, int transpose_out,
                                 int64_t ldq, float* sb, int64_t sb_stride_kb,
                                 int64_t sb_stride_nb)
{
    int64_t nkb = (K + ORC_TILE - 1) / ORC_TILE;
    int64_t nnb = (N + ORC_TILE - 1) / ORC_TILE;
    int64_t blk;
#pragma omp parallel for schedule(static)
    for (blk = 0; blk < nkb * nnb; blk++) {
        int64_t kb = blk / nnb, nb = blk % nnb;
        int64_t k0 = kb * ORC_TILE, n0 = nb * ORC_TILE;
        int64_t k1 = k0 + ORC_TILE < K ? k0 + ORC_TILE : K;
        int64_t n1 = n0 + ORC_TILE < N ? n0 + ORC_TILE : N;
        int64_t k, n;
        float amax = 0.0f, s;
        for (k = k0; k < k1; k++)
            for (n = n0; n < n1; n++) {
                float a = fabsf(load_in(w, in_type, k * ldw + n));
                if (a > amax)
                    amax = a;
            }
        s = scale_from_amax(amax);
        sb[kb * sb_stride_kb + nb * sb_stride_nb] = s;
        for (k = k0; k < k1; k++)
            for (n = n0; n < n1; n++) {
                uint8_t code = orc_e4m3_encode(load_in(w, in_type, k * ldw + n) / s);
                if (transpose_out)
                    q[n * ldq + k] = code;
                else
                    q[k * ldq + n] = code;
            }
    }
}

/* ------------------------------------------------------------------ */
/* Block-scaled GEMM reference in fp64 ([KB] "Ökad                      */
/* ackumuleringsprecision", "Unified E4M3 Format"; [HS] 2.2 dequantize)  */
/*                                                                      */
/*   C[m,n] = sum_k (sa[m,k/128] dec(qa[m,k])) (sb[k/128,n/128] dec(qb(k,n)))  */
/*   T[m,n] = sum_k |same product|     (the size of the error bound)     */
/*                                                                      */
/* qb(k,n) = qb[n*ldb + k] when b_kmajor (B stored [N][K]),             */
/*           qb[k*ldb + n] otherwise    (B stored [K][N]).              */
/* ------------------------------------------------------------------ */

static double g_dec[256];
static int g_dec_ready = 0;

static void dec_table_init(void)
{
    int c;
    if (g_dec_ready)
        return;
    for (c = 0; c < 256; c++)
        g_dec[c] = orc_e4m3_decode((uint8_t)c);
    g_dec_ready = 1;
}

static void gemm_entry(const uint8_t* qa, int64_t lda, const float* sa,
                       int64_t sa_sm, int64_t sa_skb, const uint8_t* qb,
                       int64_t ldb, int b_kmajor, const float* sb,
                       int64_t sb_skb, int64_t sb_snb, int64_t K, int64_t m,
                       int64_t n, double* c_out, double* t_out)
{
    double c = 0.0, t = 0.0;
    int64_t k;
    for (k = 0; k < K; k++) {
        int64_t kb = k / ORC_TILE, nb = n / ORC_TILE;
        uint8_t cb = b_kmajor ? qb[n * ldb + k] : qb[k * ldb + n];
        double av = (double)sa[m * sa_sm + kb * sa_skb] * g_dec[qa[m * lda + k]];
        double bv = (double)sb[kb * sb_skb + nb * sb_snb] * g_dec[cb];
        c += av * bv;
        t += fabs(av * bv);
    }
    *c_out = c;
    if (t_out)
        *t_out = t;
}

void orc_gemm_ref(const uint8_t* qa, int64_t lda, const float* sa, int64_t sa_stride_m,
                  int64_t sa_stride_kb, const uint8_t* qb, int64_t ldb, int b_kmajor,
                  const float* sb, int64_t sb_stride_kb, int64_t sb_stride_nb,
                  int64_t M, int64_t N, int64_t K, double* C, double* T)
{
    int64_t m;
    dec_table_init();
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; m++) {
        int64_t n;
        for (n = 0; n < N; n++)
            gemm_entry(qa, lda, sa, sa_stride_m, sa_stride_kb, qb, ldb, b_kmajor, sb,
                       sb_stride_kb, sb_stride_nb, K, m, n, &C[m * N + n],
                       T ? &T[m * N + n] : NULL);
    }
}

void orc_gemm_ref_entries(const uint8_t* qa, int64_t lda, const float* sa,
                          int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* qb,
                          int64_t ldb, int b_kmajor, const float* sb,
                          int64_t sb_stride_kb, int64_t sb_stride_nb, int64_t K,
                          int64_t n_entries, const int64_t* rows, const int64_t* cols,
                          double* C, double* T)
{
    int64_t i;
    dec_table_init();
#pragma omp parallel for schedule(static)
    for (i = 0; i < n_entries; i++)
        gemm_entry(qa, lda, sa, sa_stride_m, sa_stride_kb, qb, ldb, b_kmajor, sb,
                   sb_stride_kb, sb_stride_nb, K, rows[i], cols[i], &C[i],
                   T ? &T[i] : NULL);
}

/* Grouped (MoE expert) form: rows [off[g], off[g+1]) of A use expert g's
 * B_g = qb + g*b_group_stride (stored [N][K], row stride ldb) and scales
 * sb + g*sb_stride_g.  C is [total_M][N]. */
void orc_grouped_gemm_ref(const uint8_t* qa, int64_t lda, const float* sa,
                          int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* qb,
                          int64_t ldb, int64_t b_group_stride, const float* sb,
                          int64_t sb_stride_g, int64_t sb_stride_kb, int64_t sb_stride_nb,
                          const int32_t* offsets, int G, int64_t N, int64_t K,
                          double* C, double* T)
{
    int g;
    dec_table_init();
    for (g = 0; g < G; g++) {
        int64_t m;
        const uint8_t* qb_g = qb + (int64_t)g * b_group_stride;
        const float* sb_g = sb + (int64_t)g * sb_stride_g;
#pragma omp parallel for schedule(static)
        for (m = offsets[g]; m < offsets[g + 1]; m++) {
            int64_t n;
            for (n = 0; n < N; n++)
                gemm_entry(qa, lda, sa, sa_stride_m, sa_stride_kb, qb_g, ldb, 1, sb_g,
                           sb_stride_kb, sb_stride_nb, K, m, n, &C[m * N + n],
                           T ? &T[m * N + n] : NULL);
        }
    }
}

/* Unquantized fp64 GEMM on the original operands, for reporting the
 * quantization error:  E[m,n] = sum_k x[m,k] * w(k,n), w(k,n) = w[k*ldw+n]. */
void orc_gemm_exact(const void* x, int x_type, int64_t ldx, const void* w, int w_type,
                    int64_t ldw, int64_t M, int64_t N, int64_t K, double* E)
{
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; m++) {
        int64_t n, k;
        for (n = 0; n < N; n++) {
            double acc = 0.0;
            for (k = 0; k < K; k++)
                acc += (double)load_in(x, x_type, m * ldx + k) *
                       (double)load_in(w, w_type, k * ldw + n);
            E[m * N + n] = acc;
        }
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

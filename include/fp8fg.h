/*
 * fp8fg.h -- C ABI of the fine-grained online FP8 library for NVIDIA B200
 * (sm_100a): online 1x128 / 128x128 E4M3 quantization and the block-scaled
 * FP8 GEMM (dense and MoE-grouped) that consumes its output.
 *
 * The method these calls implement is the FP8 mixed-precision scheme of
 * DeepSeek-V3 as described in
 *   [KB] codingmall.com knowledge base, "Kan du förklara rollen för FP8
 *        precision i träningsprocessen för DeepSeek-V3"
 *        (sections "Mixed Precision Framework", "Finkornig kvantisering",
 *        "Online-kvantisering", "Ökad ackumuleringsprecision",
 *        "Unified E4M3 Format"), and
 *   [HS] holysheep.ai, "FP8 混精度训练 DeepSeek 671B" (Chinese edition),
 *        section "2.2 细粒度量化实现" (scale = amax / 448, divide, cast to
 *        E4M3; dequantize = code value x scale).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - E4M3 is the "e4m3fn" encoding: bias 7, no infinities, NaN = S.1111.111,
 *    largest finite magnitude 448.  Codes are stored as raw bytes (uint8).
 *  - Quantization rounds x / scale (one IEEE fp32 division) to the nearest
 *    E4M3 value, ties to even, saturating to +-448; scale = amax / 448 in
 *    IEEE fp32, replaced by 1 when it is zero.  Results are bit-identical
 *    to that definition.
 *  - Pointers named as device pointers must be device (or managed) memory
 *    of the CURRENT CUDA device; the caller owns every buffer.  The library
 *    allocates no device memory and keeps no per-call state.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default
 *    stream).  Nothing synchronizes, prints, aborts or throws.
 *  - Matrices are row-major with a leading dimension (`ld*`, in ELEMENTS)
 *    between consecutive rows; the innermost dimension is contiguous.
 *  - Argument errors are reported synchronously by the return value, before
 *    any work is queued.  A problem with zero rows (or zero columns) is a
 *    valid no-op that returns FP8_OK; its pointers may then be NULL.
 *  - Requires a compute-capability 10.0 device (B200); any other device
 *    gives FP8_ERR_DEVICE.
 */
#ifndef FP8FG_H
#define FP8FG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FP8FG_API __attribute__((visibility("default")))
#else
#define FP8FG_API
#endif

struct CUstream_st;                       /* cudaStream_t == struct CUstream_st* */
typedef struct CUstream_st* fp8_stream_t;

typedef enum fp8_status {
    FP8_OK = 0,
    FP8_ERR_NULL = 1,          /* a required pointer is NULL                          */
    FP8_ERR_SHAPE = 2,         /* negative size, or a dimension not a multiple of 128 */
    FP8_ERR_ALIGN = 3,         /* a pointer or leading dimension breaks 16-byte rules */
    FP8_ERR_LAYOUT = 4,        /* strides/orientation this call does not support      */
    FP8_ERR_DTYPE = 5,         /* unknown element-type enum value                     */
    FP8_ERR_DEVICE = 6,        /* no current device, or it is not sm_100             */
    FP8_ERR_CUDA = 7,          /* a CUDA runtime/driver call failed                   */
    FP8_ERR_UNIMPLEMENTED = 8,
    FP8_ERR_DEVICE_TIMEOUT = 9 /* (from fp8_get_device_error) a kernel gave up waiting */
} fp8_status_t;

typedef enum fp8_in_type { FP8_IN_BF16 = 0, FP8_IN_FP32 = 1 } fp8_in_t;
typedef enum fp8_out_type { FP8_OUT_FP32 = 0, FP8_OUT_BF16 = 1 } fp8_out_t;

/*
 * fp8_quantize_act_1x128 -- online fine-grained activation quantization.
 * [KB] "Finkornig kvantisering" (activations in 1x128 tiles, each scaled on
 * its own) and "Online-kvantisering" (scale from the current values on every
 * call); [HS] 2.2 (scale = amax / 448, x / scale cast to E4M3).
 *
 * For every row m and every 128-wide tile kb of x [M, K]:
 *     amax        = max_k |x[m, k]|           (k in the tile)
 *     sa[m, kb]   = amax / 448   (1 if that is 0)
 *     q[m, k]     = E4M3_RNE_satfinite(x[m, k] / sa[m, kb])
 *
 *  x      device, [M, ldx] elements of type x_type (bf16 or fp32); 16-byte
 *         aligned, ldx * sizeof(elem) a multiple of 16, ldx >= K.
 *  M, K   M >= 0 any value; K >= 0 and a multiple of 128.
 *  q      device, [M, ldq] bytes written (codes); 16-byte aligned,
 *         ldq a multiple of 16, ldq >= K.
 *  sa     device fp32; sa[m * sa_stride_m + kb * sa_stride_kb] written for
 *         0 <= kb < K/128.  Any non-negative strides (e.g. [M, K/128]
 *         row-major: sa_stride_m = K/128, sa_stride_kb = 1).
 *  Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_DTYPE,
 *          FP8_ERR_LAYOUT (negative stride), FP8_ERR_DEVICE, FP8_ERR_CUDA.
 */
FP8FG_API fp8_status_t fp8_quantize_act_1x128(const void* x, fp8_in_t x_type, int64_t M, int64_t K,
                                    int64_t ldx, uint8_t* q, int64_t ldq, float* sa,
                                    int64_t sa_stride_m, int64_t sa_stride_kb,
                                    fp8_stream_t stream);

/*
 * fp8_quantize_act_1x128_gather -- fp8_quantize_act_1x128 of a row gather:
 * output row r is the 1x128 quantization of input row rows[r] (the MoE
 * dispatch that sorts routed tokens by expert), bit-identical to gathering
 * x[rows] first and quantizing that, without writing the gathered copy.
 * [KB] "Finkornig kvantisering", "Online-kvantisering"; [HS] 2.2.
 *
 *  x        device [src_rows, ldx] of x_type; alignment as fp8_quantize_act_1x128.
 *  rows     device int32 [R]: source row of each output row, 0 <= rows[r] <
 *           src_rows.  An index out of range leaves that output row
 *           unwritten and records FP8_ERR_SHAPE in the device error word.
 *  q, sa    output [R, ldq] codes and sa[r * sa_stride_m + kb * sa_stride_kb],
 *           as in fp8_quantize_act_1x128.
 *  K        a multiple of 128.
 */
FP8FG_API fp8_status_t fp8_quantize_act_1x128_gather(const void* x, fp8_in_t x_type,
                                                     int64_t src_rows, int64_t K, int64_t ldx,
                                                     const int32_t* rows, int64_t R, uint8_t* q,
                                                     int64_t ldq, float* sa, int64_t sa_stride_m,
                                                     int64_t sa_stride_kb, fp8_stream_t stream);

/*
 * fp8_quantize_act_1x128_scatter -- the MoE dispatch in token order: each
 * input row (token) t is quantized once, as fp8_quantize_act_1x128 would,
 * and its codes and scales are written to every output row named by
 * dest[t * topk + j], j < topk.  With dest the inverse of a gather's `rows`
 * (dest[t * topk + j] = r exactly when rows[r] = t), the output equals that
 * of fp8_quantize_act_1x128_gather bit for bit, but every token is read and
 * quantized once instead of once per destination.
 * [KB] "Finkornig kvantisering", "Online-kvantisering"; [HS] 2.2.
 *
 *  x        device bf16 [T, ldx]; 16-byte aligned, ldx * 2 % 16 == 0,
 *           ldx >= K.  fp32 input gives FP8_ERR_DTYPE (use the gather form).
 *  T, K     T >= 0 tokens; K >= 0 a multiple of 128.
 *  dest     device int32 [T, topk] (row-major, 4-byte aligned): output rows
 *           of token t; -1 marks no destination.  Any other value outside
 *           [0, R) is skipped and records FP8_ERR_SHAPE in the device error
 *           word.  An output row named twice receives one of the writers'
 *           tiles (which one is undefined); rows named by no entry are not
 *           written.
 *  topk     >= 0 destinations per token (0: nothing to do).
 *  q        device codes [R, ldq]; 32-byte aligned and ldq a multiple of 32
 *           (the codes leave as 32-byte stores), ldq >= K.
 *  R        rows of q and sa.
 *  sa       device fp32, sa[r * sa_stride_m + kb * sa_stride_kb], 4-byte aligned.
 *  Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_DTYPE,
 *          FP8_ERR_LAYOUT, FP8_ERR_DEVICE, FP8_ERR_CUDA.
 */
FP8FG_API fp8_status_t fp8_quantize_act_1x128_scatter(const void* x, fp8_in_t x_type, int64_t T,
                                                      int64_t K, int64_t ldx,
                                                      const int32_t* dest, int64_t topk,
                                                      uint8_t* q, int64_t R, int64_t ldq,
                                                      float* sa, int64_t sa_stride_m,
                                                      int64_t sa_stride_kb, fp8_stream_t stream);

/*
 * fp8_quantize_weight_128x128 -- online fine-grained weight quantization.
 * [KB] "Finkornig kvantisering" (weights in 128x128 blocks, each scaled on
 * its own), "Online-kvantisering"; [HS] 2.2.
 *
 * For every 128x128 block (kb, nb) of w [K, N]:
 *     sb[kb, nb] = amax(block) / 448   (1 if that is 0)
 *     code(k, n) = E4M3_RNE_satfinite(w[k, n] / sb[kb, nb])
 * written to q[k * ldq + n] (transpose_out == 0, q is [K, N]) or
 * q[n * ldq + k] (transpose_out == 1, q is [N, K]: the K-major operand the
 * forward GEMM reads).  The untransposed [K, N] form is itself the K-major
 * operand of the transposed product (dgrad, dX = dY W^T), with sb read as
 * [nb][kb]; one quantization of w serves both products.
 *
 *  w      device, [K, ldw] elements of w_type; 16-byte aligned,
 *         ldw * sizeof(elem) a multiple of 16, ldw >= N.
 *  K, N   multiples of 128 (>= 0).
 *  q      device bytes, 16-byte aligned, ldq a multiple of 16,
 *         ldq >= N (transpose_out == 0) or >= K (transpose_out == 1).
 *  sb     device fp32, sb[kb * sb_stride_kb + nb * sb_stride_nb].
 */
FP8FG_API fp8_status_t fp8_quantize_weight_128x128(const void* w, fp8_in_t w_type, int64_t K,
                                         int64_t N, int64_t ldw, uint8_t* q,
                                         int transpose_out, int64_t ldq, float* sb,
                                         int64_t sb_stride_kb, int64_t sb_stride_nb,
                                         fp8_stream_t stream);

/*
 * fp8_blockscaled_gemm -- FP8 GEMM with per-chunk FP32 promotion.
 * [KB] "Mixed Precision Framework" (the GEMMs run in FP8), "Ökad
 * ackumuleringsprecision" (tensor-core partial sums promoted to FP32
 * registers at fixed intervals), "Unified E4M3 Format"; [HS] 2.2 dequantize.
 *
 *     C[m, n] = sum_kb  sa[m, kb] * sb[kb, n/128] * P_kb[m, n]
 *     P_kb[m, n] = sum_{k in chunk kb} E4M3(a[m, k]) * E4M3(b(n, k))
 *
 * The promotion interval is one 128-wide K chunk (the scaling unit): each
 * chunk's tensor-core partial P_kb is scaled and added into an FP32
 * accumulator.  C is written as fp32 or bf16 (round to nearest even).
 *
 *  a      device codes [M, lda] (K-major), 16-byte aligned, lda % 16 == 0,
 *         lda >= K.
 *  sa     device fp32, sa[m * sa_stride_m + kb * sa_stride_kb].
 *  b      device codes; b_kmajor must be 1: b is [N, ldb], b(n, k) =
 *         b[n * ldb + k], 16-byte aligned, ldb % 16 == 0, ldb >= K.
 *         (b_kmajor == 0 gives FP8_ERR_LAYOUT; quantize with
 *         transpose_out = 1 to obtain the K-major operand.)
 *  sb     device fp32, sb[kb * sb_stride_kb + nb * sb_stride_nb].
 *  c      device [M, ldc] of c_type, 16-byte aligned,
 *         ldc * sizeof(elem) % 16 == 0, ldc >= N.
 *  M      >= 0, any value (rows beyond M are never written).
 *  N, K   multiples of 128 (>= 0).  K == 0 writes C = 0.
 */
FP8FG_API fp8_status_t fp8_blockscaled_gemm(const uint8_t* a, int64_t lda, const float* sa,
                                  int64_t sa_stride_m, int64_t sa_stride_kb,
                                  const uint8_t* b, int64_t ldb, int b_kmajor,
                                  const float* sb, int64_t sb_stride_kb,
                                  int64_t sb_stride_nb, void* c, fp8_out_t c_type,
                                  int64_t ldc, int64_t M, int64_t N, int64_t K,
                                  fp8_stream_t stream);

/*
 * fp8_blockscaled_gemm_quant -- fp8_blockscaled_gemm whose output leaves
 * already quantized for the next layer: the GEMM epilogue rounds each row
 * of C to bf16 and quantizes every 1x128 tile of that bf16 row as
 * fp8_quantize_act_1x128 does ([KB] "Finkornig kvantisering",
 * "Online-kvantisering"), so codes and scales are bit-identical to
 * fp8_blockscaled_gemm (bf16 out) followed by fp8_quantize_act_1x128 on C,
 * without the round trip of C through memory.
 *
 *  a, sa, b, sb  as in fp8_blockscaled_gemm (b K-major, [N, ldb]).
 *  qc     device codes [M, ldqc]; 16-byte aligned, ldqc % 16 == 0, ldqc >= N.
 *  sc     device fp32, sc[m * sc_stride_m + (n / 128) * sc_stride_nb]
 *         (e.g. [M, N/128] row-major: sc_stride_m = N/128, sc_stride_nb = 1).
 *  c      optional device bf16 [M, ldc] copy of the rounded output (NULL: not
 *         written); 16-byte aligned, ldc * 2 % 16 == 0, ldc >= N.
 *  M >= 0 any value; N and K multiples of 128, K > 0 (K == 0: FP8_ERR_SHAPE).
 *  Errors: as fp8_blockscaled_gemm.
 */
FP8FG_API fp8_status_t fp8_blockscaled_gemm_quant(const uint8_t* a, int64_t lda, const float* sa,
                                                  int64_t sa_stride_m, int64_t sa_stride_kb,
                                                  const uint8_t* b, int64_t ldb, const float* sb,
                                                  int64_t sb_stride_kb, int64_t sb_stride_nb,
                                                  uint8_t* qc, int64_t ldqc, float* sc,
                                                  int64_t sc_stride_m, int64_t sc_stride_nb,
                                                  void* c, int64_t ldc, int64_t M, int64_t N,
                                                  int64_t K, fp8_stream_t stream);

/*
 * fp8_quantize_act_128x1 -- 1x128 quantization of x^T, for the weight-
 * gradient product dW = x^T dY, whose contraction runs over the M rows
 * (tokens) of x: the activation tiles of [KB] "Finkornig kvantisering",
 * taken along M, scaled on every call ("Online-kvantisering"), in the one
 * E4M3 format of forward and backward ("Unified E4M3 Format"); [HS] 2.2.
 * For every column k of x [M, K] and every 128 rows mb:
 *     amax           = max_m |x[m, k]|          (m in [128 mb, 128 mb + 128))
 *     st[k, mb]      = amax / 448   (1 if that is 0)
 *     qt[k, m]       = E4M3_RNE_satfinite(x[m, k] / st[k, mb])
 * i.e. fp8_quantize_act_1x128 of the transposed matrix, written [K, M].
 *
 *  x      device bf16 [M, ldx]; 16-byte aligned, ldx * 2 % 16 == 0, ldx >= K.
 *         fp32 input: FP8_ERR_DTYPE.
 *  qt     device codes [K, ldq]; 16-byte aligned, ldq % 16 == 0, ldq >= M.
 *  st     device fp32, st[k * st_stride_k + mb * st_stride_mb] for
 *         0 <= mb < M/128 (e.g. [K, M/128]: st_stride_k = M/128,
 *         st_stride_mb = 1, the layout of sa for fp8_blockscaled_gemm_colscale;
 *         or [M/128, K]: st_stride_k = 1, st_stride_mb = K, its sb layout).
 *  M, K   multiples of 128 (else FP8_ERR_SHAPE); 0 is a no-op.
 *  NaN inputs are skipped by amax and encode to the NaN code.
 */
FP8FG_API fp8_status_t fp8_quantize_act_128x1(const void* x, fp8_in_t x_type, int64_t M, int64_t K,
                                              int64_t ldx, uint8_t* qt, int64_t ldq, float* st,
                                              int64_t st_stride_k, int64_t st_stride_mb,
                                              fp8_stream_t stream);

/*
 * fp8_blockscaled_gemm_colscale -- the block-scaled GEMM with 1x128 tiles
 * on BOTH operands, as the weight gradient needs (both x^T and dY^T are
 * quantized along the tokens, fp8_quantize_act_128x1): B has one scale
 * per row n and 128-wide K chunk instead of one per 128 x 128 block.  Each
 * chunk's tensor-core partial is promoted into FP32 with the scale
 * products ([KB] "Ökad ackumuleringsprecision"):
 *
 *     C[m, n] = sum_kb sa[m, kb] * sb[kb, n] * P_kb[m, n]
 *
 *  a, sa  as in fp8_blockscaled_gemm ([M, lda] codes, sa[m * sa_stride_m +
 *         kb * sa_stride_kb]).
 *  b      device codes [N, ldb], K contiguous; alignment as a.
 *  sb     device fp32 [K/128, sb_stride_kb]: sb[kb * sb_stride_kb + n], n
 *         contiguous; 16-byte aligned; when K > 128 also
 *         sb_stride_kb % 4 == 0 and sb_stride_kb >= N (one chunk: any
 *         stride).
 *  c      device [M, ldc] of c_type; as fp8_blockscaled_gemm.
 *  M >= 0 any value; N and K multiples of 128; K == 0 writes C = 0.
 *  Errors: as fp8_blockscaled_gemm.
 */
FP8FG_API fp8_status_t fp8_blockscaled_gemm_colscale(const uint8_t* a, int64_t lda, const float* sa,
                                                     int64_t sa_stride_m, int64_t sa_stride_kb,
                                                     const uint8_t* b, int64_t ldb, const float* sb,
                                                     int64_t sb_stride_kb, void* c,
                                                     fp8_out_t c_type, int64_t ldc, int64_t M,
                                                     int64_t N, int64_t K, fp8_stream_t stream);

/*
 * fp8_grouped_gemm -- the block-scaled GEMM over MoE expert groups.
 * Same arithmetic as fp8_blockscaled_gemm ([KB] "Mixed Precision
 * Framework", "Ökad ackumuleringsprecision"), applied per expert g to the
 * rows [offsets[g], offsets[g+1]) of a (rows sorted by expert):
 *
 *     C[m, n] = sum_kb sa[m, kb] * sb_g[kb, n/128] * P_kb[m, n]   with B_g
 *
 *  a, sa  as in fp8_blockscaled_gemm, total_M rows.
 *  b      device codes [G][N][ldb] (each expert K-major, experts contiguous:
 *         expert g starts at b + g * N * ldb); alignment as above.
 *  sb     device fp32, sb[g * sb_stride_g + kb * sb_stride_kb + nb * sb_stride_nb].
 *  c      device [total_M, ldc] of c_type.
 *  offsets device int32 [G + 1]: offsets[0] = 0, non-decreasing,
 *         offsets[G] = total_M.  Read on the device (no host sync).  A
 *         decreasing pair makes that group empty and records
 *         FP8_ERR_SHAPE in the device error word; rows at or beyond
 *         total_M are never read or written.
 *  G      1 <= G <= 1024.
 *  Launches: for K >= 4096 two kernels on `stream` (CTA-pair tiles of 256
 *  rows for each group's whole 256-row blocks and remainders over 128 rows,
 *  then one-CTA tiles of 128 rows for remainders of 1-128 rows; they write
 *  disjoint rows of c), else one.  Both read offsets on the device.
 */
FP8FG_API fp8_status_t fp8_grouped_gemm(const uint8_t* a, int64_t lda, const float* sa,
                              int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* b,
                              int64_t ldb, const float* sb, int64_t sb_stride_g,
                              int64_t sb_stride_kb, int64_t sb_stride_nb, void* c,
                              fp8_out_t c_type, int64_t ldc, const int32_t* offsets, int G,
                              int64_t total_M, int64_t N, int64_t K, fp8_stream_t stream);

/*
 * fp8_dequantize -- E4M3 codes back to real values.
 * [HS] 2.2 (dequantize: code value times the tile's scale), the inverse
 * direction of the two quantize calls above.
 *
 *     out[r, c] = E4M3(q[r, c]) * s[r / tile_rows, c / 128]
 *
 * one IEEE fp32 multiply, round to nearest; written as fp32, or as bf16
 * (that fp32 value rounded to nearest even).  NaN codes give NaN.
 *
 *  q          device codes [rows, ldq]; 16-byte aligned, ldq % 16 == 0, ldq >= cols.
 *  rows       >= 0, any value.  cols >= 0, a multiple of 128.
 *  s          device fp32, s[(r / tile_rows) * s_stride_r + (c / 128) * s_stride_c]
 *             (non-negative strides).
 *  tile_rows  1 (activation tiles, sa [M, K/128]) or 128 (weight blocks,
 *             sb [K/128, N/128]); anything else gives FP8_ERR_SHAPE.
 *  out        device [rows, ldo] of out_type; 16-byte aligned,
 *             ldo * sizeof(elem) % 16 == 0, ldo >= cols.
 *  Errors: FP8_ERR_NULL, FP8_ERR_SHAPE, FP8_ERR_ALIGN, FP8_ERR_LAYOUT,
 *          FP8_ERR_DTYPE, FP8_ERR_DEVICE, FP8_ERR_CUDA.
 */
FP8FG_API fp8_status_t fp8_dequantize(const uint8_t* q, int64_t rows, int64_t cols, int64_t ldq,
                                      const float* s, int64_t s_stride_r, int64_t s_stride_c,
                                      int tile_rows, void* out, fp8_out_t out_type, int64_t ldo,
                                      fp8_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
FP8FG_API const char* fp8_status_string(fp8_status_t status);

/*
 * fp8_get_device_error -- synchronizes `stream`, then reads and clears the
 * current device's error word.  Kernels record into it when a bounded wait
 * gives up (FP8_ERR_DEVICE_TIMEOUT; the kernel then stops early and its
 * outputs are undefined) or when the grouped GEMM or the gathering
 * quantizer meets invalid offsets or row indices (FP8_ERR_SHAPE).  *code
 * receives the recorded status (FP8_OK if none).
 *
 * There is ONE error word per device, shared by every stream and every call
 * of this library on that device: the first error recorded since the last
 * read is kept (later ones are dropped), and whoever reads it clears it.
 * Only `stream` is synchronized, so a kernel still running on another
 * stream may record an error after this read.  Callers that use several
 * streams should read the word only after synchronizing all of them, and
 * from one place.
 * Returns FP8_ERR_NULL if `code` is NULL, FP8_ERR_CUDA if the
 * synchronization or the read fails.
 */
FP8FG_API fp8_status_t fp8_get_device_error(fp8_stream_t stream, fp8_status_t* code);

/*
 * fp8_set_wait_limit -- sets, for the current device, how many SM clock
 * cycles any wait of this library's kernels may last before the kernel
 * gives up (records FP8_ERR_DEVICE_TIMEOUT, waits for its own copies and
 * tensor-core work in flight, releases its tensor memory and returns, so
 * that the context stays usable).  cycles == 0 restores the default,
 * 2^31 cycles (about one second at the B200's clock).  A test sets a few
 * hundred cycles to make real waits run out and exercise that path; the
 * results of calls made under such a limit are undefined.
 * Synchronizes the device before the change.  Not for use while other
 * threads queue work on the device.
 * Errors: FP8_ERR_SHAPE (cycles < 0), FP8_ERR_DEVICE, FP8_ERR_CUDA.
 */
FP8FG_API fp8_status_t fp8_set_wait_limit(int64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* FP8FG_H */

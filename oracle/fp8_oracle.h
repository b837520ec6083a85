/*
 * fp8_oracle.h -- declarations of the plain CPU oracle (test
 * infrastructure only; see fp8_oracle.c for what each function follows).
 * This header belongs to the oracle alone: the CUDA library neither
 * includes it nor links the oracle.
 */
#ifndef FP8_ORACLE_H
#define FP8_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_IN_BF16 = 0, ORC_IN_FP32 = 1 };

double  orc_e4m3_decode(uint8_t c);
uint8_t orc_e4m3_encode(float v);
void    orc_e4m3_decode_array(const uint8_t* c, int64_t n, double* out);
void    orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out);

void orc_quantize_act_1x128(const void* x, int in_type, int64_t M, int64_t K,
                            int64_t ldx, uint8_t* q, int64_t ldq, float* sa,
                            int64_t sa_stride_m, int64_t sa_stride_kb);

void orc_quantize_weight_128x128(const void* w, int in_type, int64_t K, int64_t N,
                                 int64_t ldw, uint8_t* q, int transpose_out,
                                 int64_t ldq, float* sb, int64_t sb_stride_kb,
                                 int64_t sb_stride_nb);

void orc_gemm_ref(const uint8_t* qa, int64_t lda, const float* sa, int64_t sa_stride_m,
                  int64_t sa_stride_kb, const uint8_t* qb, int64_t ldb, int b_kmajor,
                  const float* sb, int64_t sb_stride_kb, int64_t sb_stride_nb,
                  int64_t M, int64_t N, int64_t K, double* C, double* T);

void orc_gemm_ref_entries(const uint8_t* qa, int64_t lda, const float* sa,
                          int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* qb,
                          int64_t ldb, int b_kmajor, const float* sb,
                          int64_t sb_stride_kb, int64_t sb_stride_nb, int64_t K,
                          int64_t n_entries, const int64_t* rows, const int64_t* cols,
                          double* C, double* T);

void orc_grouped_gemm_ref(const uint8_t* qa, int64_t lda, const float* sa,
                          int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* qb,
                          int64_t ldb, int64_t b_group_stride, const float* sb,
                          int64_t sb_stride_g, int64_t sb_stride_kb, int64_t sb_stride_nb,
                          const int32_t* offsets, int G, int64_t N, int64_t K,
                          double* C, double* T);

void orc_gemm_exact(const void* x, int x_type, int64_t ldx, const void* w, int w_type,
                    int64_t ldw, int64_t M, int64_t N, int64_t K, double* E);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8_ORACLE_H */

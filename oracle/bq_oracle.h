/*
 * bq_oracle.h -- declarations of the CPU oracle (test infrastructure only; see
 * bq_oracle.c). This header belongs to the oracle alone: the product library neither
 * includes it nor is included by it.
 */
#ifndef BQ_ORACLE_H
#define BQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { BQO_BINARY = 0, BQO_TERNARY = 1, BQO_TERNARY_B3 = 2 };
enum { BQO_X_F16 = 0, BQO_X_BF16 = 1 };
enum { BQO_OK = 0, BQO_ERR_SHAPE = 1, BQO_ERR_CODE = 2 };

double bqo_f16_to_f64(uint16_t h);
double bqo_bf16_to_f64(uint16_t b);
uint16_t bqo_f64_to_bf16(double v);
uint16_t bqo_f64_to_f16(double v);
void bqo_f64_to_bf16_array(const double *v, int64_t n, uint16_t *out);

int64_t bqo_words_per_row(int fmt, int64_t K);
int64_t bqo_row_bytes(int fmt, int64_t K);

int bqo_pack_binary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                         uint32_t *words, uint16_t *s_out);
int bqo_pack_ternary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                          uint32_t *words, uint16_t *s_out);
int64_t bqo_unpack_binary_g128(const uint32_t *words, int64_t N, int64_t K, int8_t *q);
int64_t bqo_unpack_ternary_g128(const uint32_t *words, int64_t N, int64_t K, int8_t *q);
int bqo_pack_ternary_b3(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                        uint8_t *bytes, uint16_t *s_out);
int64_t bqo_unpack_ternary_b3(const uint8_t *bytes, int64_t N, int64_t K, int8_t *q);

double bqo_weight(int fmt, const uint32_t *words, const uint16_t *scales, int64_t K,
                  int64_t n, int64_t k);
int bqo_dequant(int fmt, const uint32_t *words, const uint16_t *scales, int64_t N, int64_t K,
                double *Wd);
int bqo_gemv_rows(int fmt, const uint16_t *x, int xt, int64_t M, int64_t K,
                  const uint32_t *words, const uint16_t *scales, int64_t N,
                  const int64_t *rows, int64_t R, double *y, double *bound);
int64_t bqo_embed(int fmt, const int32_t *ids, int64_t T, const uint32_t *words,
                  const uint16_t *scales, int64_t N, int64_t K, double *out);
uint16_t bqo_mlx_affine_dequant(uint16_t s_f16, int q01);
int bqo_mlp_swiglu(int fmt_gu, const uint16_t *x, int xt, int64_t M, int64_t K, const uint32_t *wg,
                   const uint16_t *sg, const uint32_t *wu, const uint16_t *su, int64_t F, int fmt_d,
                   const uint32_t *wd, const uint16_t *sd, int64_t N, double *a, double *y, double *bound);
int bqo_quantize_g128(int fmt, const float *w, int64_t N, int64_t K, int8_t *q, uint16_t *s);
int bqo_topk(const double *y, int64_t M, int64_t N, int k, int64_t *idx, double *vals);
int64_t bqo_sample_topk(const double *vals, const int64_t *idx, int k, double T, double top_p, double u);

#ifdef __cplusplus
}
#endif
#endif

/*
 * mx_oracle.h -- declarations of the CPU oracle (test infrastructure only).
 * See mx_oracle.c for the definitions each function follows.
 */
#ifndef MX_ORACLE_H
#define MX_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

double mxo_e4m3_decode(uint8_t code);
void mxo_e4m3_table(double out[256]);
uint8_t mxo_e4m3_encode(double v);
double mxo_ue8m0_decode(uint8_t code);
int mxo_floor_log2(double a);
double mxo_bf16_to_double(uint16_t bits);

void mxo_quantize_block(const uint16_t *x, uint8_t *q, uint8_t *scale);
void mxo_quantize(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, uint8_t *sf);
void mxo_quantize_block_f32(const float *x, uint8_t *q, uint8_t *scale);
void mxo_quantize_f32(const float *x, int64_t rows, int64_t k, uint8_t *q, uint8_t *sf);
double mxo_silu(double x);
void mxo_swiglu(const double *g, const double *u, int64_t n, double *h);

int64_t mxo_scale_bytes(int64_t rows, int64_t k);
int64_t mxo_sf_offset(int64_t r, int64_t c, int64_t k);
void mxo_sf_tile(const uint8_t *sf_rm, int64_t rows, int64_t k, uint8_t *tiled);
void mxo_sf_untile(const uint8_t *tiled, int64_t rows, int64_t k, uint8_t *sf_rm);

void mxo_gemm(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb, const uint8_t *sfb,
              int64_t m, int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows,
              double *d, double *abssum);
void mxo_grouped_contiguous(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                            const uint8_t *sfb, const int32_t *offsets, int32_t groups,
                            int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows,
                            double *d, double *abssum);
void mxo_grouped_masked(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                        const uint8_t *sfb, const int32_t *masked_m, int32_t groups,
                        int64_t max_m, int64_t n, int64_t k, const int64_t *row_ids,
                        int64_t nrows, double *d, double *abssum);
void mxo_grouped_kgrouped(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                          const uint8_t *sfb, const int32_t *offsets, int32_t groups,
                          int64_t m, int64_t n, int64_t k_total, const int64_t *row_ids,
                          int64_t nrows, double *d, double *abssum);
void mxo_tw_quantize_rows(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, float *s);
void mxo_tw_quantize_blocks(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, float *s);
void mxo_tw_gemm(const uint8_t *qa, const float *sa, const uint8_t *qb, const float *sb, int64_t m,
                 int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows, double *d,
                 double *abssum);
int64_t mxo_moe_route(const int32_t *ids, int64_t n, int32_t E, int32_t pad, int32_t *counts,
                      int32_t *offsets, int32_t *row);
void mxo_moe_peer_plan(const int32_t *ids, const int64_t *n_of, int32_t ranks, int32_t E, int32_t pad,
                       int32_t *dst_rank, int32_t *dst_row, int32_t *counts_local, int32_t *offsets_local);
void mxo_moe_dispatch(const uint16_t *x, int64_t T, int64_t k, const int32_t *row, int64_t topk,
                      int64_t m_rows, uint8_t *q, uint8_t *sf_rm);
void mxo_moe_combine(const uint16_t *y, int64_t n, const int32_t *row, const float *w, int64_t T,
                     int64_t topk, double *out, double *abssum);
int mxo_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif

/* W4A8 oracle: plain CPU reference.  TEST INFRASTRUCTURE ONLY (see the
 * header comment of w4a8_oracle.c).  This header belongs to the oracle alone;
 * the CUDA library has its own, unrelated header. */
#ifndef W4A8_ORACLE_H
#define W4A8_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

float orc_bf16_to_f32(uint16_t h);
uint16_t orc_f64_to_bf16(double y);
void orc_f64_to_bf16_array(const double* y, size_t n, uint16_t* out);

int orc_quant_row_f32(const float* x, int K, int8_t* q, float* s_out);
int orc_quant_act_bf16(const uint16_t* X, int M, int K, int ldx, int group,
                       int8_t* q, float* s_x, int32_t* rowsum);

int orc_quant_weights(const float* W, int K, int N, int group, int symmetric,
                      int8_t* codes, float* s, uint8_t* z);
void orc_dequant_weights(const int8_t* codes, const float* s, const uint8_t* z,
                         int K, int N, int group, double* What);
void orc_pack_canonical(const int8_t* codes, int K, int N, uint8_t* out);
void orc_pack_tiled(const int8_t* codes, int K, int N, int group, uint8_t* out);

void orc_partials(const int8_t* qx, const int8_t* codes, const uint8_t* z,
                  int M, int K, int N, int group, int32_t* P);
void orc_scale_partials(const int32_t* P, const float* s_x, const float* s_w,
                        int M, int G, int N, double* Y, double* absY);
void orc_dequant_gemm(const int8_t* qx, const float* s_x, const int8_t* codes,
                      const float* s_w, const uint8_t* z, int M, int K, int N,
                      int group, double* Y);

int orc_route(const float* logits, int T, int E, int topk, int32_t* idx, double* p);
void orc_dispatch(const int32_t* idx, int T, int E, int topk,
                  int32_t* offsets, int32_t* perm, int32_t* inv);
double orc_silu(double x);
void orc_silu_mul(const double* H, int R, int I, uint16_t* h);
void orc_combine(const uint16_t* Yd, const double* p, const int32_t* inv,
                 int T, int topk, int Hd, uint16_t* out, double* out_f64);

#ifdef __cplusplus
}
#endif
#endif

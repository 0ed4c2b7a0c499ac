/*
 * oref.h -- the oracle's own declarations (test infrastructure only; shares
 * nothing with the CUDA library or its header).
 */
#ifndef OREF_H
#define OREF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OREF_OK = 0, OREF_ERR_SHAPE = -1, OREF_ERR_VALUE = -2, OREF_ERR_ALLOC = -3 };

double   oref_half_to_double(uint16_t h);
float    oref_half_to_float(uint16_t h);
uint16_t oref_double_to_half(double v);
uint16_t oref_float_to_half(float v);

int oref_pack_ternary(const int8_t *w, int N, int K, uint32_t *w2);
int oref_pack_sign(const uint16_t *w, int N, int K, uint32_t *s1);
int oref_quant_act(const uint16_t *x, int M, int K, int8_t *q, float *s);
int oref_ternary_linear(const uint16_t *x, int M, int K, int N, const uint32_t *w2,
                        float w_scale, uint16_t *y, int32_t *acc_out);
int oref_ob_linear(const uint16_t *x, int M, int K, int N, const uint32_t *s1,
                   const uint16_t *g, const uint16_t *h, uint16_t *y, double *z_out);
int oref_svid(const float *W, int N, int K, int8_t *S, double *a, double *b,
              double *sigma_out, int max_iter, double tol);
int oref_rmsnorm(const uint16_t *x, int M, int K, const uint16_t *gamma, double eps, uint16_t *y);
int oref_swiglu(const uint16_t *a, const uint16_t *b, int n, uint16_t *y);
int oref_billm_binarize(const float *W, int N, int K, int8_t *Bo, int8_t *Br, double *alpha_o,
                        double *alpha_r);
int oref_billm_linear(const uint16_t *x, int M, int K, int N, const uint32_t *bo1,
                      const uint32_t *br1, const uint16_t *alpha_o, const uint16_t *alpha_r,
                      uint16_t *y, double *z_out);
int64_t oref_onebit_bits(int64_t N, int64_t K);
int64_t oref_onebit_params(int64_t N, int64_t K);

#ifdef __cplusplus
}
#endif
#endif

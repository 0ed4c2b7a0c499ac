/*
 * oref.c -- the oracle: a plain, slow, scalar CPU restatement of what the
 * extreme-low-bit linear layer computes.  TEST INFRASTRUCTURE ONLY: the test
 * suite, the smoke check and the benchmark's CPU-baseline leg call it; the
 * product path (the CUDA library) never does, and the two share no code.
 *
 * Sources (web pages, cited by title and section):
 *   [B158] "微软、国科大开启1Bit时代：大模型转三进制，速度快4倍能耗降至1/41"
 *          (BitNet b1.58), sections "BitNet b1.58 介绍", "内存和延迟", "能耗".
 *   [ONEBIT] "清华、哈工大把大模型压缩到了1bit，把大模型放在手机里跑的愿望就快要实现了！"
 *          (OneBit), sections "1. 新的 1bit 结构", "2. 基于 SVID 初始化量化模型",
 *          "3. 通过知识蒸馏迁移原模型能力", "讨论与分析 / 1. 效率".
 *   [BILLM] "BiLLM: Pushing the Limit of Post-Training Quantization for LLMs",
 *          section "方法细节：残差近似与最优断点拆分", step 2 (binary residual
 *          approximation).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (float arithmetic
 * is IEEE binary32 with round-to-nearest-even; no fused multiply-add).  A
 * second build adds -fopenmp: the two linear forms then compute their output
 * rows n in parallel on the host cores (each output is still the same scalar
 * loop over k, in the same order, so the results are identical); the plain
 * build ignores the pragmas and runs on one core.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - activation range [-Qb, Qb] with Qb = 127, symmetric, no zero point;
 *   - scale computed as inv = 127/amax, then q = RNE(x*inv) clamped to +-127;
 *   - an all-zero token gives q = 0 and scale 0;
 *   - the ternary weight and its per-tensor scale are given inputs (the pages
 *     do not say how they are obtained);
 *   - sign(0) = +1 (exactly two states are needed);
 *   - g scales the input dimension K, h the output dimension N;
 *   - OneBit accumulates in fp64 here (the exact definition the GPU's fp32
 *     accumulation is judged against).
 *
 * Packed formats (little-endian 32-bit words, row-major):
 *   ternary: weight (n,k) occupies bits [2*(k%16), 2*(k%16)+1] of word
 *            [n][k/16]; the stored code is t+1 (0 -> -1, 1 -> 0, 2 -> +1),
 *            code 3 is never written and is rejected when read;
 *   sign:    bit (k%32) of word [n][k/32] is 1 iff the sign is +1.
 */
#include "oref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------
 * IEEE 754 binary16 <-> binary32/64, written from the format definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).
 * ------------------------------------------------------------------- */
double oref_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);  /* (1.f) * 2^(e-15) */
    return sign ? -v : v;
}

float oref_half_to_float(uint16_t h) { return (float)oref_half_to_double(h); }

/* Round a double to the nearest binary16, ties to even (single rounding). */
uint16_t oref_double_to_half(double v)
{
    uint16_t sign = 0;
    if (isnan(v)) return 0x7e00;
    if (signbit(v)) { sign = 0x8000; v = -v; }
    if (v == 0.0) return sign;
    /* Largest finite half is 65504; the midpoint to the next binade step
     * (65536, not representable) is 65520, which rounds to even = overflow. */
    if (v >= 65520.0) return sign | 0x7c00;
    if (v < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24 */
        double m = nearbyint(v * ldexp(1.0, 24));
        return sign | (uint16_t)m;              /* m == 1024 gives min normal */
    }
    int E;
    frexp(v, &E);                               /* v = f*2^E, f in [0.5,1) */
    int e = E - 1;                              /* v in [2^e, 2^(e+1)) */
    double m = nearbyint(ldexp(v, 10 - e));     /* in [1024, 2048] */
    if (m == 2048.0) { m = 1024.0; e += 1; }
    if (e + 15 >= 31) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)m - 1024));
}

uint16_t oref_float_to_half(float v) { return oref_double_to_half((double)v); }

/* ---------------------------------------------------------------------
 * Packing.  [B158] "BitNet b1.58 介绍": every weight is one of {-1, 0, 1}
 * (1.58 bits of information); "内存和延迟" measures with a 2-bit kernel, so
 * the weight is stored in 2 bits.  [ONEBIT] "3. 通过知识蒸馏…": after
 * training the post-Sign() parameters are saved and used for inference;
 * "讨论与分析 / 1. 效率": a pure binary parameter is one 0/1 bit.
 * ------------------------------------------------------------------- */
int oref_pack_ternary(const int8_t *w, int N, int K, uint32_t *w2)
{
    if (N < 0 || K < 0 || K % 16 != 0) return OREF_ERR_SHAPE;
    int words = K / 16;
    for (int n = 0; n < N; ++n) {
        for (int j = 0; j < words; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 16; ++i) {
                int t = w[(size_t)n * K + (size_t)j * 16 + i];
                if (t < -1 || t > 1) return OREF_ERR_VALUE;
                uint32_t code = (uint32_t)(t + 1);
                word |= code << (2 * i);
            }
            w2[(size_t)n * words + j] = word;
        }
    }
    return OREF_OK;
}

/* sign(w) as the bit stored: 1 for +1, 0 for -1; sign(+-0) = +1. */
int oref_pack_sign(const uint16_t *w, int N, int K, uint32_t *s1)
{
    if (N < 0 || K < 0 || K % 32 != 0) return OREF_ERR_SHAPE;
    int words = K / 32;
    for (int n = 0; n < N; ++n) {
        for (int j = 0; j < words; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 32; ++i) {
                double v = oref_half_to_double(w[(size_t)n * K + (size_t)j * 32 + i]);
                if (isnan(v)) return OREF_ERR_VALUE;
                uint32_t bit = (v < 0.0) ? 0u : 1u;
                word |= bit << i;
            }
            s1[(size_t)n * words + j] = word;
        }
    }
    return OREF_OK;
}

/* Decode one ternary weight from the packed format; -2 marks code 3. */
static int ternary_at(const uint32_t *w2, int K, int n, int k)
{
    uint32_t word = w2[(size_t)n * (K / 16) + k / 16];
    int code = (int)((word >> (2 * (k % 16))) & 3u);
    return code == 3 ? -2 : code - 1;
}

static int sign_at(const uint32_t *s1, int K, int n, int k)
{
    uint32_t word = s1[(size_t)n * (K / 32) + k / 32];
    return ((word >> (k % 32)) & 1u) ? 1 : -1;
}

/* ---------------------------------------------------------------------
 * [B158] "BitNet b1.58 介绍": activations are quantised per token to the
 * symmetric range [-Qb, Qb] (no zero point), Qb = 127 for 8 bits.
 * Per token m: amax = max_k |x|; inv = 127/amax (fp32); q = RNE(x*inv)
 * clamped to [-127, 127]; scale s = amax/127 (fp32).  All-zero -> 0, 0.
 * ------------------------------------------------------------------- */
int oref_quant_act(const uint16_t *x, int M, int K, int8_t *q, float *s)
{
    if (M < 0 || K < 0) return OREF_ERR_SHAPE;
    for (int m = 0; m < M; ++m) {
        const uint16_t *row = x + (size_t)m * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(oref_half_to_float(row[k]));
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            for (int k = 0; k < K; ++k) q[(size_t)m * K + k] = 0;
            s[m] = 0.0f;
            continue;
        }
        float inv = 127.0f / amax;
        for (int k = 0; k < K; ++k) {
            float v = oref_half_to_float(row[k]) * inv;
            float r = nearbyintf(v);            /* ties to even */
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[(size_t)m * K + k] = (int8_t)r;
        }
        s[m] = amax / 127.0f;
    }
    return OREF_OK;
}

/* ---------------------------------------------------------------------
 * [B158] BitLinear forward (no bias: "BitNet b1.58 介绍" removes all
 * biases).  acc = sum_k q[m,k]*t[n,k] in integers (add/subtract only,
 * "能耗": INT8 additions), then y = fp16(((float)acc * s_m) * w_scale).
 * acc_out (may be NULL) receives the int32 accumulators [M,N];
 * q_out/s_out (may be NULL) receive the quantised activations.
 * ------------------------------------------------------------------- */
int oref_ternary_linear(const uint16_t *x, int M, int K, int N, const uint32_t *w2,
                        float w_scale, uint16_t *y, int32_t *acc_out)
{
    if (M < 0 || N < 0 || K < 0 || K % 16 != 0) return OREF_ERR_SHAPE;
    int8_t *q = (int8_t *)malloc((size_t)M * K + 1);
    float *s = (float *)malloc((size_t)M * sizeof(float) + 4);
    if (!q || !s) { free(q); free(s); return OREF_ERR_ALLOC; }
    oref_quant_act(x, M, K, q, s);
    int rc = OREF_OK;
    for (int m = 0; m < M && rc == OREF_OK; ++m) {
        int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
        for (int n = 0; n < N; ++n) {
            int64_t acc = 0;
            int row_bad = 0;
            for (int k = 0; k < K; ++k) {
                int t = ternary_at(w2, K, n, k);
                if (t == -2) { row_bad = 1; break; }
                int qv = q[(size_t)m * K + k];
                if (t == 1) acc += qv;
                else if (t == -1) acc -= qv;
            }
            if (row_bad) { bad = 1; continue; }
            float a = (float)(int32_t)acc;      /* |acc| <= 127*K < 2^24 here */
            float v = (a * s[m]) * w_scale;
            if (acc_out) acc_out[(size_t)m * N + n] = (int32_t)acc;
            if (y) y[(size_t)m * N + n] = oref_float_to_half(v);
        }
        if (bad) rc = OREF_ERR_VALUE;
    }
    free(q);
    free(s);
    return rc;
}

/* ---------------------------------------------------------------------
 * [ONEBIT] "1. 新的 1bit 结构": the 1-bit linear layer keeps a +-1 matrix
 * and two FP16 value vectors g and h:  y = ((x (.) g) . sign(W)^T) (.) h,
 * g over the input dimension K, h over the output dimension N.
 * Contraction in fp64 (exact products of fp16 values, fp64 sums);
 * z_out (may be NULL) receives z*h in fp64 before the final fp16 rounding.
 * ------------------------------------------------------------------- */
int oref_ob_linear(const uint16_t *x, int M, int K, int N, const uint32_t *s1,
                   const uint16_t *g, const uint16_t *h, uint16_t *y, double *z_out)
{
    if (M < 0 || N < 0 || K < 0 || K % 32 != 0) return OREF_ERR_SHAPE;
    for (int m = 0; m < M; ++m) {
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double z = 0.0;
            for (int k = 0; k < K; ++k) {
                double xg = oref_half_to_double(x[(size_t)m * K + k]) *
                            oref_half_to_double(g[k]);
                z += sign_at(s1, K, n, k) > 0 ? xg : -xg;
            }
            double v = z * oref_half_to_double(h[n]);
            if (z_out) z_out[(size_t)m * N + n] = v;
            if (y) y[(size_t)m * N + n] = oref_double_to_half(v);
        }
    }
    return OREF_OK;
}

/* ---------------------------------------------------------------------
 * [ONEBIT] "2. 基于 SVID 初始化量化模型": split W into its sign matrix and
 * its magnitude, and approximate |W| by a rank-1 product a b^T (the page
 * allows SVD or NMF).  The dominant singular pair of the non-negative
 * matrix |W| is found by power iteration in fp64 from the all-ones start
 * vector, stopping when sigma changes by < tol relative or after max_iter
 * rounds; sqrt(sigma) is split evenly so a = sqrt(sigma) u, b = sqrt(sigma) v.
 * By the order swap the page describes, a plays the role of h (over N) and
 * b of g (over K).  S receives sign(W) as +-1 with sign(0) = +1.
 * Returns the number of iterations used (>0), or a negative error.
 * ------------------------------------------------------------------- */
int oref_svid(const float *W, int N, int K, int8_t *S, double *a, double *b,
              double *sigma_out, int max_iter, double tol)
{
    if (N <= 0 || K <= 0) return OREF_ERR_SHAPE;
    double *u = (double *)malloc((size_t)N * sizeof(double));
    double *v = (double *)malloc((size_t)K * sizeof(double));
    if (!u || !v) { free(u); free(v); return OREF_ERR_ALLOC; }
    for (size_t i = 0; i < (size_t)N * K; ++i) S[i] = W[i] < 0.0f ? -1 : 1;
    for (int k = 0; k < K; ++k) v[k] = 1.0 / sqrt((double)K);
    double sigma = 0.0;
    int it;
    for (it = 1; it <= max_iter; ++it) {
        double nu = 0.0;
        for (int n = 0; n < N; ++n) {            /* u = |W| v */
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += fabs((double)W[(size_t)n * K + k]) * v[k];
            u[n] = acc;
            nu += acc * acc;
        }
        nu = sqrt(nu);
        for (int n = 0; n < N; ++n) u[n] /= nu;
        for (int k = 0; k < K; ++k) v[k] = 0.0;   /* v = |W|^T u */
        for (int n = 0; n < N; ++n)
            for (int k = 0; k < K; ++k) v[k] += fabs((double)W[(size_t)n * K + k]) * u[n];
        double nv = 0.0;
        for (int k = 0; k < K; ++k) nv += v[k] * v[k];
        nv = sqrt(nv);
        for (int k = 0; k < K; ++k) v[k] /= nv;
        double prev = sigma;
        sigma = nv;                               /* ||A^T u|| with unit u */
        if (it > 1 && fabs(sigma - prev) <= tol * sigma) break;
    }
    if (it > max_iter) it = max_iter;
    double r = sqrt(sigma);
    for (int n = 0; n < N; ++n) a[n] = r * u[n];
    for (int k = 0; k < K; ++k) b[k] = r * v[k];
    if (sigma_out) *sigma_out = sigma;
    free(u);
    free(v);
    return it;
}

/* ---------------------------------------------------------------------
 * [B158] "BitNet b1.58 介绍": the model keeps LLaMA's components, RMSNorm and
 * SwiGLU, around its BitLinear layers.  Reading used here (the page gives no
 * formulas): RMSNorm of one token
 *     r = 1 / sqrt(sum_k x_k^2 / K + eps),   y_k = fp16((x_k * r) * gamma_k)
 * and SwiGLU  y = fp16((a / (1 + exp(-a))) * b).
 * Precision: fp64.  The sum of squares is exact (integers) and rounded once
 * to fp64; every later operation is one IEEE fp64 rounding, then one
 * rounding to fp16.  So a result is fixed by its inputs alone (SwiGLU up to
 * the accuracy of exp).
 * ------------------------------------------------------------------- */

/* nearest double (ties to even) of the 128-bit integer hi * 2^64 + lo */
static double u128_to_double(uint64_t hi, uint64_t lo)
{
    if (hi == 0) return (double)lo;             /* one IEEE conversion */
    int nbits = 64;                             /* bit length of hi */
    while (!(hi >> (nbits - 1))) --nbits;
    int sh = nbits;                             /* drop the low sh bits: keep 64 */
    uint64_t top = sh == 64 ? hi : (hi << (64 - sh)) | (lo >> sh);
    uint64_t rest = sh == 64 ? lo : lo & ((((uint64_t)1) << sh) - 1);
    /* top has 64 significant bits, 53 are kept: a set bit 0 stands for any
     * nonzero rest (it lies below the rounding position) */
    double d = (double)(top | (rest ? 1u : 0u));
    return ldexp(d, sh);
}

int oref_rmsnorm(const uint16_t *x, int M, int K, const uint16_t *gamma, double eps, uint16_t *y)
{
    if (M < 0 || K <= 0) return OREF_ERR_SHAPE;
    for (int m = 0; m < M; ++m) {
        const uint16_t *row = x + (size_t)m * K;
        /* x = mant * 2^e exactly (mant < 2^11, e in [-24, 5]); x^2 * 2^48 is an
         * integer below 2^80; the sum of K of them fits 128 bits */
        uint64_t hi = 0, lo = 0;
        for (int k = 0; k < K; ++k) {
            int ex = (row[k] >> 10) & 31, f = row[k] & 1023;
            if (ex == 31) return OREF_ERR_VALUE;
            uint64_t mant = ex ? (uint64_t)(1024 | f) : (uint64_t)f;
            int e = (ex ? ex : 1) - 25;
            int sh = 2 * e + 48;                 /* 0 .. 58 */
            uint64_t sq = mant * mant;           /* < 2^22 */
            uint64_t add_lo = sh < 64 ? sq << sh : 0, add_hi = sh == 0 ? 0 : sq >> (64 - sh);
            uint64_t nlo = lo + add_lo;
            hi += add_hi + (nlo < lo ? 1u : 0u);
            lo = nlo;
        }
        double ss = ldexp(u128_to_double(hi, lo), -48);
        double r = 1.0 / sqrt(ss / (double)K + eps);
        for (int k = 0; k < K; ++k)
            y[(size_t)m * K + k] = oref_double_to_half((oref_half_to_double(row[k]) * r) *
                                                       oref_half_to_double(gamma[k]));
    }
    return OREF_OK;
}

int oref_swiglu(const uint16_t *a, const uint16_t *b, int n, uint16_t *y)
{
    if (n < 0) return OREF_ERR_SHAPE;
    for (int i = 0; i < n; ++i) {
        double av = oref_half_to_double(a[i]);
        double silu = av / (1.0 + exp(-av));
        y[i] = oref_double_to_half(silu * oref_half_to_double(b[i]));
    }
    return OREF_OK;
}

/* [ONEBIT] "1. 新的 1bit 结构" worked example: storage of an N x K OneBit
 * layer = N*K one-bit signs + (N + K) fp16 values. */
int64_t oref_onebit_bits(int64_t N, int64_t K) { return N * K + 16 * (N + K); }
int64_t oref_onebit_params(int64_t N, int64_t K) { return N * K + N + K; }

/* ---------------------------------------------------------------------
 * [BILLM] step 2, binary residual approximation: binarise W (alpha_o B_o),
 * binarise what is left (alpha_r B_r), and use W ~ alpha_o B_o + alpha_r B_r.
 * Readings (the page gives neither the granularity nor the formula of the
 * scales): one scale per output row n; B = sign(.) with sign(0) = +1; alpha =
 * the mean absolute value of the row being binarised, which is the scale that
 * minimises || row - alpha B ||_2 once B = sign(row).  fp64 throughout.
 * ------------------------------------------------------------------- */
int oref_billm_binarize(const float *W, int N, int K, int8_t *Bo, int8_t *Br, double *alpha_o,
                        double *alpha_r)
{
    if (N < 0 || K <= 0) return OREF_ERR_SHAPE;
    for (int n = 0; n < N; ++n) {
        const float *row = W + (size_t)n * K;
        double so = 0.0;
        for (int k = 0; k < K; ++k) so += fabs((double)row[k]);
        const double ao = so / (double)K;
        double sr = 0.0;
        for (int k = 0; k < K; ++k) {
            int8_t b = row[k] < 0.0f ? -1 : 1;
            Bo[(size_t)n * K + k] = b;
            sr += fabs((double)row[k] - ao * (double)b);
        }
        const double ar = sr / (double)K;
        for (int k = 0; k < K; ++k) {
            double r = (double)row[k] - ao * (double)Bo[(size_t)n * K + k];
            Br[(size_t)n * K + k] = r < 0.0 ? -1 : 1;
        }
        alpha_o[n] = ao;
        alpha_r[n] = ar;
    }
    return OREF_OK;
}

/* The two-plane binary linear layer: y = x W~^T with
 *     W~[n][k] = alpha_o[n] B_o[n][k] + alpha_r[n] B_r[n][k],
 * B_o and B_r as packed sign planes (the s1 format), alpha_o and alpha_r as
 * fp16 [N] (the stored scales), activations fp16 and not quantised (the page:
 * only the weights are binarised).  z = sum_k x_k W~[n][k] in fp64, in k
 * order, y = fp16(z). */
int oref_billm_linear(const uint16_t *x, int M, int K, int N, const uint32_t *bo1,
                      const uint32_t *br1, const uint16_t *alpha_o, const uint16_t *alpha_r,
                      uint16_t *y, double *z_out)
{
    if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return OREF_ERR_SHAPE;
    const int words = K / 32;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const double ao = oref_half_to_double(alpha_o[n]);
        const double ar = oref_half_to_double(alpha_r[n]);
        for (int m = 0; m < M; ++m) {
            double z = 0.0;
            for (int k = 0; k < K; ++k) {
                const int so = (bo1[(size_t)n * words + k / 32] >> (k % 32)) & 1 ? 1 : -1;
                const int sr = (br1[(size_t)n * words + k / 32] >> (k % 32)) & 1 ? 1 : -1;
                const double w = ao * (double)so + ar * (double)sr;
                z += oref_half_to_double(x[(size_t)m * K + k]) * w;
            }
            y[(size_t)m * N + n] = oref_double_to_half(z);
            if (z_out) z_out[(size_t)m * N + n] = z;
        }
    }
    return OREF_OK;
}

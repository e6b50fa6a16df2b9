/*
 * W4A8 oracle: a plain, slow, obviously-correct CPU implementation of what the
 * W4A8 quantized Linear / MoE-expert path computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm may load this code.  It shares nothing with
 * the CUDA path (no headers, helpers, tables or generators): every function
 * below is written from the pages' definitions.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * OpenMP only splits independent output rows; no result depends on it.
 *
 * Sources (page title, section):
 *   [Q-FMT]  "Quantization: formats, error and the real execution path",
 *            sections "Basic mapping", "Symmetric group-wise reference",
 *            "Correctness contract".
 *   [LIN]    "Inference Quantization ch.1 (the Linear layer)", §1 problem
 *            statement, §2 worked INT8 example, §4 W8A8 ideal path, §5 outlier
 *            example, §6 scale/zero-point mapping, §7 zero-point expansion,
 *            §8.2-8.4 granularity, §9.2 dynamic per-token scale.
 *   [KIMI]   "Kimi 2.7 MoE, 4-bit storage to INT8", §3.3 per-token INT8 code,
 *            §4.1-4.4 MoE flow (router in high precision, top-k, dispatch,
 *            expert GEMM, weighted combine in 16-bit), §5.2 two codes per byte.
 *   [DEPLOY] "Kimi 2.7 MoE W4A8 deployment in practice", §2.1 (min/max affine
 *            4-bit formula), §2.2 (per-token dynamic INT8 activations).
 *
 * Readings taken where the pages are silent or disagree (each one is listed
 * with its reason in the design notes):
 *   R1 rounding: round-half-to-even of the fp32 quotient (torch.round).
 *   R2 division: the correctly rounded fp32 quotient x / s, then rounding.
 *   R3 activation clamp +-127, no epsilon in the scale.
 *   R4 zero scale: divide by 1, keep the stored scale 0 (codes all 0).
 *   R6 asymmetric: range widened to include 0, integer zero-point
 *      z = clamp(rne(-lo/s), 0, 15), q = clamp(rne(w/s) + z, 0, 15).
 *   R7 scales are fp32.
 *   R8 groups run along K of W[K,N] (never across an output column n).
 *   R10 top-k: logits descending, ties to the lower expert index.
 *   R11 routing weights: softmax over all E experts, not renormalised.
 *   R12 gate = columns [0, I), up = [I, 2I) of the gate_up output.
 *   R13 h and expert outputs are rounded to bf16; combine in high precision.
 *   R14 dispatch order: stable by (expert, token, slot).
 */
#include "w4a8_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16 <-> binary64                                                   */
/* ------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h)
{
    /* bf16 is the top half of an IEEE binary32: widening is exact. */
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

uint16_t orc_f64_to_bf16(double y)
{
    /* Correctly rounded (nearest, ties to even) binary64 -> bf16, taken in one
     * step from the double so there is no double rounding through binary32.
     * bf16 has 8 significant bits; its smallest quantum (subnormals) is
     * 2^-133; its largest finite value is 255 * 2^120. */
    if (isnan(y)) return (uint16_t)0x7FC0;
    uint16_t sign = signbit(y) ? (uint16_t)0x8000 : (uint16_t)0;
    double a = fabs(y);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    (void)frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int qexp = e - 8;                   /* spacing of bf16 values near a */
    if (qexp < -133) qexp = -133;
    double r = nearbyint(ldexp(a, -qexp)); /* exact scaling, RNE to integer */
    double v = ldexp(r, qexp);
    if (v > ldexp(255.0, 120)) return (uint16_t)(sign | 0x7F80);
    float f = (float)v;                 /* exact: <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ------------------------------------------------------------------ */
/* Per-token INT8 activation quantization                              */
/* [LIN] §9.2: s_x[i] = max|X[i,:]| / 127;  [KIMI] §3.3; [DEPLOY] §2.2. */
/* ------------------------------------------------------------------ */

int orc_quant_row_f32(const float* x, int K, int8_t* q, float* s_out)
{
    int bad = 0;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
        if (!isfinite(x[k])) bad = 1;
        float a = fabsf(x[k]);
        if (a > amax) amax = a;
    }
    float s = amax / 127.0f;                 /* IEEE binary32 division (R2) */
    float d = (s > 0.0f) ? s : 1.0f;         /* R4 */
    for (int k = 0; k < K; ++k) {
        float t = nearbyintf(x[k] / d);      /* RNE of the fp32 quotient (R1) */
        if (t > 127.0f) t = 127.0f;          /* R3 */
        if (t < -127.0f) t = -127.0f;
        q[k] = (int8_t)t;
    }
    *s_out = s;
    return bad;
}

int orc_quant_act_bf16(const uint16_t* X, int M, int K, int ldx, int group,
                       int8_t* q, float* s_x, int32_t* rowsum)
{
    if (M < 0 || K <= 0 || ldx < K) return -1;
    if (rowsum && (group <= 0 || K % group != 0)) return -1;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int m = 0; m < M; ++m) {
        float* row = (float*)malloc(sizeof(float) * (size_t)K);
        for (int k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(X[(size_t)m * ldx + k]);
        bad |= orc_quant_row_f32(row, K, q + (size_t)m * K, s_x + m);
        free(row);
        if (rowsum) {
            /* [LIN] §7: the per-group sum of activation codes that multiplies
             * the weight zero-point in the expanded product. */
            int G = K / group;
            for (int gi = 0; gi < G; ++gi) {
                int32_t acc = 0;
                for (int k = gi * group; k < (gi + 1) * group; ++k) acc += q[(size_t)m * K + k];
                rowsum[(size_t)m * G + gi] = acc;
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* Group-wise 4-bit weight quantization                                 */
/* ------------------------------------------------------------------ */

int orc_quant_weights(const float* W, int K, int N, int group, int symmetric,
                      int8_t* codes, float* s, uint8_t* z)
{
    /* [Q-FMT] "Symmetric group-wise reference": the group length must tile
     * the reduced dimension exactly, otherwise the call is rejected. */
    if (group <= 0 || K <= 0 || N <= 0 || K % group != 0) return -1;
    const int G = K / group;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int gi = 0; gi < G; ++gi) {
            const int k0 = gi * group, k1 = k0 + group;
            if (symmetric) {
                /* [Q-FMT] "Basic mapping": s = max|x| / (2^(b-1) - 1), z = 0;
                 * codes clip to [-7, 7]. */
                float amax = 0.0f;
                for (int k = k0; k < k1; ++k) {
                    float w = W[(size_t)k * N + n];
                    if (!isfinite(w)) bad = 1;
                    if (fabsf(w) > amax) amax = fabsf(w);
                }
                float sc = amax / 7.0f;
                float d = (sc > 0.0f) ? sc : 1.0f;
                for (int k = k0; k < k1; ++k) {
                    float t = nearbyintf(W[(size_t)k * N + n] / d);
                    if (t > 7.0f) t = 7.0f;
                    if (t < -7.0f) t = -7.0f;
                    codes[(size_t)n * K + k] = (int8_t)t;
                }
                s[(size_t)gi * N + n] = sc;
                if (z) z[(size_t)gi * N + n] = 0;
            } else {
                /* [Q-FMT] "Basic mapping" affine form, with [LIN] §6:
                 * s = (max - min) / (2^b - 1), q = clip(round(x/s) + z, 0, 15),
                 * x_hat = s (q - z).  R6: range widened to include 0 and an
                 * integer zero-point. */
                float lo = 0.0f, hi = 0.0f;
                for (int k = k0; k < k1; ++k) {
                    float w = W[(size_t)k * N + n];
                    if (!isfinite(w)) bad = 1;
                    if (w < lo) lo = w;
                    if (w > hi) hi = w;
                }
                float sc = (hi - lo) / 15.0f;
                float d = (sc > 0.0f) ? sc : 1.0f;
                float zf = nearbyintf(-lo / d);
                if (zf < 0.0f) zf = 0.0f;
                if (zf > 15.0f) zf = 15.0f;
                for (int k = k0; k < k1; ++k) {
                    float t = nearbyintf(W[(size_t)k * N + n] / d) + zf;
                    if (t < 0.0f) t = 0.0f;
                    if (t > 15.0f) t = 15.0f;
                    codes[(size_t)n * K + k] = (int8_t)t;
                }
                s[(size_t)gi * N + n] = sc;
                z[(size_t)gi * N + n] = (uint8_t)zf;
            }
        }
    }
    return bad;
}

void orc_dequant_weights(const int8_t* codes, const float* s, const uint8_t* z,
                         int K, int N, int group, double* What)
{
    /* x_hat = s (q - z), in binary64 (exact for 4-bit codes and fp32 s). */
    const int G = K / group;
    (void)G;
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n) {
            int gi = k / group;
            int zz = z ? (int)z[(size_t)gi * N + n] : 0;
            What[(size_t)k * N + n] = (double)s[(size_t)gi * N + n] *
                                      (double)((int)codes[(size_t)n * K + k] - zz);
        }
}

/* ------------------------------------------------------------------ */
/* Packing: two 4-bit codes per byte ([KIMI] §5.2)                      */
/* ------------------------------------------------------------------ */

static uint8_t nib(int8_t code) { return (uint8_t)(((unsigned)code) & 0xFu); }

void orc_pack_canonical(const int8_t* codes, int K, int N, uint8_t* out)
{
    /* Canonical order: W^T [N][K/2], K-major, low nibble = even k, codes as
     * 4-bit two's complement (symmetric) or uint4 (asymmetric). */
    for (int n = 0; n < N; ++n)
        for (int kb = 0; kb < K / 2; ++kb)
            out[(size_t)n * (K / 2) + kb] =
                (uint8_t)(nib(codes[(size_t)n * K + 2 * kb]) |
                          (nib(codes[(size_t)n * K + 2 * kb + 1]) << 4));
}

void orc_pack_tiled(const int8_t* codes, int K, int N, int group, uint8_t* out)
{
    /* The device layout as the library header specifies it, restated here
     * from that written specification:
     *   blocks of 64 output columns x one K-group, block (nb, gi) at byte
     *   (nb * G + gi) * 32 * group;
     *   inside a block, 16-byte chunk (c, r) at (c * 64 + r) * 16 for
     *   c in [0, group/32) and r in [0, 64), n = 64 nb + r;
     *   byte b of chunk c holds k = gi*group + 32c + b in its low nibble and
     *   k + 16 in its high nibble. */
    const int G = K / group;
    const int NB = N / 64;
    for (int nb = 0; nb < NB; ++nb)
        for (int gi = 0; gi < G; ++gi)
            for (int c = 0; c < group / 32; ++c)
                for (int r = 0; r < 64; ++r)
                    for (int b = 0; b < 16; ++b) {
                        int n = 64 * nb + r;
                        int k = gi * group + 32 * c + b;
                        size_t off = ((size_t)nb * G + gi) * 32u * (size_t)group +
                                     ((size_t)c * 64 + r) * 16 + b;
                        out[off] = (uint8_t)(nib(codes[(size_t)n * K + k]) |
                                             (nib(codes[(size_t)n * K + k + 16]) << 4));
                    }
}

/* ------------------------------------------------------------------ */
/* Exact integer partials and the factorised-scale product              */
/* ------------------------------------------------------------------ */

void orc_partials(const int8_t* qx, const int8_t* codes, const uint8_t* z,
                  int M, int K, int N, int group, int32_t* P)
{
    /* P[m,g,n] = sum_{k in g} q_x[m,k] * (q_w[k,n] - z[g,n])  (exact int32).
     * [LIN] §4 ideal path (int32 accumulation) and §7 (zero-point term). */
    const int G = K / group;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int gi = 0; gi < G; ++gi)
            for (int n = 0; n < N; ++n) {
                int zz = z ? (int)z[(size_t)gi * N + n] : 0;
                int32_t acc = 0;
                for (int k = gi * group; k < (gi + 1) * group; ++k)
                    acc += (int32_t)qx[(size_t)m * K + k] *
                           ((int32_t)codes[(size_t)n * K + k] - zz);
                P[((size_t)m * G + gi) * N + n] = acc;
            }
}

void orc_scale_partials(const int32_t* P, const float* s_x, const float* s_w,
                        int M, int G, int N, double* Y, double* absY)
{
    /* Y[m,n] = s_x[m] * sum_g s_w[g,n] * P[m,g,n]   ([LIN] §8.3 epilogue
     * form, per group), in binary64.  absY (optional) = sum_g |terms|. */
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int gi = 0; gi < G; ++gi) {
                double t = (double)s_w[(size_t)gi * N + n] * (double)P[((size_t)m * G + gi) * N + n];
                acc += t;
                aacc += fabs(t);
            }
            Y[(size_t)m * N + n] = (double)s_x[m] * acc;
            if (absY) absY[(size_t)m * N + n] = fabs((double)s_x[m]) * aacc;
        }
}

void orc_dequant_gemm(const int8_t* qx, const float* s_x, const int8_t* codes,
                      const float* s_w, const uint8_t* z, int M, int K, int N,
                      int group, double* Y)
{
    /* The "dequantize, then GEMM" form ([LIN] §3.1, §11 "bad path"):
     * Y = (s_x q_x) (s_w (q_w - z)), every product formed in binary64.
     * Used only as an identity check against the factorised form. */
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) {
                int gi = k / group;
                int zz = z ? (int)z[(size_t)gi * N + n] : 0;
                double xa = (double)s_x[m] * (double)qx[(size_t)m * K + k];
                double wb = (double)s_w[(size_t)gi * N + n] *
                            (double)((int)codes[(size_t)n * K + k] - zz);
                acc += xa * wb;
            }
            Y[(size_t)m * N + n] = acc;
        }
}

/* ------------------------------------------------------------------ */
/* MoE routing, dispatch order, SiLU gate, combine ([KIMI] §4.1-4.4)    */
/* ------------------------------------------------------------------ */

int orc_route(const float* logits, int T, int E, int topk, int32_t* idx, double* p)
{
    if (T < 0 || E <= 0 || topk <= 0 || topk > E) return -1;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        char* taken = (char*)calloc((size_t)E, 1);
        for (int e = 0; e < E; ++e)
            if (!isfinite(l[e])) bad = 1;
        /* top-k of the logits (= top-k of the softmax, which is monotone):
         * repeated selection of the largest remaining logit, ties to the
         * lower expert index (R10). */
        for (int j = 0; j < topk; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            idx[(size_t)t * topk + j] = best;
        }
        /* softmax over all E experts in binary64 (R11: not renormalised). */
        double mx = -INFINITY;
        for (int e = 0; e < E; ++e) if ((double)l[e] > mx) mx = (double)l[e];
        double den = 0.0;
        for (int e = 0; e < E; ++e) den += exp((double)l[e] - mx);
        for (int j = 0; j < topk; ++j)
            p[(size_t)t * topk + j] = exp((double)l[idx[(size_t)t * topk + j]] - mx) / den;
        free(taken);
    }
    return bad;
}

void orc_dispatch(const int32_t* idx, int T, int E, int topk,
                  int32_t* offsets, int32_t* perm, int32_t* inv)
{
    /* Count per expert, exclusive prefix sum, then place every (token, slot)
     * pair in (expert, token, slot) order (R14).  perm[pos] = t*topk + j,
     * inv[t*topk + j] = pos. */
    int32_t* cnt = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (size_t i = 0; i < (size_t)T * topk; ++i) cnt[idx[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + cnt[e];
    for (int e = 0; e < E; ++e) {
        int32_t pos = offsets[e];
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < topk; ++j)
                if (idx[(size_t)t * topk + j] == e) {
                    perm[pos] = t * topk + j;
                    inv[(size_t)t * topk + j] = pos;
                    ++pos;
                }
    }
    free(cnt);
}

double orc_silu(double x)
{
    /* SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x)). */
    return x / (1.0 + exp(-x));
}

void orc_silu_mul(const double* H, int R, int I, uint16_t* h)
{
    /* h = silu(gate) * up with gate = H[:, :I], up = H[:, I:] (R12),
     * rounded once to bf16 (R13). */
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r)
        for (int i = 0; i < I; ++i) {
            double gte = H[(size_t)r * 2 * I + i];
            double up = H[(size_t)r * 2 * I + I + i];
            h[(size_t)r * I + i] = orc_f64_to_bf16(orc_silu(gte) * up);
        }
}

void orc_combine(const uint16_t* Yd, const double* p, const int32_t* inv,
                 int T, int topk, int Hd, uint16_t* out, double* out_f64)
{
    /* out[t] = sum_j p[t,j] * y_{t,j} in binary64, slot order j = 0..k-1,
     * rounded once to bf16 ([KIMI] §4.3: weighted accumulate kept in
     * 16-bit-or-wider precision, not in the integer domain). */
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < Hd; ++n) {
            double acc = 0.0;
            for (int j = 0; j < topk; ++j) {
                int32_t r = inv[(size_t)t * topk + j];
                acc += p[(size_t)t * topk + j] * (double)orc_bf16_to_f32(Yd[(size_t)r * Hd + n]);
            }
            if (out_f64) out_f64[(size_t)t * Hd + n] = acc;
            if (out) out[(size_t)t * Hd + n] = orc_f64_to_bf16(acc);
        }
}

void orc_f64_to_bf16_array(const double* y, size_t n, uint16_t* out)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(y[i]);
}

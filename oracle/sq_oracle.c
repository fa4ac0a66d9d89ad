/*
 * CPU oracle for the SmoothQuant W8A8 linear-layer path and the LLM.int8()
 * mixed-precision decomposition.
 *
 * TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
 * baseline leg may call it; the product path never does. It shares no code
 * with the CUDA library. Build with strict IEEE semantics:
 *     gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * so that every float operation below is one correctly rounded fp32 (or fp64)
 * operation, exactly as written.
 *
 * Sources (page title, section):
 *   [SQ-p1] lpnh.cn SmoothQuant practice article, §2.1 (s_j formula), §3.2
 *           (calibrate: clamp(min=1e-5) on both statistics and on s), §3.3
 *           (weight * s, activation divided by s).
 *   [SQ-p2] "大语言模型量化技术（四）：SmoothQuant", sections 为什么激活不能用逐通道量化
 *           (scales only per token / per output channel), SmoothQuant 的原理
 *           (Y = (X S^-1)(S W)), 缩放因子 (x_j, w_j, s_j = x_j^a / w_j^(1-a),
 *           closed forms at a = 0, 0.5, 1), 缩放的代价 (per-channel weight
 *           quantisation is invariant to channel scaling), 缩放的效果 (worked
 *           two-channel example), 融入 LayerNorm (gamma' = gamma/s,
 *           beta' = beta/s).
 *   [SQ-p4] "如何通过 SmoothQuant 解决激活值离群点难题", §3 (smooth_layer_weights:
 *           per-channel max of |input|, max of |weight| over the output
 *           dimension, s clamped at 1e-5, weight multiplied by s on the input
 *           dimension, input divided by s).
 *   [SQ-p5] "8位量化：异常值与混合精度分解实战", §2.1 (absmax and vector-wise
 *           quantisation: scale = 127 / max(|x|, 1e-8), round, clip to
 *           [-127, 127], int32 accumulation, dequantisation by the outer
 *           product of the scales), §2.2 (outlier dimensions |x| > 6.0 with a
 *           min_ratio of tokens, 16-bit product of the outlier columns plus
 *           the int8 product of the rest), §4.1 (any value over the threshold
 *           marks its dimension).
 *
 * Readings where the pages leave a step open (each is restated where used):
 *   R1 calibration statistics are running maxima over all batches;
 *   R2 s_j is computed in fp64 from fp32 statistics and rounded once to fp32;
 *      the clamps of [SQ-p1] §3.2 are applied to x_j, w_j and s_j;
 *   R3 the weight fold is done in fp32 (one rounding per product);
 *   R4 quantisation: qs = 127 / max(m, 1e-8), q = clip(round_half_even(v*qs))
 *      in fp32; dequantisation divides by qs_x * qs_w in fp64;
 *   R5 the normalisation sums follow a fixed reduction order (below);
 *   R6 LLM.int8: the outlier test is strict (|x| > thr); min_ratio = 0 means
 *      any one element marks the column; the 16-bit path is exact products
 *      summed in ascending outlier order, added to the dequantised int8 path;
 *   R9 the MLP activation SiLU is evaluated with a fixed fp32 exponential
 *      (below); R10 the fold into the previous linear divides its output
 *      channels by s in fp32; R11 FP8 is OCP E4M3 with the absmax rule
 *      scaled to its largest value 448.
 */
#include "sq_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float absf(float v) { return v < 0.0f ? -v : v; }
static double absd(double v) { return v < 0.0 ? -v : v; }

/* round half to even, clipped to [-127, 127]   [SQ-p5] §2.1 */
static int8_t q_clip(float t) {
    float r = rintf(t); /* default rounding mode: to nearest, ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* quantisation scale from an absmax   [SQ-p5] §2.1 quantize_vectorwise */
static float scale_of(float m) {
    float d = m > 1e-8f ? m : 1e-8f;
    return 127.0f / d;
}

/* ------------------------------------------------------------------ calibration absmax
 * x_j = max_i |X_ij| over all calibration tokens; w_j = max over every output
 * channel of |W| in input channel j.   [SQ-p2] 缩放因子; [SQ-p1] §3.2;
 * [SQ-p4] §3.  Reading R1: running max across calls (p1's hook keeps only
 * the last batch).  Pinned by: brute force on small inputs (exact). */
void or_col_absmax(const float* X, int64_t M, int64_t K, int64_t ld, float* io) {
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j) {
            float a = absf(X[i * ld + j]);
            if (a > io[j]) io[j] = a;
        }
}

/* ------------------------------------------------------------------ smoothing factors and folds
 * s_j = x_j^alpha / w_j^(1-alpha)   [SQ-p2] 缩放因子, [SQ-p1] §2.1, [SQ-p4] §3.
 * Clamps at 1e-5 before and after   [SQ-p1] §3.2 (R2).
 * alpha = 0, 1/2, 1 use the page's closed forms 1/w, sqrt(x/w), x.
 * Pinned by: closed forms at powers of two for alpha in {0.4, 0.5, 0.6},
 * the worked example of [SQ-p2] 缩放的效果, and the alpha = 1/2 balance. */
void or_smooth_scales(const float* x, const float* w, int64_t K, double alpha, float* s) {
    for (int64_t j = 0; j < K; ++j) {
        float xc = x[j] > 1e-5f ? x[j] : 1e-5f;
        float wc = w[j] > 1e-5f ? w[j] : 1e-5f;
        double v;
        if (alpha == 0.5)
            v = sqrt((double)xc / (double)wc);
        else if (alpha == 0.0)
            v = 1.0 / (double)wc;
        else if (alpha == 1.0)
            v = (double)xc;
        else
            v = pow((double)xc, alpha) / pow((double)wc, 1.0 - alpha);
        float r = (float)v; /* one rounding, to nearest even */
        s[j] = r > 1e-5f ? r : 1e-5f;
    }
}

/* ------------------------------------------------------------------ weight fold
 * W' = S W: input channel j of the weight times s_j. With W stored [N,K]
 * that is column k of every row.  [SQ-p2] SmoothQuant 的原理; [SQ-p4] §3
 * (weight.mul_(s.view(1,-1)) on [out, in]).  Pinned by: the fp64 identity
 * (X S^-1)(S W) = X W (exact products) and, with round_f32, by the fact that
 * an fp64 product of two fp32 values is exact so its fp32 rounding is the
 * fp32 product. */
void or_fold_weight(const double* W, int64_t N, int64_t K, const double* s,
                    int round_f32, double* Wp) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double p = W[n * K + k] * s[k];
            Wp[n * K + k] = round_f32 ? (double)(float)p : p;
        }
}

/* gamma'_j = gamma_j / s_j, beta'_j = beta_j / s_j   [SQ-p2] 融入 LayerNorm.
 * Pinned by: the fp64 identity norm(h; gamma', beta') = norm(h; gamma, beta)/s. */
void or_fold_norm(const double* gamma, const double* beta, const double* s, int64_t K,
                  int round_f32, double* gamma_out, double* beta_out) {
    for (int64_t j = 0; j < K; ++j) {
        double g = gamma[j] / s[j];
        gamma_out[j] = round_f32 ? (double)((float)gamma[j] / (float)s[j]) : g;
        if (beta && beta_out) {
            double b = beta[j] / s[j];
            beta_out[j] = round_f32 ? (double)((float)beta[j] / (float)s[j]) : b;
        }
    }
}

/* ------------------------------------------------------------------ fold into the previous linear
 * Fold 1/s into the previous linear layer   [SQ-p2] 融入前序线性层的权重 and
 * the table after it (down_proj: up_proj's output channels; o_proj: v_proj's
 * output channels): output channel j of the previous layer (row j of W [N,K],
 * and bias_j) is divided by s_j, so its output, the next layer's input
 * channel j, arrives divided by s_j; the next layer's weight takes s_j on its
 * input channel j (or_fold_weight).  round_f32: one fp32 division per value
 * (an fp64 quotient of two fp32 values rounded once to fp32 is the fp32
 * quotient).  Pinned by: the fp64 identity down(act(gate) * up) unchanged
 * under (up / s, down * s), with a negative control folding the wrong axis. */
void or_fold_prev_linear(const double* W, int64_t N, int64_t K, const double* bias, const double* s,
                         int round_f32, double* Wp, double* bias_out) {
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double q = W[n * K + k] / s[n];
            Wp[n * K + k] = round_f32 ? (double)((float)W[n * K + k] / (float)s[n]) : q;
        }
        if (bias && bias_out) {
            double b = bias[n] / s[n];
            bias_out[n] = round_f32 ? (double)((float)bias[n] / (float)s[n]) : b;
        }
    }
}

/* ------------------------------------------------------------------ MLP activation + int8
 * The input of down_proj (FC2) is act(gate_proj(x)) * up_proj(x) ([SQ-p2]
 * 融入前序线性层的权重), or relu(fc1(x)) for a ReLU MLP; with 1/s folded into
 * up_proj's (fc1's) output channels it arrives already smoothed, and is
 * quantised to int8 like any activation ([SQ-p5] §2.1).
 *
 * The pages name the activation but no way to evaluate it. Reading R9: SiLU,
 * silu(g) = g / (1 + exp(-g)), with exp evaluated by a fixed sequence of fp32
 * operations (Cody-Waite reduction x = n ln2 + r with ln 2 in two parts, and
 * the Taylor polynomial of exp(r) to degree 7 by Horner's rule), the same
 * sequence the CUDA kernel evaluates, so h and the codes it decides agree bit
 * for bit. Pinned by: exp within 4 ulp of the fp64 exp on a dense grid;
 * silu(g) - silu(-g) = g; the fp64 identity of the fold. */
#define OR_LOG2E 0x1.715476p+0f   /* log2(e) rounded to fp32 */
#define OR_LN2_HI 0x1.62e000p-1f  /* 2839/4096: ln 2 to 12 bits, so n*LN2_HI is exact */
#define OR_LN2_LO 0x1.0bfbe8p-15f /* ln 2 - LN2_HI, rounded to fp32 */

float or_expf(float x) {
    if (x > 88.0f) return (float)INFINITY;
    if (x < -87.0f) return 0.0f;
    const float n = rintf(x * OR_LOG2E); /* in [-126, 127] */
    float r = fmaf(-n, OR_LN2_HI, x);
    r = fmaf(-n, OR_LN2_LO, r);
    /* 1/k! for k = 7 .. 0 */
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    union { uint32_t u; float f; } two_n;
    two_n.u = (uint32_t)((int)n + 127) << 23;
    return p * two_n.f;
}

float or_silu(float g) { return g / (1.0f + or_expf(-g)); }

/* GELU, the tanh form 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3),
 * that GPT-class MLPs use. Reading R15: the pages name GELU beside SwiGLU for
 * the activation in front of FC2 but give no formula or evaluation; the tanh
 * form is evaluated as a fixed fp32 sequence on the exp above, written as
 * x / (1 + exp(-2u)) (the same function, since 1 + tanh(u) = 2 / (1 +
 * exp(-2u)), without the cancellation of 1 + tanh for negative x), one
 * rounding per step (fmaf for the inner polynomial). Pinned by: a library
 * GELU (tanh form, fp64) within a small relative bound, gelu(x) - gelu(-x) =
 * x to rounding, gelu(0) = 0, the limits x and 0, and the codes it decides
 * against those of the fp64 GELU away from ties. */
float or_gelu(float x) {
    const float c = 0.7978845608028654f; /* sqrt(2/pi), rounded to fp32 */
    const float k = 0.044715f;           /* rounded to fp32 */
    const float x3 = (x * x) * x;
    const float u = c * fmaf(k, x3, x);
    return x / (1.0f + or_expf(-2.0f * u));
}
void or_gelu_array(const float* x, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_gelu(x[i]);
}

void or_expf_array(const float* x, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_expf(x[i]);
}
void or_silu_array(const float* x, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_silu(x[i]);
}

void or_act_quant(const float* A, int64_t M, int64_t I, int64_t ld, int act, int per_token,
                  const float* static_qs, int8_t* Xq, float* qs_x, float* absmax_io, float* H) {
    float* h = (float*)malloc(sizeof(float) * (size_t)(I > 0 ? I : 1));
    for (int64_t i = 0; i < M; ++i) {
        const float* a = A + i * ld;
        float m = 0.0f;
        for (int64_t j = 0; j < I; ++j) {
            float v;
            if (act == 0) v = or_silu(a[j]) * a[I + j]; /* gate | up halves of the row */
            else if (act == 2) v = or_gelu(a[j]);
            else v = a[j] > 0.0f ? a[j] : 0.0f;
            h[j] = v;
            const float av = absf(v);
            if (av > m) m = av;
            if (absmax_io && av > absmax_io[j]) absmax_io[j] = av;
            if (H) H[i * I + j] = v;
        }
        if (!Xq) continue;
        float qs;
        if (per_token) {
            qs = scale_of(m);
            qs_x[i] = qs;
        } else {
            qs = *static_qs;
            if (i == 0) qs_x[0] = qs;
        }
        for (int64_t j = 0; j < I; ++j) Xq[i * I + j] = q_clip(h[j] * qs);
    }
    free(h);
}

/* ------------------------------------------------------------------ FP8 variant
 * The same W8A8 path on FP8 units   [SQ-p3] 技術原理與特性 (the smoothed
 * model can run on INT8 or FP8 compute units). The pages give no FP8
 * details. Reading R11: the format is OCP FP8 E4M3 (1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; largest finite value 448, subnormals
 * spaced 2^-9, no infinities); the absmax rule of [SQ-p5] §2.1 keeps its form
 * with the format's largest value: qs = 448 / max(m, 1e-8); q = the E4M3
 * value nearest to fl32(v * qs), ties to the even mantissa, magnitudes past
 * 448 saturated to 448; the GEMM accumulates the exact products; the
 * dequantisation divides by qs_x * qs_w as for int8.  Pinned by: every one of
 * the 254 finite codes decodes and re-encodes to itself; midpoints between
 * neighbours go to the even code; torch's float8_e4m3fn conversion agrees
 * inside the finite range; the GEMM by brute force. */
float or_e4m3_round(float x) {
    const double a = fabs((double)x);
    if (a >= 448.0) return x < 0 ? -448.0f : 448.0f;
    if (a == 0.0) return x;
    int e;
    frexp(a, &e); /* a in [2^(e-1), 2^e) */
    int ex = e - 1;
    if (ex < -6) ex = -6; /* below the smallest normal: the spacing stays 2^-9 */
    const double q = ldexp(1.0, ex - 3);
    double v = nearbyint(a / q) * q; /* a / q is exact; ties to even */
    if (v > 448.0) v = 448.0;
    return (float)(x < 0 ? -v : v);
}

/* bits of an E4M3 value (already representable); the sign bit is kept for a
 * zero too: a negative value that rounds to zero is -0 (0x80) */
uint8_t or_e4m3_bits(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int ex = e - 1;
    if (ex < -6) return (uint8_t)(sign | (int)(a / ldexp(1.0, -9))); /* subnormal: E = 0 */
    const int m = (int)((a / ldexp(1.0, ex) - 1.0) * 8.0);
    return (uint8_t)(sign | ((ex + 7) << 3) | m);
}

double or_e4m3_value(uint8_t b) {
    const int E = (b >> 3) & 15, m = b & 7;
    const double mag = E == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);
    return (b & 0x80) ? -mag : mag;
}

static float scale_fp8(float m) {
    float d = m > 1e-8f ? m : 1e-8f;
    return 448.0f / d;
}

/* FP8 quantisation of rows: v = fp32(X) (optionally * s_k or / s_k as in
 * the int8 weight / activation paths), then per row or one static scale. */
void or_quantize_fp8(const float* X, int64_t M, int64_t K, int64_t ld, const float* s, int s_div,
                     int per_row, const float* static_qs, uint8_t* Q, float* qs) {
    float* v = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float gmax = 0.0f;
    if (!per_row && !static_qs) {
        for (int64_t i = 0; i < M; ++i)
            for (int64_t j = 0; j < K; ++j) {
                float x = X[i * ld + j];
                if (s) x = s_div ? x / s[j] : x * s[j];
                if (absf(x) > gmax) gmax = absf(x);
            }
    }
    for (int64_t i = 0; i < M; ++i) {
        float m = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            float x = X[i * ld + j];
            if (s) x = s_div ? x / s[j] : x * s[j];
            v[j] = x;
            if (absf(x) > m) m = absf(x);
        }
        float q;
        if (per_row) {
            q = scale_fp8(m);
            qs[i] = q;
        } else {
            q = static_qs ? *static_qs : scale_fp8(gmax);
            qs[0] = q;
        }
        for (int64_t j = 0; j < K; ++j) Q[i * K + j] = or_e4m3_bits(or_e4m3_round(v[j] * q));
    }
    free(v);
}

/* acc[i - r0, j] = sum_k A[i,k] * B[j,k] of E4M3 codes, in fp64 (each product
 * is exact; the sum is exact to fp64 rounding). */
void or_gemm_fp8(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t r0, int64_t r1,
                 double* acc) {
    (void)M;
    for (int64_t i = r0; i < r1; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double t = 0.0;
            for (int64_t k = 0; k < K; ++k) t += or_e4m3_value(A[i * K + k]) * or_e4m3_value(B[j * K + k]);
            acc[(i - r0) * N + j] = t;
        }
}

/* y = acc / (qs_x[i or 0] * qs_w[j or 0]) (+ bias_j) in fp64 for an fp64
 * accumulator (the FP8 GEMM's exact sums). */
void or_dequant_f64(const double* acc, int64_t r0, int64_t r1, int64_t N, const float* qs_x, int x_per_token,
                    const float* qs_w, int w_per_channel, const float* bias, double* y) {
    for (int64_t i = r0; i < r1; ++i)
        for (int64_t j = 0; j < N; ++j) {
            const double d = (double)qs_x[x_per_token ? i : 0] * (double)qs_w[w_per_channel ? j : 0];
            double v = acc[(i - r0) * N + j] / d;
            if (bias) v += (double)bias[j];
            y[(i - r0) * N + j] = v;
        }
}

/* ------------------------------------------------------------------ weight quantisation
 * Weight int8, per output channel (row) or per tensor   [SQ-p2]
 * 为什么激活不能用逐通道量化 (weight scales per output channel factor out);
 * [SQ-p5] §2.1.  Pinned by: per-channel invariance under a power-of-two
 * channel scaling ([SQ-p2] 缩放的代价) and round-half-even ties. */
void or_quantize_weight(const float* Wp, int64_t N, int64_t K, int per_channel,
                        int8_t* Wq, float* qs_w) {
    if (per_channel) {
        for (int64_t n = 0; n < N; ++n) {
            float m = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float a = absf(Wp[n * K + k]);
                if (a > m) m = a;
            }
            float qs = scale_of(m);
            qs_w[n] = qs;
            for (int64_t k = 0; k < K; ++k) Wq[n * K + k] = q_clip(Wp[n * K + k] * qs);
        }
    } else {
        float m = 0.0f;
        for (int64_t i = 0; i < N * K; ++i) {
            float a = absf(Wp[i]);
            if (a > m) m = a;
        }
        float qs = scale_of(m);
        qs_w[0] = qs;
        for (int64_t i = 0; i < N * K; ++i) Wq[i] = q_clip(Wp[i] * qs);
    }
}

/* ------------------------------------------------------------------ activation quantisation without a norm
 * X' = X / s (explicit divide, [SQ-p4] §3 and §4, [SQ-p1] §3.3), then int8
 * per token or per tensor ([SQ-p5] §2.1).  Pinned by: the worked example of
 * [SQ-p2] 缩放的效果 (q = 1 before smoothing, q = 7 after). */
void or_quantize_act(const float* X, int64_t M, int64_t K, int64_t ld, const float* s,
                     int gran, const float* static_qs, int8_t* Xq, float* qs_x) {
    float* v = (float*)malloc(sizeof(float) * (size_t)(M * K > 0 ? M * K : 1));
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j) {
            float x = X[i * ld + j];
            v[i * K + j] = s ? x / s[j] : x;
        }
    if (gran == 1) {
        for (int64_t i = 0; i < M; ++i) {
            float m = 0.0f;
            for (int64_t j = 0; j < K; ++j) {
                float a = absf(v[i * K + j]);
                if (a > m) m = a;
            }
            float qs = scale_of(m);
            qs_x[i] = qs;
            for (int64_t j = 0; j < K; ++j) Xq[i * K + j] = q_clip(v[i * K + j] * qs);
        }
    } else {
        float qs;
        if (static_qs) {
            qs = *static_qs;
        } else {
            float m = 0.0f;
            for (int64_t i = 0; i < M * K; ++i) {
                float a = absf(v[i]);
                if (a > m) m = a;
            }
            qs = scale_of(m);
        }
        qs_x[0] = qs;
        for (int64_t i = 0; i < M * K; ++i) Xq[i] = q_clip(v[i] * qs);
    }
    free(v);
}

float or_scale_from_absmax(const float* absmax, int64_t n) {
    float m = 0.0f;
    for (int64_t j = 0; j < n; ++j)
        if (absmax[j] > m) m = absmax[j];
    return scale_of(m);
}

/* ------------------------------------------------------------------ fused norm + smoothing + int8
 * Fixed reduction order of the fp32 normalisation sums (reading R5; the pages
 * give the formula, not an order). With 256 lanes and chunks of 8 consecutive
 * elements:
 *   lane t folds chunks t, t+256, t+512, ... in increasing order; inside a
 *   chunk it folds elements in index order with acc = fma(a_j, b_j, acc);
 *   each group of 32 lanes is combined by the butterfly p[i] += p[i ^ off]
 *   for off = 16, 8, 4, 2, 1 (every lane ends with the same value);
 *   the eight group totals combine as ((G0+G1)+(G2+G3)) + ((G4+G5)+(G6+G7)).
 * The GPU kernels reduce in exactly this order, so sums, and with them every
 * int8 code, are bit-identical. Parity of the exact fp32 bits is pinned only by
 * this convention ("parity unpinned" for the bits themselves); the value is
 * pinned to the fp64 normalisation to 1e-6 relative. */
#define OR_LANES 256
#define OR_GROUPS (OR_LANES / 32)
#define OR_CHUNK 8
static float canon_dot(const float* a, const float* b, int64_t K) {
    float p[OR_LANES];
    int64_t nchunks = K / OR_CHUNK;
    for (int t = 0; t < OR_LANES; ++t) {
        float acc = 0.0f;
        for (int64_t c = t; c < nchunks; c += OR_LANES)
            for (int e = 0; e < OR_CHUNK; ++e) {
                int64_t j = c * OR_CHUNK + e;
                acc = fmaf(a[j], b ? b[j] : 1.0f, acc);
            }
        p[t] = acc;
    }
    float g[OR_GROUPS];
    for (int w = 0; w < OR_GROUPS; ++w) {
        float q[32], nq[32];
        for (int i = 0; i < 32; ++i) q[i] = p[32 * w + i];
        for (int off = 16; off >= 1; off >>= 1) {
            for (int i = 0; i < 32; ++i) nq[i] = q[i] + q[i ^ off];
            memcpy(q, nq, sizeof(q));
        }
        g[w] = q[0];
    }
    return ((g[0] + g[1]) + (g[2] + g[3])) + ((g[4] + g[5]) + (g[6] + g[7]));
}

/* LayerNorm / RMSNorm with the folded gamma' (and beta'), fused with int8
 * quantisation   [SQ-p2] 融入 LayerNorm (y_j = (x_j - mu)/sigma * gamma_j +
 * beta_j; the page names RMSNorm but prints the LayerNorm form, so both are
 * provided: RMSNorm has no mean and no beta); [SQ-p5] §2.1 for the int8 step.
 *   LayerNorm: mu = S(x)/K; d = x - mu; var = S(d*d)/K (biased);
 *              r = 1/sqrt(var + eps); v = (d * r) * gamma' + beta'
 *   RMSNorm:   ms = S(x*x)/K; r = 1/sqrt(ms + eps); v = (x * r) * gamma'
 * Every operation is one fp32 rounding (no contraction). */
void or_norm_smooth_quant(const float* H, int64_t M, int64_t K, int64_t ld, int norm,
                          const float* gamma, const float* beta, float eps,
                          int gran, const float* static_qs,
                          int8_t* Xq, float* qs_x, float* absmax_io, float* V) {
    float* d = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float* v = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float Kf = (float)K;
    for (int64_t i = 0; i < M; ++i) {
        const float* x = H + i * ld;
        float r;
        if (norm == 0) {
            float mu = canon_dot(x, NULL, K) / Kf;
            for (int64_t j = 0; j < K; ++j) d[j] = x[j] - mu;
            float var = canon_dot(d, d, K) / Kf;
            r = 1.0f / sqrtf(var + eps);
            for (int64_t j = 0; j < K; ++j) {
                float t = (d[j] * r) * gamma[j];
                v[j] = beta ? t + beta[j] : t;
            }
        } else {
            float ms = canon_dot(x, x, K) / Kf;
            r = 1.0f / sqrtf(ms + eps);
            for (int64_t j = 0; j < K; ++j) v[j] = (x[j] * r) * gamma[j];
        }
        if (V)
            for (int64_t j = 0; j < K; ++j) V[i * K + j] = v[j];
        if (absmax_io)
            for (int64_t j = 0; j < K; ++j) {
                float a = absf(v[j]);
                if (a > absmax_io[j]) absmax_io[j] = a;
            }
        if (Xq) {
            float qs;
            if (gran == 1) {
                float m = 0.0f;
                for (int64_t j = 0; j < K; ++j) {
                    float a = absf(v[j]);
                    if (a > m) m = a;
                }
                qs = scale_of(m);
                qs_x[i] = qs;
            } else {
                qs = *static_qs;
                if (i == 0) qs_x[0] = qs;
            }
            for (int64_t j = 0; j < K; ++j) Xq[i * K + j] = q_clip(v[j] * qs);
        }
    }
    free(d);
    free(v);
}

void or_norm_f64(const double* H, int64_t M, int64_t K, int norm, const double* gamma,
                 const double* beta, double eps, double* V) {
    for (int64_t i = 0; i < M; ++i) {
        const double* x = H + i * K;
        if (norm == 0) {
            double mu = 0.0;
            for (int64_t j = 0; j < K; ++j) mu += x[j];
            mu /= (double)K;
            double var = 0.0;
            for (int64_t j = 0; j < K; ++j) var += (x[j] - mu) * (x[j] - mu);
            var /= (double)K;
            double r = 1.0 / sqrt(var + eps);
            for (int64_t j = 0; j < K; ++j)
                V[i * K + j] = (x[j] - mu) * r * gamma[j] + (beta ? beta[j] : 0.0);
        } else {
            double ms = 0.0;
            for (int64_t j = 0; j < K; ++j) ms += x[j] * x[j];
            ms /= (double)K;
            double r = 1.0 / sqrt(ms + eps);
            for (int64_t j = 0; j < K; ++j) V[i * K + j] = x[j] * r * gamma[j];
        }
    }
}

/* ------------------------------------------------------------------ int8 GEMM
 * int8 x int8 -> integer accumulation   [SQ-p5] §2.1 (int32 accumulation);
 * [SQ-p2] 为什么激活不能用逐通道量化 (Y = diag(dX) Xq Wq diag(dW)).
 * Accumulated in int64 so that a sum beyond int32 would show; the test asserts
 * it fits int32.  Pinned by: brute force against an independent integer
 * product on small shapes, exhaustive K <= 3 sweeps, and the all-127 bound. */
void or_gemm_i8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                int64_t r0, int64_t r1, int64_t* acc) {
    (void)M;
    for (int64_t i = r0; i < r1; ++i)
        for (int64_t j = 0; j < N; ++j) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k) a += (int64_t)Xq[i * K + k] * (int64_t)Wq[j * K + k];
            acc[(i - r0) * N + j] = a;
        }
}

/* Dequantisation by the outer product of the scales   [SQ-p5] §2.1
 * (out_i32 / (cx * cw)), plus the bias. Reading R4: fp64, one rounding to the
 * output type afterwards (the page's fp16 division would overflow). */
void or_dequant(const int64_t* acc, int64_t r0, int64_t r1, int64_t N,
                const float* qs_x, int per_token, const float* qs_w, int per_channel,
                const double* bias, double* y) {
    for (int64_t i = r0; i < r1; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double cx = per_token ? (double)qs_x[i] : (double)qs_x[0];
            double cw = per_channel ? (double)qs_w[j] : (double)qs_w[0];
            double v = (double)acc[(i - r0) * N + j] / (cx * cw);
            if (bias) v += bias[j];
            y[(i - r0) * N + j] = v;
        }
}

/* Round to the nearest value with `sig` significant bits, normal exponent
 * range starting at 2^emin, ties to even; inf beyond 2^(emax+1). */
static double round_to_format(double y, int sig, int emin, int emax) {
    if (y != y) return y;
    double a = absd(y);
    if (a == 0.0) return y;
    int ex;
    frexp(a, &ex);   /* a = m * 2^ex, m in [0.5, 1) */
    int E = ex - 1;  /* a in [2^E, 2^(E+1)) */
    if (E < emin) E = emin;
    double quantum = ldexp(1.0, E - (sig - 1));
    double r = nearbyint(a / quantum) * quantum; /* exact scaling by 2^n */
    if (r >= ldexp(1.0, emax + 1)) r = INFINITY;
    return y < 0 ? -r : r;
}

uint16_t or_round_bf16(double y) {
    if (y != y) return 0x7fc0;
    double r = round_to_format(y, 8, -126, 127);
    float f = (float)r; /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

uint16_t or_round_fp16(double y) {
    if (y != y) return 0x7e00;
    double r = round_to_format(y, 11, -14, 15);
    uint16_t sign = signbit(r) ? 0x8000 : 0;
    double a = absd(r);
    if (isinf(a)) return sign | 0x7c00;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) return sign | (uint16_t)(a / ldexp(1.0, -24));
    int ex;
    frexp(a, &ex);
    int E = ex - 1;
    uint16_t mant = (uint16_t)(a / ldexp(1.0, E - 10) - 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

void or_round_bf16_array(const double* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_round_bf16(y[i]);
}

void or_round_fp16_array(const double* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_round_fp16(y[i]);
}

/* ------------------------------------------------------------------ LLM.int8() decomposition
 * Outlier dimensions   [SQ-p5] §2.2 split_outliers (over = |x| > alpha;
 * ratio = over.mean(axis=0); keep ratio > min_ratio), §4.1 (any value over
 * the threshold marks the dimension). Reading R6: the garbled comparison is
 * ">", and min_ratio = 0 by default.  Pinned by: brute force on small inputs
 * and planted outlier sets. */
int64_t or_llmint8_outliers(const float* X, int64_t M, int64_t K, int64_t ld, float thr,
                            double min_ratio, int32_t* idx) {
    int64_t n = 0;
    for (int64_t j = 0; j < K; ++j) {
        int64_t count = 0;
        for (int64_t i = 0; i < M; ++i)
            if (absf(X[i * ld + j]) > thr) ++count;
        double ratio = M > 0 ? (double)count / (double)M : 0.0;
        if (ratio > min_ratio) idx[n++] = (int32_t)j;
    }
    return n;
}

static int in_set(const int32_t* idx, int64_t n, int64_t j) {
    for (int64_t o = 0; o < n; ++o)
        if (idx[o] == j) return 1;
    return 0;
}

/* Vector-wise row quantisation of the non-outlier columns   [SQ-p5]
 * §2.1 quantize_vectorwise(x, axis=1) applied to x[:, mask] (§2.2). */
void or_llmint8_quant_rows(const float* X, int64_t M, int64_t K, int64_t ld,
                           const int32_t* idx, int64_t n_idx, int8_t* Xq, float* qs_x) {
    char* out = (char*)calloc((size_t)(K > 0 ? K : 1), 1);
    for (int64_t o = 0; o < n_idx; ++o) out[idx[o]] = 1;
    for (int64_t i = 0; i < M; ++i) {
        float m = 0.0f;
        for (int64_t j = 0; j < K; ++j)
            if (!out[j]) {
                float a = absf(X[i * ld + j]);
                if (a > m) m = a;
            }
        float qs = scale_of(m);
        qs_x[i] = qs;
        for (int64_t j = 0; j < K; ++j) Xq[i * K + j] = out[j] ? 0 : q_clip(X[i * ld + j] * qs);
    }
    free(out);
}

/* Weight side: quantize_vectorwise(w[mask, :], axis=0) of [SQ-p5] §2.2;
 * their W is [K, N], so axis 0 gives one scale per output channel. */
void or_llmint8_quant_weight(const float* W, int64_t N, int64_t K,
                             const int32_t* idx, int64_t n_idx, int8_t* Wq, float* qs_w) {
    char* out = (char*)calloc((size_t)(K > 0 ? K : 1), 1);
    for (int64_t o = 0; o < n_idx; ++o) out[idx[o]] = 1;
    for (int64_t n = 0; n < N; ++n) {
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (!out[k]) {
                float a = absf(W[n * K + k]);
                if (a > m) m = a;
            }
        float qs = scale_of(m);
        qs_w[n] = qs;
        for (int64_t k = 0; k < K; ++k) Wq[n * K + k] = out[k] ? 0 : q_clip(W[n * K + k] * qs);
    }
    free(out);
}

/* The two paths summed   [SQ-p5] §2.2 mixed_precision_matmul. */
void or_llmint8_combine(const int64_t* acc, int64_t r0, int64_t r1, int64_t N, int64_t K,
                        const float* qs_x, const float* qs_w, const float* X, int64_t ldx,
                        const float* W, const int32_t* idx, int64_t n_idx, double* y) {
    for (int64_t i = r0; i < r1; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double v = (double)acc[(i - r0) * N + j] / ((double)qs_x[i] * (double)qs_w[j]);
            double h = 0.0;
            for (int64_t o = 0; o < n_idx; ++o)
                h += (double)X[i * ldx + idx[o]] * (double)W[j * K + idx[o]];
            y[(i - r0) * N + j] = v + h;
        }
}

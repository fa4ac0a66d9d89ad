/*
 * CPU oracle for the SmoothQuant W8A8 linear-layer path and the LLM.int8()
 * mixed-precision decomposition.
 *
 * TEST INFRASTRUCTURE ONLY. This library exists so that tests, the smoke
 * check and the CPU baseline leg of the benchmark have an independent,
 * obviously-correct statement of what the GPU path computes. The product
 * path never links, loads or calls it. It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Conventions
 *   - Activations X are [M,K] row-major (tokens x input channels), given as
 *     fp32 arrays. A 16-bit tensor converts to fp32 exactly, so the caller
 *     passes the fp32 image of fp16/bf16 data.
 *   - Weights are stored [N,K] (output channel x input channel), the layout
 *     of a torch nn.Linear weight. The pages' W[K,N] (d_in x d_out) is the
 *     transpose; w_j = max over row j of their W = max over column j here.
 *   - Exact results are computed in fp64 or int64. Steps whose result is an
 *     integer (a quantised code) are taken in fp32, the precision of the
 *     GPU kernels, with correctly rounded operations only.
 *
 * Parity status of each function is written beside it: "pinned by ..." or
 * "parity unpinned" with the reason.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Column absmax, running: io[j] = max(io[j], max_i |X[i*ld + j]|). */
void or_col_absmax(const float* X, int64_t M, int64_t K, int64_t ld, float* io);

/* s_j from x_j, w_j and alpha; fp64 arithmetic, one rounding to fp32. */
void or_smooth_scales(const float* x, const float* w, int64_t K, double alpha, float* s);

/* W'[n,k] = W[n,k] * s[k]. round_f32 != 0 rounds each product to fp32
 * (the library's fold); 0 keeps the exact fp64 product. */
void or_fold_weight(const double* W, int64_t N, int64_t K, const double* s,
                    int round_f32, double* Wp);

/* gamma' = gamma / s, beta' = beta / s (beta may be NULL). Same rounding
 * switch as or_fold_weight. */
void or_fold_prev_linear(const double* W, int64_t N, int64_t K, const double* bias, const double* s,
                         int round_f32, double* Wp, double* bias_out);
float or_e4m3_round(float x);
uint8_t or_e4m3_bits(float v);
double or_e4m3_value(uint8_t b);
void or_quantize_fp8(const float* X, int64_t M, int64_t K, int64_t ld, const float* s, int s_div,
                     int per_row, const float* static_qs, uint8_t* Q, float* qs);
void or_gemm_fp8(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t r0, int64_t r1,
                 double* acc);
void or_dequant_f64(const double* acc, int64_t r0, int64_t r1, int64_t N, const float* qs_x, int x_per_token,
                    const float* qs_w, int w_per_channel, const float* bias, double* y);
float or_expf(float x);
float or_silu(float g);
float or_gelu(float x);
void or_gelu_array(const float* x, int64_t n, float* out);
void or_expf_array(const float* x, int64_t n, float* out);
void or_silu_array(const float* x, int64_t n, float* out);
void or_act_quant(const float* A, int64_t M, int64_t I, int64_t ld, int act, int per_token,
                  const float* static_qs, int8_t* Xq, float* qs_x, float* absmax_io, float* H);
void or_fold_norm(const double* gamma, const double* beta, const double* s, int64_t K,
                  int round_f32, double* gamma_out, double* beta_out);

/* Symmetric absmax int8 quantisation of a fp32 weight [N,K].
 * per_channel != 0: one scale per output channel (row); else one scale. */
void or_quantize_weight(const float* Wp, int64_t N, int64_t K, int per_channel,
                        int8_t* Wq, float* qs_w);

/* v = x / s_j (s may be NULL: v = x), then int8 quantisation.
 * gran: 1 = per token (row), 0 = per tensor. For per tensor, static_qs
 * (may be NULL) gives the scale; NULL means the tensor's own absmax. */
void or_quantize_act(const float* X, int64_t M, int64_t K, int64_t ld, const float* s,
                     int gran, const float* static_qs, int8_t* Xq, float* qs_x);

/* qs = 127 / max(max_j absmax[j], 1e-8) in fp32. */
float or_scale_from_absmax(const float* absmax, int64_t n);

/* LayerNorm (norm=0) or RMSNorm (norm=1) with folded gamma'/beta', fused
 * with int8 quantisation. Xq and qs_x may be NULL (no quantisation);
 * absmax_io (may be NULL) receives the running per-channel max |v|;
 * V (may be NULL) receives v in fp32. beta is ignored for RMSNorm. */
void or_norm_smooth_quant(const float* H, int64_t M, int64_t K, int64_t ld, int norm,
                          const float* gamma, const float* beta, float eps,
                          int gran, const float* static_qs,
                          int8_t* Xq, float* qs_x, float* absmax_io, float* V);

/* The same normalisation computed in fp64 without any intermediate
 * rounding; used to pin the fp32 path and the fold identity. */
void or_norm_f64(const double* H, int64_t M, int64_t K, int norm, const double* gamma,
                 const double* beta, double eps, double* V);

/* acc[i,j] = sum_k Xq[i,k] * Wq[j,k] in int64, rows [r0, r1) of X only. */
void or_gemm_i8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                int64_t r0, int64_t r1, int64_t* acc);

/* y = acc / (qs_x[i] * qs_w[j]) + bias[j] in fp64. per_token/per_channel
 * select vector or scalar scales; bias may be NULL. acc rows [r0, r1). */
void or_dequant(const int64_t* acc, int64_t r0, int64_t r1, int64_t N,
                const float* qs_x, int per_token, const float* qs_w, int per_channel,
                const double* bias, double* y);

/* Round fp64 to the nearest bf16 / fp16 (ties to even); returns the bits. */
uint16_t or_round_bf16(double y);
uint16_t or_round_fp16(double y);
void or_round_bf16_array(const double* y, int64_t n, uint16_t* out);
void or_round_fp16_array(const double* y, int64_t n, uint16_t* out);

/* LLM.int8 outlier set: columns j with count_i(|X_ij| > thr) / M > min_ratio,
 * ascending. Returns |O|. */
int64_t or_llmint8_outliers(const float* X, int64_t M, int64_t K, int64_t ld, float thr,
                            double min_ratio, int32_t* idx);

/* Vector-wise row quantisation of X over the columns not in O; columns in
 * O are set to 0 in Xq. */
void or_llmint8_quant_rows(const float* X, int64_t M, int64_t K, int64_t ld,
                           const int32_t* idx, int64_t n_idx, int8_t* Xq, float* qs_x);

/* Vector-wise quantisation of the weight over the input channels not in O:
 * one scale per output channel (row of [N,K]); columns in O set to 0. */
void or_llmint8_quant_weight(const float* W, int64_t N, int64_t K,
                             const int32_t* idx, int64_t n_idx, int8_t* Wq, float* qs_w);

/* y = acc/(qs_x qs_w) + sum_{o in O, ascending} X[i,o] W[j,o] in fp64,
 * rows [r0, r1). acc holds the int8 path over the same rows. */
void or_llmint8_combine(const int64_t* acc, int64_t r0, int64_t r1, int64_t N, int64_t K,
                        const float* qs_x, const float* qs_w, const float* X, int64_t ldx,
                        const float* W, const int32_t* idx, int64_t n_idx, double* y);

#ifdef __cplusplus
}
#endif
#endif

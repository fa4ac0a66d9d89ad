/*
 * sq_api.h — C ABI of the SmoothQuant W8A8 linear-layer library for NVIDIA
 * B200 (sm_100a), plus the LLM.int8() mixed-precision decomposition.
 *
 * Sources (page title, section) cited below:
 *   [SQ-p1] lpnh.cn SmoothQuant practice article (§2.1 scale formula, §3.2
 *           calibrate, §3.3 apply_smoothquant)
 *   [SQ-p2] "大语言模型量化技术（四）：SmoothQuant" (wangyu.me): sections
 *           为什么激活不能用逐通道量化, SmoothQuant 的原理, 缩放因子, 缩放的代价,
 *           缩放的效果, 融入 LayerNorm
 *   [SQ-p4] "如何通过 SmoothQuant 解决激活值离群点难题：实现端侧 LLM 全量化推理的关键"
 *           (tbr8.org) §3 smooth_layer_weights, §4 deployment notes
 *   [SQ-p5] "8位量化：异常值与混合精度分解实战" (xdnf.cn) §2.1 absmax and
 *           vector-wise quantisation, §2.2 mixed-precision decomposition,
 *           §2.3 threshold 6.0, §4.1 threshold semantics
 *
 * Conventions (all entry points)
 *   - Pointers are DEVICE pointers owned by the caller unless stated. The
 *     library never allocates device memory; where an operation needs scratch
 *     it takes a caller-provided `workspace` of at least sq_workspace_size()
 *     bytes, 256-byte aligned.
 *   - Matrices are row-major. Activations X are [M,K] (tokens x input
 *     channels) with row stride ldx elements. Weights are [N,K] (output x
 *     input channel, K contiguous), the torch nn.Linear layout; the pages'
 *     W[K,N] is its transpose. Outputs Y are [M,N] with row stride ldy.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *     never synchronises it, except sq_workspace_status().
 *   - Return value: SQ_OK, or an error code with no kernel launched and no
 *     output touched (argument errors), or SQ_ERR_CUDA if a launch failed.
 *     sq_last_error_string() (thread-local) describes the last error.
 *   - M == 0 (no rows) is valid and launches nothing. K == 0 and N == 0 are
 *     rejected with SQ_ERR_UNSUPPORTED_SHAPE.
 *   - Results are deterministic: the same inputs give bit-identical outputs
 *     on every call, whatever the launch order of the blocks.
 *   - The library is built for sm_100a only; calls on another device return
 *     SQ_ERR_CUDA ("no kernel image").
 */
#ifndef SQ_API_H
#define SQ_API_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sq_stream_t; /* a cudaStream_t */

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size */
    SQ_ERR_UNSUPPORTED_SHAPE = 2, /* size outside what the kernels handle  */
    SQ_ERR_ALIGNMENT = 3,         /* pointer or stride not 16-byte aligned */
    SQ_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed     */
    SQ_ERR_TIMEOUT = 5            /* a bounded device-side wait gave up    */
} sq_status_t;

typedef enum { SQ_F32 = 0, SQ_F16 = 1, SQ_BF16 = 2, SQ_I32 = 3, SQ_I8 = 4 } sq_dtype_t;

typedef enum { SQ_LAYERNORM = 0, SQ_RMSNORM = 1 } sq_norm_t;

/* MLP activation feeding down_proj / FC2 (sq_act_quant, sq_gemm_w8a8_act). */
typedef enum { SQ_ACT_SWIGLU = 0, SQ_ACT_RELU = 1, SQ_ACT_GELU = 2 } sq_act_t;

typedef enum {
    SQ_OP_GEMM = 0,           /* sq_gemm_w8a8                               */
    SQ_OP_QUANT_ACT = 1,      /* sq_quantize_act (per-tensor dynamic)       */
    SQ_OP_QUANT_WEIGHT = 2,   /* sq_quantize_weight (per-tensor)            */
    SQ_OP_LLMINT8_DETECT = 3, /* sq_llmint8_detect                          */
    SQ_OP_LLMINT8 = 4         /* sq_llmint8_matmul                          */
} sq_op_t;

/* Bytes of workspace an operation needs for the given sizes (0 if none is
 * needed; callers may still pass one). Never fails; unknown op -> 0. */
SQ_API size_t sq_workspace_size(sq_op_t op, int64_t M, int64_t N, int64_t K);

/* Description of the last error on this host thread ("" if none). */
SQ_API const char* sq_last_error_string(void);

/* Synchronises `stream`, reads the status word that bounded device waits
 * write into `workspace`, clears it and returns SQ_OK or SQ_ERR_TIMEOUT. On
 * SQ_ERR_TIMEOUT it also zeroes the stream-K counters of the last GEMM that
 * used them on this workspace (their size is recorded in the header), so the
 * workspace is ready for the next call without the caller zeroing it again.
 * Applies to workspaces passed to sq_gemm_w8a8, sq_gemm_fp8, sq_bmm_w8a8,
 * sq_llmint8_matmul and sq_selftest_wait_timeout. */
SQ_API sq_status_t sq_workspace_status(void* workspace, sq_stream_t stream);

/* Check of the failure path of the bounded device waits: launches one block
 * that waits on an mbarrier nothing completes, with the bounded wait every
 * waiting kernel of the library uses, but a timeout of timeout_ns (at most
 * 2 s) instead of 2 s. The block gives up, records the timeout code in the
 * workspace status word and returns: sq_workspace_status then returns
 * SQ_ERR_TIMEOUT and the context stays usable. Nothing faults, traps or
 * hangs. The pages have no counterpart; it exists to test the failure path. */
SQ_API sq_status_t sq_selftest_wait_timeout(void* workspace, size_t ws_bytes, uint64_t timeout_ns,
                                            sq_stream_t stream);

/* Library version as an integer (major*10000 + minor*100 + patch). */
SQ_API int sq_version(void);

/* --------------------------------------------------------------------------
 * Calibration absmax                            [SQ-p2] 缩放因子;
 *          [SQ-p1] §3.2 (act.abs().amax over tokens; weight.abs().amax(dim=0));
 *          [SQ-p4] §3 (max over batch and sequence; max over output dim).
 *
 * sq_calib_absmax:  xmax[j] = max(xmax[j], max_i |X[i,j]|)  over i < M.
 *   Running maximum across calls: call once per calibration batch after the
 *   caller has zero-filled xmax once. X: [M,K] of dtype dt in {F16, BF16,
 *   F32}, row stride ldx >= K. xmax: [K] fp32, read and written.
 * sq_weight_absmax: wmax[j] = max(wmax[j], max_n |W[n,j]|), W [N,K] (torch
 *   layout: the max runs over output channels). For an input shared by
 *   several linears (q/k/v, gate/up) call it on each, or on their
 *   concatenation; the result is one scale per input channel.
 * Requirements: X (W) 16-byte aligned; K and ldx multiples of 8 (16-bit)
 * or 4 (fp32). NaN inputs give an unspecified result. Inputs of 16 MB and
 * more stream through shared memory with bounded waits (about 2 s); a wait
 * that gives up (not expected: the copies read the caller's input) leaves NaN
 * in the maxima of the columns concerned, never a silently wrong value.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_calib_absmax(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                            float* xmax_inout, sq_stream_t stream);
SQ_API sq_status_t sq_weight_absmax(const void* W, sq_dtype_t dt, int64_t N, int64_t K, int64_t ldw,
                             float* wmax_inout, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * Smoothing factors                                [SQ-p2] 缩放因子;
 *     [SQ-p1] §2.1, §3.2; [SQ-p4] §3.
 *   s[j] = max(1e-5, x^alpha / w^(1-alpha)),  x = max(xmax[j], 1e-5),
 *   w = max(wmax[j], 1e-5), evaluated in fp64 and rounded once to fp32.
 *   alpha in [0, 1]; alpha = 0, 0.5, 1 use the closed forms 1/w, sqrt(x/w), x.
 *   Outside [0,1] -> SQ_ERR_INVALID_ARG. xmax, wmax, s: [K] fp32.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_smooth_scales(const float* xmax, const float* wmax, int64_t K, double alpha,
                             float* s_out, sq_stream_t stream);

/* Weight fold  W' = diag(s) W in the pages' notation: input channel k of every
 * output row times s[k]      [SQ-p2] SmoothQuant 的原理; [SQ-p4] §3
 * (weight.mul_(s.view(1,-1))).  W: [N,K] of dt in {F16, BF16, F32};
 * Wp_out: [N,K] fp32 (one fp32 rounding per product). K % 8 == 0. */
SQ_API sq_status_t sq_fold_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s,
                           float* Wp_out, sq_stream_t stream);

/* Fold into the norm  gamma' = gamma / s, beta' = beta / s  (fp32 IEEE
 * division)                  [SQ-p2] 融入 LayerNorm.
 * beta / beta_out may both be NULL (RMSNorm). All [K] fp32. In-place
 * (gamma_out == gamma) is allowed. */
SQ_API sq_status_t sq_fold_norm(const float* gamma, const float* beta, const float* s, int64_t K,
                         float* gamma_out, float* beta_out, sq_stream_t stream);

/* sq_smooth_scales and sq_fold_norm in one launch: s_out as sq_smooth_scales,
 * then gamma_out = gamma / s_out and beta_out = beta / s_out as sq_fold_norm
 * (the same operations, so the same bits as the two calls in sequence).
 * beta / beta_out may both be NULL. All [K] fp32; alpha in [0, 1]. */
SQ_API sq_status_t sq_smooth_fold_norm(const float* xmax, const float* wmax, int64_t K, double alpha,
                                       const float* gamma, const float* beta, float* s_out, float* gamma_out,
                                       float* beta_out, sq_stream_t stream);

/* Fold into the previous linear layer    [SQ-p2] 融入前序线性层的权重 and
 * the table after it: for down_proj the smoothing goes into up_proj's output
 * channels, for o_proj into v_proj's. Output channel n of the previous layer
 * is divided by s[n]: Wp[n,k] = fp32(W[n,k]) / s[n], bias_out[n] = bias[n] /
 * s[n] (fp32 IEEE division). The next layer's input channels then take s
 * with sq_fold_weight (or sq_quantize_weight with s). W: [N,K] of dt in
 * {F16, BF16, F32}; Wp_out: [N,K] fp32; s: [N]; bias / bias_out: [N] fp32,
 * both NULL or both given. K % 8 == 0. With grouped KV heads, one s per
 * v_proj output channel serves every query head that reads it. */
SQ_API sq_status_t sq_fold_prev_linear(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* bias,
                                const float* s, float* Wp_out, float* bias_out, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * Weight quantisation (offline)     [SQ-p5] §2.1; [SQ-p2]
 *     为什么激活不能用逐通道量化 (weight scales per output channel).
 *   W' = fp32(W) * s[k]  (s may be NULL: W' = fp32(W)), then
 *   m = max |W'| over the row (per_channel != 0) or the tensor;
 *   qs = 127 / max(m, 1e-8)  (fp32);  Wq = clip(rne(W' * qs), -127, 127).
 *   W: [N,K] of dt in {F16, BF16, F32}. Wq: [N,K] int8. qs_w: [N] or [1].
 *   Per-tensor needs workspace (SQ_OP_QUANT_WEIGHT). K % 16 == 0.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_quantize_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K,
                               const float* s, int per_channel, int8_t* Wq, float* qs_w,
                               void* workspace, size_t ws_bytes, sq_stream_t stream);

/* The fold into this layer's output channels and the int8 quantisation in one
 * pass     [SQ-p2] 融入前序线性层的权重 with the weight step above: a layer whose
 * output feeds a smoothed linear (up_proj before down_proj) takes 1/s_next on
 * its output channels, and its own input smoothing s:
 *   W'[n,k] = (W[n,k] / s_next[n]) * s[k]  (two fp32 roundings, the values
 *   sq_fold_prev_linear then sq_quantize_weight would give), then per output
 *   channel int8 as sq_quantize_weight with per_channel = 1.
 * s_next: [N] fp32; s: [K] fp32 (16-byte aligned). W: [N,K] of dt in {F16,
 * BF16, F32}. K % 16 == 0. */
SQ_API sq_status_t sq_quantize_weight_fold_prev(const void* W, sq_dtype_t dt, int64_t N, int64_t K,
                                                const float* s_next, const float* s, int8_t* Wq, float* qs_w,
                                                sq_stream_t stream);

/* --------------------------------------------------------------------------
 * Activation quantisation without a norm     [SQ-p4] §3 (input / s);
 *      [SQ-p1] §3.3; [SQ-p5] §2.1.
 *   v = fp32(X[i,j]) / s[j]  (IEEE division; s may be NULL: v = X),
 *   per_token != 0: qs_x[i] = 127 / max(max_j |v[i,j]|, 1e-8);
 *   per_token == 0: qs_x[0] = *static_qs if static_qs != NULL, else
 *                   127 / max(max_ij |v|, 1e-8) (needs workspace);
 *   Xq[i,j] = clip(rne(v * qs), -127, 127).
 *   X: [M,K] dt in {F16, BF16, F32}, stride ldx. Xq: [M,K] contiguous.
 *   K % 16 == 0.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_quantize_act(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                            const float* s, int per_token, const float* static_qs,
                            int8_t* Xq, float* qs_x, void* workspace, size_t ws_bytes,
                            sq_stream_t stream);

/* Static per-tensor scale from calibration maxima: qs = 127 / max(max_j
 * absmax[j], 1e-8), written to qs_out[0]. absmax: [n] fp32. */
SQ_API sq_status_t sq_scale_from_absmax(const float* absmax, int64_t n, float* qs_out,
                                 sq_stream_t stream);

/* --------------------------------------------------------------------------
 * Fused norm + smoothing + int8           [SQ-p2] 融入 LayerNorm;
 *     [SQ-p4] §4 item 2; [SQ-p5] §2.1.
 *   LayerNorm: mu = S(x)/K, d = x - mu, var = S(d*d)/K, r = 1/sqrt(var+eps),
 *              v = (d*r)*gamma' + beta'  (beta' may be NULL)
 *   RMSNorm:   r = 1/sqrt(S(x*x)/K + eps),  v = (x*r)*gamma'
 *   Every step is one correctly rounded fp32 operation. S() is a sum in a
 *   fixed order: 256 lanes; lane t folds 8-element chunks t, t+256, ... with
 *   fma in index order; each 32-lane group combines by the xor butterfly
 *   (16, 8, 4, 2, 1); the eight group totals add as
 *   ((G0+G1)+(G2+G3))+((G4+G5)+(G6+G7)).
 *   Then, if Xq != NULL: per_token != 0 -> qs_x[i] = 127/max(max_j|v|,1e-8);
 *   per_token == 0 -> qs = *static_qs (required), qs_x[0] = qs;
 *   Xq = clip(rne(v*qs), -127, 127).
 *   Optional outputs: absmax_inout [K] fp32 running max of |v| per channel
 *   (calibration mode); V_out [M,K] (stride K) v rounded to dt.
 *   gamma_p (and beta_p) are the folded parameters from sq_fold_norm, or the
 *   original ones to calibrate. H: [M,K] dt in {F16, BF16}, stride ldh.
 *   K % 8 == 0, 8 <= K <= 16384. For K > 4096 rows stream through shared
 *   memory with bounded waits (about 2 s); a wait that gives up (not
 *   expected) leaves NaN in the scales of the rows not finished (the static
 *   scale's copy in qs_x[0]) and in the calibration maxima.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_norm_smooth_quant(const void* H, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldh,
                                 sq_norm_t norm, const float* gamma_p, const float* beta_p,
                                 float eps, int per_token, const float* static_qs,
                                 int8_t* Xq, float* qs_x, float* absmax_inout, void* V_out,
                                 sq_stream_t stream);

/* --------------------------------------------------------------------------
 * MLP activation + int8 for the input of down_proj / FC2
 *     [SQ-p2] 融入前序线性层的权重 (down_proj input = act(gate) * up, its
 *     smoothing folded into up_proj by sq_fold_prev_linear); [SQ-p5] §2.1.
 *   SQ_ACT_SWIGLU: A is [M, 2I] (stride lda >= 2I), gate = A[:, :I],
 *     up = A[:, I:]; h = silu(gate) * up, silu(g) = g / (1 + exp(-g)).
 *   SQ_ACT_RELU: A is [M, I] (stride lda >= I); h = max(A, 0).
 *   SQ_ACT_GELU: A is [M, I]; h = gelu(A), the tanh form
 *     0.5 a (1 + tanh(u)), u = c (a + 0.044715 a^3), c = sqrt(2/pi), written
 *     a / (1 + exp(-2u)) (the same function) and evaluated as the fp32
 *     sequence x3 = (a*a)*a; u = c * fma(k, x3, a); h = a / (1 + exp(-2u))
 *     with c and k = 0.044715 rounded to fp32 and exp as below.
 *   exp is a fixed sequence of correctly rounded fp32 operations: n =
 *   rint(x * fp32(log2 e)), r = x - n*LN2_HI - n*LN2_LO (two fma, LN2_HI =
 *   2839/4096), exp(r) by the degree-7 Taylor polynomial in Horner form with
 *   fma, times 2^n; exp(x) = +inf above 88 and 0 below -87. The result is
 *   within 4 ulp of exp and is reproducible bit for bit on any IEEE machine.
 *   Then, if Xq != NULL: per_token != 0 -> qs_x[i] = 127/max(max_j|h|,1e-8);
 *   per_token == 0 -> qs = *static_qs (required), qs_x[0] = qs;
 *   Xq[i,j] = clip(rne(h*qs), -127, 127), Xq [M,I] contiguous.
 *   Optional: absmax_inout [I] fp32 running max of |h| (calibration; I <=
 *   57344), H_out [M,I] (stride I) h rounded to dt.
 *   dt in {F16, BF16}; I % 8 == 0, lda % 8 == 0; A, Xq, H_out 16-byte aligned.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_act_quant(const void* A, sq_dtype_t dt, int64_t M, int64_t I, int64_t lda, sq_act_t act,
                                int per_token, const float* static_qs, int8_t* Xq, float* qs_x,
                                float* absmax_inout, void* H_out, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * INT8 GEMM with dequantisation epilogue   [SQ-p5] §2.1 (int32
 *     accumulation, out / (c_x outer c_w)); [SQ-p2] 为什么激活不能用逐通道量化
 *     (Y = diag(dX) Xq Wq diag(dW)).
 *   acc[i,j] = sum_k Xq[i,k] * Wq[j,k]   (exact int32; |acc| <= 127^2 K)
 *   out_dt = SQ_I32: Y = acc.
 *   otherwise: Y = acc / (qs_x[i or 0] * qs_w[j or 0]) + bias[j], computed in
 *   fp32 as acc * ((1/qs_x) * (1/qs_w)) (+ bias), rounded once to out_dt in
 *   {F32, F16, BF16}. bias: [N] fp32 or NULL.
 *   Xq: [M,K] int8 contiguous; Wq: [N,K] int8 contiguous; Y: [M,N] stride ldy.
 *   K % 16 == 0, K <= 133144 (int32 bound); Xq, Wq 16-byte aligned.
 *   Workspace (SQ_OP_GEMM, size from sq_workspace_size for the same M, N, K)
 *   holds the status word of the bounded waits and, for shapes whose last
 *   wave of whole tiles would be at most three quarters full, the scratch of
 *   a stream-K split of that wave (arrival counters and parked int32 partial
 *   sums). Zero it once before first use; every call that completes leaves
 *   the status word and the counters at zero again (the parked sums need no
 *   clearing). The counters sit at the same bytes (an 8 KiB region after the
 *   256-byte header) for every shape, so one workspace, sized for the largest,
 *   serves GEMM calls of several shapes in turn (not calls of other ops,
 *   whose counters sit elsewhere). After a call that timed out, sq_workspace_status (which
 *   reports SQ_ERR_TIMEOUT) clears the counters as well. A smaller workspace (at
 *   least 256 bytes) is accepted and runs every tile whole. Calls sharing one
 *   workspace must not run concurrently.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_gemm_w8a8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                         const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                         const float* bias, sq_dtype_t out_dt, void* Y, int64_t ldy,
                         void* workspace, size_t ws_bytes, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * INT8 GEMM with the MLP activation in its epilogue   [SQ-p2]
 *     融入前序线性层的权重 (down_proj's input is act(gate) * up of the
 *     gate/up projection's output; FC2's is act(fc1)); [SQ-p5] §2.1.
 *   The GEMM of sq_gemm_w8a8 (same operands, scales, bias and workspace), whose
 *   16-bit outputs Y (out_dt F16 or BF16, each one rounding of the fp32
 *   dequantised value) are not written; instead:
 *   SQ_ACT_SWIGLU: the weight's output channels come in interleaved pairs,
 *     channel 2c the gate and 2c+1 the up projection of MLP channel c (N
 *     even); H[i, c] = silu(Y[i, 2c]) * Y[i, 2c + 1], H is [M, N/2];
 *   SQ_ACT_RELU / SQ_ACT_GELU: H[i, j] = act(Y[i, j]), H is [M, N];
 *   each h computed in fp32 from the 16-bit Y values exactly as sq_act_quant
 *   computes it (for the same Y, de-interleaved for SwiGLU). Then:
 *   static_qs == NULL: H holds h rounded once to out_dt (16-bit elements, the
 *     H_out of sq_act_quant); per-token int8 of H then comes from
 *     sq_quantize_act;
 *   static_qs != NULL (a device scale): H holds the int8 codes
 *     clip(rne(h * qs), -127, 127) with the fp32 h, the codes sq_act_quant
 *     gives with that static scale, and nothing else is written.
 *   H has row stride ldh (elements). The [M, N] output Y never reaches
 *   memory: for SwiGLU half the 16-bit bytes go out, with a static scale a
 *   quarter (one byte per MLP channel, no second pass), and the activation's
 *   arithmetic runs while the next tile's MMAs do.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_gemm_w8a8_act(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                                    const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                                    const float* bias, sq_act_t act, const float* static_qs, sq_dtype_t out_dt,
                                    void* H, int64_t ldh, void* workspace, size_t ws_bytes, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * Batched INT8 GEMM for attention     lpnh.cn SmoothQuant practice article
 *     §2.2 (the QK^T and PV products of attention can be quantised).
 *   Y[b] = Aq[b] Bq[b]^T dequantised as sq_gemm_w8a8 for b < batch:
 *   Aq: [batch, M, K] int8, Bq: [batch, N, K] int8 (each contiguous, problems
 *   back to back); qs_a: [batch, M] (a_per_row) or [batch] scales, qs_b:
 *   [batch, N] (b_per_row) or [batch]; Y: [batch, M, ldy] of out_dt in {I32,
 *   F32, F16, BF16}. For QK^T: A = Q, B = K, one scale per (head, token). For
 *   PV: A = P (per row), B = V^T (V transposed to [d, T], one scale per (head,
 *   channel): a scale along the summed token axis would not factor out).
 *   K % 16 == 0. Workspace as sq_gemm_w8a8.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_bmm_w8a8(const int8_t* Aq, const int8_t* Bq, int64_t batch, int64_t M, int64_t N, int64_t K,
                               const float* qs_a, int a_per_row, const float* qs_b, int b_per_row,
                               sq_dtype_t out_dt, void* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                               sq_stream_t stream);

/* --------------------------------------------------------------------------
 * The same W8A8 path on FP8 units      [SQ-p3] 技術原理與特性 (the
 *     smoothed model runs on INT8 or FP8 compute units). Format: OCP FP8
 *     E4M3 (largest finite value 448, no infinities), codes stored one byte
 *     per value.
 * sq_quantize_weight_fp8 / sq_quantize_act_fp8: as sq_quantize_weight /
 *   sq_quantize_act (same operands, s semantics, per-row or per-tensor
 *   scales, workspace rules), with qs = 448 / max(m, 1e-8) and the code of
 *   fl32(v * qs) rounded to the nearest E4M3 value (ties to even),
 *   magnitudes past 448 saturated. Wq / Xq: [rows, K] uint8.
 * sq_gemm_fp8: Y = acc / (qs_x * qs_w) (+ bias) as sq_gemm_w8a8, where acc is
 *   the fp32 tensor-core sum of the exact E4M3 products (its error is within
 *   K * 2^-23 * sum |a b|). out_dt in {F32, F16, BF16}. K % 16 == 0.
 * ------------------------------------------------------------------------ */
SQ_API sq_status_t sq_quantize_weight_fp8(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s,
                                          int per_channel, uint8_t* Wq, float* qs_w, void* workspace,
                                          size_t ws_bytes, sq_stream_t stream);
SQ_API sq_status_t sq_quantize_act_fp8(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                                       const float* s, int per_token, const float* static_qs, uint8_t* Xq,
                                       float* qs_x, void* workspace, size_t ws_bytes, sq_stream_t stream);
SQ_API sq_status_t sq_gemm_fp8(const uint8_t* Xq, const uint8_t* Wq, int64_t M, int64_t N, int64_t K,
                               const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                               const float* bias, sq_dtype_t out_dt, void* Y, int64_t ldy, void* workspace,
                               size_t ws_bytes, sq_stream_t stream);

/* --------------------------------------------------------------------------
 * LLM.int8() mixed-precision decomposition     [SQ-p5] §2.2, §2.3,
 *        §4.1.
 * ------------------------------------------------------------------------ */

/* Outlier dimensions O = { j : count_i(|X[i,j]| > threshold) / M >
 * min_ratio } in ascending order (fp64 ratio and comparison; the threshold
 * test is strict, in fp32). min_ratio = 0 marks a column on any single
 * value over the threshold. X: [M,K] dt in {F16, BF16}, stride ldx.
 * outlier_idx: [K] int32 (first *n_outliers entries valid); n_outliers: [1]
 * int32, device. Workspace: SQ_OP_LLMINT8_DETECT, zeroed once before its
 * first use: it holds arrival counters that every completed call leaves at
 * zero (one pass over X counts per 128-row band; the last band of each
 * 256-column group adds the group up, the last group writes O). The counters
 * sit at the same bytes for every M and K, so a workspace serves any later
 * call it is large enough for. Calls sharing a workspace must not run
 * concurrently. K % 8 == 0, K <= 2^20. */
SQ_API sq_status_t sq_llmint8_detect(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                              float threshold, double min_ratio, int32_t* outlier_idx,
                              int32_t* n_outliers, void* workspace, size_t ws_bytes,
                              sq_stream_t stream);

/* sq_llmint8_detect_noalloc: sq_llmint8_detect without the workspace
 * argument. The pages have no counterpart to this entry point; it only changes
 * where the scratch memory comes from. It is for callers that cannot allocate
 * device memory or hand scratch to the library: a component that runs where
 * another layer owns every buffer and passes in only inputs and outputs (an
 * inference engine's plugin slot, a memory arena planned ahead of time with
 * nothing to spare), or a service that must not allocate once it is serving.
 * The scratch is a fixed 4 MiB device array inside this library, one per
 * device that loads it, held until the process exits. It holds the per-band
 * counts (4 * ceil(M / 128) * K bytes) after a 256-byte header, 16 KiB of
 * arrival counters and 32 bytes of outlier mask per 256 columns (rounded up
 * to 256 bytes), so for example M <= 32512 at K = 4096; larger sizes return
 * SQ_ERR_UNSUPPORTED_SHAPE and launch nothing.
 * The first call in a CUDA context looks up the array's device address there
 * (cudaGetSymbolAddress), keyed by the context's unique id, so a new context
 * (another driver-API context, or the primary context again after
 * cudaDeviceReset) gets its own lookup; make that first call before any
 * stream capture.
 * Every call uses the same array: calls that overlap on the GPU (other
 * streams, other host threads) race, so the caller must serialise them.
 * Each call first clears the array's arrival counters on its stream (a
 * memset, no allocation); the counts it reads it writes itself.
 * Arguments and results are those of sq_llmint8_detect. */
SQ_API sq_status_t sq_llmint8_detect_noalloc(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                                             float threshold, double min_ratio, int32_t* outlier_idx,
                                             int32_t* n_outliers, sq_stream_t stream);

/* Vector-wise row quantisation over the columns not in O:
 * qs_x[i] = 127 / max(max_{j not in O} |X[i,j]|, 1e-8);
 * Xq[i,j] = 0 for j in O, else clip(rne(X*qs), -127, 127).
 * idx / n_idx: device outlier list (as written by sq_llmint8_detect). */
SQ_API sq_status_t sq_llmint8_quant_rows(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                                  const int32_t* idx, const int32_t* n_idx, int8_t* Xq,
                                  float* qs_x, sq_stream_t stream);

/* Weight side: vector-wise quantisation of W over the input channels not
 * in O (one scale per output channel): qs_w[n] = 127/max(max_{k not in O}
 * |W[n,k]|, 1e-8); Wq[n,k] = 0 for k in O. W: [N,K] dt in {F16, BF16}. */
SQ_API sq_status_t sq_llmint8_quant_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K,
                                    const int32_t* idx, const int32_t* n_idx, int8_t* Wq,
                                    float* qs_w, sq_stream_t stream);

/* Weight state for sq_llmint8_matmul. W is the caller's 16-bit weight [N,K]
 * (same dtype as X). Wq [N,K] int8, qs_w [N] fp32, cached_idx [K] int32 and
 * cached_n [1] int32 are caller-allocated device buffers that the library
 * maintains: they hold the int8 weight for the outlier set in cached_idx.
 * Set *cached_n = -1 (device) before the first call to mark the cache empty.
 * wo (optional, may be NULL): a caller-allocated device buffer of
 * 32 x ceil(N/256)*256 fp32 in which the library keeps the outlier input
 * channels of W for the cached set, transposed (wo[o, n] = W[n, O_o]), so a
 * call whose O is unchanged does not gather them again; with NULL they are
 * gathered into the workspace on every call. */
typedef struct {
    const void* W;
    int64_t N;
    int8_t* Wq;
    float* qs_w;
    int32_t* cached_idx;
    int32_t* cached_n;
    float* wo;
} sq_llmint8_weight_t;

/* The whole decomposition in one call: detect O on X; if O differs from the cached set,
 * requantise the weight for O (on the device, no host synchronisation);
 * quantise the rows of X; then one GEMM whose epilogue forms
 *   Y[i,j] = acc[i,j] / (qs_x[i] * qs_w[j]) + sum_{o in O ascending} X[i,o] * W[j,o]
 * in fp32 (the 16-bit products are exact in fp32) and rounds once to dt.
 * X, Y: dt in {F16, BF16}; Y [M,N] stride ldy. idx_out [K], n_out [1]
 * receive O. Workspace: SQ_OP_LLMINT8. K % 16 == 0. */
SQ_API sq_status_t sq_llmint8_matmul(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                              const sq_llmint8_weight_t* w, float threshold, double min_ratio,
                              void* Y, int64_t ldy, int32_t* idx_out, int32_t* n_out,
                              void* workspace, size_t ws_bytes, sq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SQ_API_H */

// Smoothing factors and the offline folds, including the fold into the
// previous linear layer ("大语言模型量化技术（四）：SmoothQuant", section
// 融入前序线性层的权重: up_proj's output channel j, or v_proj's, divided by s_j).
//
// s_j = x_j^alpha / w_j^(1-alpha) ("大语言模型量化技术（四）：SmoothQuant", section
// 缩放因子; lpnh.cn SmoothQuant article §2.1) with clamp(min=1e-5) on both
// statistics and on s (same article, §3.2). The power is evaluated in fp64 and
// rounded once to fp32; alpha = 0, 1/2, 1 use the page's closed forms 1/w,
// sqrt(x/w), x (correctly rounded operations, so these three cases are exact
// to the last bit on any IEEE machine).
//
// W' = diag(s) W (section SmoothQuant 的原理): with the torch layout [N,K]
// input channel k of every row is multiplied by s_k ("如何通过 SmoothQuant
// 解决激活值离群点难题" §3, weight.mul_(s.view(1,-1))). gamma' = gamma / s and
// beta' = beta / s fold 1/s into the preceding norm (section 融入 LayerNorm).
#include "sq_common.cuh"

namespace sq {
namespace {

__device__ __forceinline__ float smooth_one(float x, float w, double alpha) {
    const float xc = fmaxf(x, 1e-5f);
    const float wc = fmaxf(w, 1e-5f);
    double v;
    if (alpha == 0.5)
        v = __dsqrt_rn(__ddiv_rn((double)xc, (double)wc));
    else if (alpha == 0.0)
        v = __ddiv_rn(1.0, (double)wc);
    else if (alpha == 1.0)
        v = (double)xc;
    else
        v = __ddiv_rn(pow((double)xc, alpha), pow((double)wc, 1.0 - alpha));
    return fmaxf(__double2float_rn(v), 1e-5f);
}

__global__ void smooth_scales_kernel(const float* __restrict__ x, const float* __restrict__ w,
                                     int64_t K, double alpha, float* __restrict__ s) {
    pdl_wait();
    pdl_trigger();
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < K;
         j += (int64_t)gridDim.x * blockDim.x)
        s[j] = smooth_one(x[j], w[j], alpha);
}

// s, then gamma' = gamma / s (and beta' = beta / s), in one pass
__global__ void smooth_fold_norm_kernel(const float* __restrict__ x, const float* __restrict__ w, int64_t K,
                                        double alpha, const float* __restrict__ g, const float* __restrict__ b,
                                        float* __restrict__ s, float* __restrict__ g_out, float* __restrict__ b_out) {
    pdl_wait();
    pdl_trigger();
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < K;
         j += (int64_t)gridDim.x * blockDim.x) {
        const float sj = smooth_one(x[j], w[j], alpha);
        s[j] = sj;
        g_out[j] = __fdiv_rn(g[j], sj);
        if (b) b_out[j] = __fdiv_rn(b[j], sj);
    }
}

template <typename T>
__global__ void fold_weight_kernel(const T* __restrict__ W, int64_t N, int64_t K,
                                   const float* __restrict__ s, float* __restrict__ Wp) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = Vec<T>::N;
    const int64_t nvec = N * K / V;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e0 = v * V;
        const int64_t k0 = e0 % K;  // K % V == 0: a vector never crosses a row
        float f[V];
        unpack<T>(ldg_nc_v4(W + e0), f);
        float o[V];
#pragma unroll
        for (int e = 0; e < V; ++e) o[e] = __fmul_rn(f[e], __ldg(s + k0 + e));
#pragma unroll
        for (int e = 0; e < V; e += 4)
            *reinterpret_cast<float4*>(Wp + e0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
    }
}

__global__ void fold_norm_kernel(const float* __restrict__ g, const float* __restrict__ b,
                                 const float* __restrict__ s, int64_t K, float* g_out, float* b_out) {
    pdl_wait();
    pdl_trigger();
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < K;
         j += (int64_t)gridDim.x * blockDim.x) {
        const float sj = s[j];
        const float gv = g[j];
        const float bv = b ? b[j] : 0.0f;
        g_out[j] = __fdiv_rn(gv, sj);
        if (b) b_out[j] = __fdiv_rn(bv, sj);
    }
}

// Fold into the previous linear: row n of the previous layer divided by s_n (and its bias).
template <typename T>
__global__ void fold_prev_kernel(const T* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ bias,
                                 const float* __restrict__ s, float* __restrict__ Wp, float* __restrict__ bias_out) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = Vec<T>::N;
    const int64_t nvec = N * K / V;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e0 = v * V;
        const int64_t n = e0 / K;  // K % V == 0: a vector never crosses a row
        const float sn = __ldg(s + n);
        float f[V];
        unpack<T>(ldg_nc_v4(W + e0), f);
#pragma unroll
        for (int e = 0; e < V; ++e) f[e] = __fdiv_rn(f[e], sn);
#pragma unroll
        for (int e = 0; e < V; e += 4)
            *reinterpret_cast<float4*>(Wp + e0 + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    }
    if (bias)
        for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x)
            bias_out[n] = __fdiv_rn(bias[n], s[n]);
}

int grid_for(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (b > cap) b = cap;
    return (int)(b > 0 ? b : 1);
}

}  // namespace
}  // namespace sq

extern "C" {

sq_status_t sq_smooth_scales(const float* xmax, const float* wmax, int64_t K, double alpha,
                             float* s_out, sq_stream_t stream) {
    SQ_REQUIRE(xmax && wmax && s_out, SQ_ERR_INVALID_ARG, "sq_smooth_scales: null pointer");
    SQ_REQUIRE(K > 0, SQ_ERR_UNSUPPORTED_SHAPE, "sq_smooth_scales: K must be > 0");
    SQ_REQUIRE(alpha >= 0.0 && alpha <= 1.0, SQ_ERR_INVALID_ARG, "sq_smooth_scales: alpha must be in [0, 1]");
    sq::launch_pdl(sq::smooth_scales_kernel, dim3(sq::grid_for(K, 256)), dim3(256), 0, sq::as_cuda(stream), xmax, wmax, K, alpha, s_out);
    return sq::check_launch("sq_smooth_scales");
}

sq_status_t sq_fold_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s,
                           float* Wp_out, sq_stream_t stream) {
    SQ_REQUIRE(W && s && Wp_out, SQ_ERR_INVALID_ARG, "sq_fold_weight: null pointer");
    SQ_REQUIRE(N >= 0 && K > 0 && K % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "sq_fold_weight: need K > 0, K %% 8 == 0");
    SQ_REQUIRE(sq::aligned16(W) && sq::aligned16(Wp_out), SQ_ERR_ALIGNMENT, "sq_fold_weight: unaligned pointer");
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG,
               "sq_fold_weight: dtype must be F16, BF16 or F32");
    if (N == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    const int64_t n = N * K;
    switch (dt) {
        case SQ_F16:
            sq::launch_pdl(sq::fold_weight_kernel<__half>, dim3(sq::grid_for(n / 8, 256)), dim3(256), 0, st, 
                static_cast<const __half*>(W), N, K, s, Wp_out);
            break;
        case SQ_BF16:
            sq::launch_pdl(sq::fold_weight_kernel<__nv_bfloat16>, dim3(sq::grid_for(n / 8, 256)), dim3(256), 0, st, 
                static_cast<const __nv_bfloat16*>(W), N, K, s, Wp_out);
            break;
        case SQ_F32:
            sq::launch_pdl(sq::fold_weight_kernel<float>, dim3(sq::grid_for(n / 4, 256)), dim3(256), 0, st, 
                static_cast<const float*>(W), N, K, s, Wp_out);
            break;
        default: return sq::set_error(SQ_ERR_INVALID_ARG, "sq_fold_weight: dtype must be F16, BF16 or F32");
    }
    return sq::check_launch("sq_fold_weight");
}

sq_status_t sq_fold_prev_linear(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* bias,
                                const float* s, float* Wp_out, float* bias_out, sq_stream_t stream) {
    SQ_REQUIRE(W && s && Wp_out, SQ_ERR_INVALID_ARG, "sq_fold_prev_linear: null pointer");
    SQ_REQUIRE((bias == nullptr) == (bias_out == nullptr), SQ_ERR_INVALID_ARG,
               "sq_fold_prev_linear: bias and bias_out must both be given or both be NULL");
    SQ_REQUIRE(N > 0 && K > 0 && K % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "sq_fold_prev_linear: need N, K > 0, K %% 8 == 0");
    SQ_REQUIRE(sq::aligned16(W) && sq::aligned16(Wp_out), SQ_ERR_ALIGNMENT, "sq_fold_prev_linear: unaligned pointer");
    cudaStream_t st = sq::as_cuda(stream);
    const int64_t n = N * K;
    switch (dt) {
        case SQ_F16:
            sq::launch_pdl(sq::fold_prev_kernel<__half>, dim3(sq::grid_for(n / 8, 256)), dim3(256), 0, st,
                           static_cast<const __half*>(W), N, K, bias, s, Wp_out, bias_out);
            break;
        case SQ_BF16:
            sq::launch_pdl(sq::fold_prev_kernel<__nv_bfloat16>, dim3(sq::grid_for(n / 8, 256)), dim3(256), 0, st,
                           static_cast<const __nv_bfloat16*>(W), N, K, bias, s, Wp_out, bias_out);
            break;
        case SQ_F32:
            sq::launch_pdl(sq::fold_prev_kernel<float>, dim3(sq::grid_for(n / 4, 256)), dim3(256), 0, st,
                           static_cast<const float*>(W), N, K, bias, s, Wp_out, bias_out);
            break;
        default: return sq::set_error(SQ_ERR_INVALID_ARG, "sq_fold_prev_linear: dtype must be F16, BF16 or F32");
    }
    return sq::check_launch("sq_fold_prev_linear");
}

sq_status_t sq_smooth_fold_norm(const float* xmax, const float* wmax, int64_t K, double alpha, const float* gamma,
                                const float* beta, float* s_out, float* gamma_out, float* beta_out, sq_stream_t stream) {
    const char* name = "sq_smooth_fold_norm";
    SQ_REQUIRE(xmax && wmax && s_out && gamma && gamma_out, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE((beta == nullptr) == (beta_out == nullptr), SQ_ERR_INVALID_ARG,
               "%s: beta and beta_out must both be given or both be NULL", name);
    SQ_REQUIRE(K > 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be > 0", name);
    SQ_REQUIRE(alpha >= 0.0 && alpha <= 1.0, SQ_ERR_INVALID_ARG, "%s: alpha must be in [0, 1]", name);
    sq::launch_pdl(sq::smooth_fold_norm_kernel, dim3(sq::grid_for(K, 256)), dim3(256), 0, sq::as_cuda(stream), xmax,
                   wmax, K, alpha, gamma, beta, s_out, gamma_out, beta_out);
    return sq::check_launch(name);
}

sq_status_t sq_fold_norm(const float* gamma, const float* beta, const float* s, int64_t K,
                         float* gamma_out, float* beta_out, sq_stream_t stream) {
    SQ_REQUIRE(gamma && s && gamma_out, SQ_ERR_INVALID_ARG, "sq_fold_norm: null pointer");
    SQ_REQUIRE((beta == nullptr) == (beta_out == nullptr), SQ_ERR_INVALID_ARG,
               "sq_fold_norm: beta and beta_out must both be given or both be NULL");
    SQ_REQUIRE(K > 0, SQ_ERR_UNSUPPORTED_SHAPE, "sq_fold_norm: K must be > 0");
    sq::launch_pdl(sq::fold_norm_kernel, dim3(sq::grid_for(K, 256)), dim3(256), 0, sq::as_cuda(stream), gamma, beta, s, K, gamma_out,
                                                                              beta_out);
    return sq::check_launch("sq_fold_norm");
}

}  // extern "C"

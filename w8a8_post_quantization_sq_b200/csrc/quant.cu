// Symmetric absmax int8 quantisation of weights and of activations
// that do not come out of a norm.
//
// "8位量化：异常值与混合精度分解实战" §2.1: scale = 127 / max(|x|, 1e-8) over the
// quantisation group, q = clip(round(x * scale), -127, 127), round half to
// even. Groups are one row (a token of X, an output channel of W) or the
// whole tensor: these are the only granularities whose scales factor out of
// the GEMM ("大语言模型量化技术（四）：SmoothQuant", 为什么激活不能用逐通道量化).
// The weight is smoothed on the fly, W' = fp32(W) * s_k (section SmoothQuant
// 的原理); the activation is divided by s, X' = X / s ("如何通过 SmoothQuant
// 解决激活值离群点难题" §3). All arithmetic is fp32 with correctly rounded
// operations, so codes and scales are bit-exact against a plain CPU loop.
//
// The same kernels write FP8 E4M3 codes for the FP8 variant of the path
// ("SmoothQuant" (newton wiki), 技術原理與特性: INT8 or FP8 units): scale =
// 448 / max(|x|, 1e-8), codes by the saturating round-to-nearest-even
// conversion.
//
// Row mode: the row is read once into the registers of one warp (K <= 2048)
// or one block (K <= 16384), reduced to its absmax and quantised from the
// registers; longer rows stream twice through a warp. Tensor mode: a
// grid-wide absmax into the workspace, then the quantising pass.
#include <cuda_fp8.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kThreads = 256;
// kRowDivMul: row n divided by rdiv[n] (the fold of the next layer's smoothing
// into this one's output channels), then column k multiplied by s[k]
enum SMode { kNoScale = 0, kMul = 1, kDiv = 2, kRowDivMul = 3 };

// Load 8 consecutive elements as fp32.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* f) {
    if constexpr (sizeof(T) == 2) {
        unpack<T>(ldg_v4(p), f);
    } else {
        unpack<float>(ldg_v4(p), f);
        unpack<float>(ldg_v4(p + 4), f + 4);
    }
}

template <int SM>
__device__ __forceinline__ void apply_s(float* f, const float* __restrict__ s, const float* __restrict__ rdiv,
                                        int64_t row, int64_t k0) {
    if constexpr (SM == kRowDivMul) {
        const float rd = __ldg(rdiv + row);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __fdiv_rn(f[e], rd);
    }
    if constexpr (SM != kNoScale) {
        const float4 a = *reinterpret_cast<const float4*>(s + k0);
        const float4 b = *reinterpret_cast<const float4*>(s + k0 + 4);
        const float sv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        if constexpr (SM == kDiv) {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __fdiv_rn(f[e], sv[e]);
        } else {
            mul8(f, sv);
        }
    }
}

__device__ __forceinline__ float block_max(float v, float* sh) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncwarp();
    __syncthreads();  // sh may still be read from a previous use
    if (lane == 0) sh[warp] = v;
    __syncwarp();
    __syncthreads();
    float m = sh[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, sh[w]);
    return m;
}

// Output formats: int8 codes, or FP8 E4M3 codes (largest finite value 448).
enum QFmt { kI8 = 0, kE4M3 = 1 };

template <int FMT>
__device__ __forceinline__ float scale_of(float m) {
    return __fdiv_rn(FMT == kE4M3 ? 448.0f : 127.0f, fmaxf(m, 1e-8f));
}

// Eight E4M3 codes of v * qs: each product one fp32 rounding, then the
// conversion rounds to the nearest E4M3 value (ties to even) and saturates
// at +-448.
__device__ __forceinline__ uint2 fp8codes8(const float* v, float qs) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(v[4 * h], qs), __fmul_rn(v[4 * h + 1], qs)), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(v[4 * h + 2], qs), __fmul_rn(v[4 * h + 3], qs)), __NV_SATFINITE, __NV_E4M3);
        w[h] = (uint32_t)a | ((uint32_t)b << 16);
    }
    return make_uint2(w[0], w[1]);
}

// Eight int8 codes; `clip` is needed only when qs does not come from the
// group's own absmax (a static per-tensor scale).
__device__ __forceinline__ uint2 codes8_i8(const float* v, float qs, bool clip) {
    uint32_t b[8];
    if (clip) {
#pragma unroll
        for (int e = 0; e < 8; ++e) b[e] = quant_bits_clip(__fmul_rn(v[e], qs));
    } else {
        quant_bits8_noclip(v, qs, b);
    }
    return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
}

template <int FMT>
__device__ __forceinline__ uint2 codes8(const float* v, float qs, bool clip) {
    if constexpr (FMT == kE4M3) return fp8codes8(v, qs);  // saturating conversion: no separate clip
    else return codes8_i8(v, qs, clip);
}

// Warp maximum of non-negative floats (the row maxima here start at 0 and
// are formed by max operations that drop NaN operands, so they are never
// NaN): their bit patterns order as their values, so one integer redux
// replaces the five-step shuffle tree.
__device__ __forceinline__ float warp_max(float v) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}

// One 256-thread block per row (rows longer than the register-held kernels
// take), rows strided over the grid: the row's maximum in a first read, the
// codes in a second. per_row != 0: the row's own scale from its absmax; else
// *tensor_qs for every row.
template <typename T, int SM, int FMT>
__global__ void __launch_bounds__(kThreads)
row_quant_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld, const float* __restrict__ s,
                 const float* __restrict__ rdiv, int per_row, const float* __restrict__ tensor_qs,
                 int8_t* __restrict__ Q, float* __restrict__ qs_out) {
    pdl_wait();
    pdl_trigger();
    __shared__ float sh[kThreads / 32];
    const int t = threadIdx.x;
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        const T* x = X + row * ld;
        float qs;
        if (per_row) {
            float m = 0.0f;
#pragma unroll 4
            for (int64_t k0 = (int64_t)t * 8; k0 < K; k0 += 8 * kThreads) {
                float f[8];
                load8<T>(x + k0, f);
                apply_s<SM>(f, s, rdiv, row, k0);
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
            }
            qs = scale_of<FMT>(block_max(m, sh));
            if (t == 0) qs_out[row] = qs;
        } else {
            qs = *tensor_qs;
            if (row == 0 && t == 0) qs_out[0] = qs;
        }
        // the second read of the row finds it in L2: the launch keeps few
        // enough rows in flight (see quantize)
        int8_t* q = Q + row * K;
#pragma unroll 4
        for (int64_t k0 = (int64_t)t * 8; k0 < K; k0 += 8 * kThreads) {
            float f[8];
            load8<T>(x + k0, f);
            apply_s<SM>(f, s, rdiv, row, k0);
            *reinterpret_cast<uint2*>(q + k0) = codes8<FMT>(f, qs, !per_row);
        }
    }
}

// Raw 8 elements of a row as loaded (one 16-byte vector for 16-bit data, two
// for fp32).
template <typename T> struct Raw8 { uint4 a; };
template <> struct Raw8<float> { uint4 a, b; };

template <typename T>
__device__ __forceinline__ void load_raw(const T* p, Raw8<T>& r) {
    r.a = ldg_nc_v4(p);
    if constexpr (sizeof(T) == 4) r.b = ldg_nc_v4(p + 4);
}
template <typename T>
__device__ __forceinline__ void unpack_raw(const Raw8<T>& r, float* f) {
    if constexpr (sizeof(T) == 2) {
        unpack<T>(r.a, f);
    } else {
        unpack<float>(r.a, f);
        unpack<float>(r.b, f + 4);
    }
}

// The row held in registers by a group of G threads (G = 32: one warp per
// row, several rows per block; G = 256: the whole block), CH chunks of 8
// elements per thread: one read of the row from memory, a group max, then the
// codes from the registers. The next row's loads are issued before the group
// reduction so they land while this row is finished. Used while
// K <= 8 * G * CH_max.
template <typename T, int SM, int G, int CH, int FMT>
__global__ void __launch_bounds__(kThreads)
row_quant_reg_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld, const float* __restrict__ s,
                     const float* __restrict__ rdiv, int per_row, const float* __restrict__ tensor_qs,
                     int8_t* __restrict__ Q, float* __restrict__ qs_out) {
    pdl_wait();
    pdl_trigger();
    __shared__ float sh[kThreads / 32];
    constexpr int GPB = kThreads / G;  // groups (rows) per block
    const int gt = threadIdx.x % G;
    const int64_t ngroups = (int64_t)gridDim.x * GPB;
    int64_t row = (int64_t)blockIdx.x * GPB + threadIdx.x / G;
    Raw8<T> raw[CH];
    if (row < M) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t k0 = ((int64_t)gt + (int64_t)c * G) * 8;
            if (k0 < K) load_raw<T>(X + row * ld + k0, raw[c]);
        }
    }
    // G == 256: every thread of the block takes the same rows; G == 32: each
    // warp takes its own, and only warp-level reductions are used
    for (; row < M; row += ngroups) {
        float v[CH][8];
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t k0 = ((int64_t)gt + (int64_t)c * G) * 8;
            if (k0 < K) {
                unpack_raw<T>(raw[c], v[c]);
                apply_s<SM>(v[c], s, rdiv, row, k0);
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[c][e]));
            }
        }
        const int64_t nxt = row + ngroups;
        if (nxt < M) {
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const int64_t k0 = ((int64_t)gt + (int64_t)c * G) * 8;
                if (k0 < K) load_raw<T>(X + nxt * ld + k0, raw[c]);
            }
        }
        float qs;
        if (per_row) {
            if constexpr (G == 32) {
                m = warp_max(m);
            } else {
                m = block_max(m, sh);
            }
            qs = scale_of<FMT>(m);
            if (gt == 0) qs_out[row] = qs;
        } else {
            qs = *tensor_qs;
            if (row == 0 && gt == 0) qs_out[0] = qs;
        }
        int8_t* q = Q + row * K;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t k0 = ((int64_t)gt + (int64_t)c * G) * 8;
            if (k0 < K) *reinterpret_cast<uint2*>(q + k0) = codes8<FMT>(v[c], qs, !per_row);
        }
    }
}

// Grid-wide max |v| over the tensor into *out (non-negative float bits).
template <typename T, int SM>
__global__ void __launch_bounds__(kThreads)
tensor_absmax_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld,
                     const float* __restrict__ s, const float* __restrict__ rdiv, float* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    __shared__ float sh[kThreads / 32];
    const int64_t vecs_per_row = K / 8;
    const int64_t nvec = M * vecs_per_row;
    float m = 0.0f;
    for (int64_t v = blockIdx.x * (int64_t)kThreads + threadIdx.x; v < nvec; v += (int64_t)gridDim.x * kThreads) {
        const int64_t row = v / vecs_per_row;
        const int64_t k0 = (v - row * vecs_per_row) * 8;
        float f[8];
        load8<T>(X + row * ld + k0, f);
        apply_s<SM>(f, s, rdiv, row, k0);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    }
    m = block_max(m, sh);
    if (threadIdx.x == 0) atomic_max_nonneg(out, m);
}

// qs = 127 (int8) or 448 (E4M3) / max(max_j a[j], 1e-8) into *qs (one block).
template <int FMT>
__global__ void __launch_bounds__(kThreads)
scale_from_absmax_kernel(const float* __restrict__ a, int64_t n, float* __restrict__ qs) {
    pdl_wait();
    pdl_trigger();
    __shared__ float sh[kThreads / 32];
    float m = 0.0f;
    for (int64_t j = threadIdx.x; j < n; j += kThreads) m = fmaxf(m, a[j]);
    m = block_max(m, sh);
    if (threadIdx.x == 0) *qs = scale_of<FMT>(m);
}


int vec_grid(int64_t nvec) {
    int64_t b = (nvec + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

template <typename T, int SM, int FMT>
sq_status_t quantize(const void* Xv, int64_t M, int64_t K, int64_t ld, const float* s, int per_row,
                     const float* static_qs, int8_t* Q, float* qs_out, void* ws, cudaStream_t st,
                     const char* name, const float* rdiv = nullptr) {
    const T* X = static_cast<const T*>(Xv);
    const float* tensor_qs = static_qs;
    if (!per_row && !static_qs) {
        // grid-wide absmax into the workspace, then qs from it
        float* wmax = reinterpret_cast<float*>(static_cast<char*>(ws) + 16);
        float* wqs = wmax + 1;
        if (cudaMemsetAsync(wmax, 0, sizeof(float), st) != cudaSuccess) return check_launch(name);
        launch_pdl(tensor_absmax_kernel<T, SM>, dim3(vec_grid(M * K / 8)), dim3(kThreads), 0, st, X, M, K, ld, s, rdiv,
                   wmax);
        launch_pdl(scale_from_absmax_kernel<FMT>, dim3(1), dim3(kThreads), 0, st, wmax, 1, wqs);
        tensor_qs = wqs;
    }
    // one resident wave of blocks; each group strides over the rows
    auto go = [&](auto kern, int rows_per_block) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        int64_t b = (M + rows_per_block - 1) / rows_per_block;
        const int64_t cap = (int64_t)num_sms() * per_sm;
        if (b > cap) b = cap;
        return launch_pdl(kern, dim3((unsigned)b), dim3(kThreads), 0, st, X, M, K, ld, s, rdiv, per_row, tensor_qs, Q,
                          qs_out);
    };
    if (K <= 256)
        go(row_quant_reg_kernel<T, SM, 32, 1, FMT>, 8);
    else if (K <= 512)
        go(row_quant_reg_kernel<T, SM, 32, 2, FMT>, 8);
    else if (K <= 1024)
        go(row_quant_reg_kernel<T, SM, 32, 4, FMT>, 8);
    else if (K <= 2048)
        go(row_quant_reg_kernel<T, SM, 32, 8, FMT>, 8);
    else if (K <= 4096)
        go(row_quant_reg_kernel<T, SM, 256, 2, FMT>, 1);
    else if (K <= 8192)
        go(row_quant_reg_kernel<T, SM, 256, 4, FMT>, 1);
    else if (K <= 12288)
        go(row_quant_reg_kernel<T, SM, 256, 6, FMT>, 1);
    else if (K <= 16384)
        go(row_quant_reg_kernel<T, SM, 256, 8, FMT>, 1);
    else {
        // longer rows: one block per row, read twice; the rows in flight are
        // capped at about 96 MB so the second read mostly finds them in L2
        // (measured on B200 at 12288 rows of 49152 bf16: 665 us for the warp
        // per row this replaced, 637 with a 48 MB cap, 505 with 96 MB)
        int per_sm = 0;
        auto kern = row_quant_kernel<T, SM, FMT>;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        int64_t b = (int64_t)num_sms() * per_sm;
        const int64_t cap = (int64_t)(96ll << 20) / (K * (int64_t)sizeof(T));
        if (b > cap) b = cap;
        if (b < num_sms()) b = num_sms();
        if (b > M) b = M;
        launch_pdl(kern, dim3((unsigned)b), dim3(kThreads), 0, st, X, M, K, ld, s, rdiv, per_row, tensor_qs, Q, qs_out);
    }
    return check_launch(name);
}

template <int SM, int FMT = kI8>
sq_status_t quantize_dt(sq_dtype_t dt, const void* X, int64_t M, int64_t K, int64_t ld, const float* s,
                        int per_row, const float* static_qs, int8_t* Q, float* qs_out, void* ws,
                        cudaStream_t st, const char* name) {
    switch (dt) {
        case SQ_F16: return quantize<__half, SM, FMT>(X, M, K, ld, s, per_row, static_qs, Q, qs_out, ws, st, name);
        case SQ_BF16:
            return quantize<__nv_bfloat16, SM, FMT>(X, M, K, ld, s, per_row, static_qs, Q, qs_out, ws, st, name);
        case SQ_F32: return quantize<float, SM, FMT>(X, M, K, ld, s, per_row, static_qs, Q, qs_out, ws, st, name);
        default: return set_error(SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32", name);
    }
}

}  // namespace
}  // namespace sq

extern "C" {

sq_status_t sq_quantize_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s,
                               int per_channel, int8_t* Wq, float* qs_w, void* workspace, size_t ws_bytes,
                               sq_stream_t stream) {
    const char* name = "sq_quantize_weight";
    SQ_REQUIRE((W && Wq && qs_w) || N == 0, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(N >= 0 && K > 0 && K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need K > 0 and K %% 16 == 0", name);
    SQ_REQUIRE(sq::aligned16(W) && sq::aligned16(Wq) && (!s || sq::aligned16(s)), SQ_ERR_ALIGNMENT,
               "%s: W, Wq and s must be 16-byte aligned", name);
    SQ_REQUIRE(per_channel || (workspace && ws_bytes >= sq::kStatusBytes), SQ_ERR_INVALID_ARG,
               "%s: per-tensor quantisation needs a workspace of %zu bytes", name, sq::kStatusBytes);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    if (N == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    if (s)
        return sq::quantize_dt<sq::kMul>(dt, W, N, K, K, s, per_channel, nullptr, Wq, qs_w, workspace, st, name);
    return sq::quantize_dt<sq::kNoScale>(dt, W, N, K, K, nullptr, per_channel, nullptr, Wq, qs_w, workspace, st,
                                         name);
}

sq_status_t sq_quantize_weight_fold_prev(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s_next,
                                         const float* s, int8_t* Wq, float* qs_w, sq_stream_t stream) {
    const char* name = "sq_quantize_weight_fold_prev";
    SQ_REQUIRE((W && Wq && qs_w && s_next && s) || N == 0, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(N >= 0 && K > 0 && K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need K > 0 and K %% 16 == 0", name);
    SQ_REQUIRE(sq::aligned16(W) && sq::aligned16(Wq) && sq::aligned16(s), SQ_ERR_ALIGNMENT,
               "%s: W, Wq and s must be 16-byte aligned", name);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    if (N == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    switch (dt) {
        case SQ_F16:
            return sq::quantize<__half, sq::kRowDivMul, sq::kI8>(W, N, K, K, s, 1, nullptr, Wq, qs_w, nullptr, st,
                                                                 name, s_next);
        case SQ_BF16:
            return sq::quantize<__nv_bfloat16, sq::kRowDivMul, sq::kI8>(W, N, K, K, s, 1, nullptr, Wq, qs_w, nullptr,
                                                                        st, name, s_next);
        case SQ_F32:
            return sq::quantize<float, sq::kRowDivMul, sq::kI8>(W, N, K, K, s, 1, nullptr, Wq, qs_w, nullptr, st,
                                                                name, s_next);
        default: return sq::set_error(SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32", name);
    }
}

sq_status_t sq_quantize_act(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx, const float* s,
                            int per_token, const float* static_qs, int8_t* Xq, float* qs_x, void* workspace,
                            size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_quantize_act";
    SQ_REQUIRE((X && Xq && qs_x) || M == 0, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(M >= 0 && K > 0 && K % 16 == 0 && ldx >= K && ldx % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: need K > 0, K %% 16 == 0, ldx >= K, ldx %% 8 == 0", name);
    SQ_REQUIRE(sq::aligned16(X) && sq::aligned16(Xq) && (!s || sq::aligned16(s)), SQ_ERR_ALIGNMENT,
               "%s: X, Xq and s must be 16-byte aligned", name);
    SQ_REQUIRE(per_token || static_qs || (workspace && ws_bytes >= sq::kStatusBytes), SQ_ERR_INVALID_ARG,
               "%s: dynamic per-tensor quantisation needs a workspace of %zu bytes", name, sq::kStatusBytes);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    if (M == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    if (s)
        return sq::quantize_dt<sq::kDiv>(dt, X, M, K, ldx, s, per_token, static_qs, Xq, qs_x, workspace, st, name);
    return sq::quantize_dt<sq::kNoScale>(dt, X, M, K, ldx, nullptr, per_token, static_qs, Xq, qs_x, workspace, st,
                                         name);
}

sq_status_t sq_quantize_weight_fp8(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const float* s,
                                   int per_channel, uint8_t* Wq, float* qs_w, void* workspace, size_t ws_bytes,
                                   sq_stream_t stream) {
    const char* name = "sq_quantize_weight_fp8";
    SQ_REQUIRE((W && Wq && qs_w) || N == 0, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(N >= 0 && K > 0 && K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need K > 0 and K %% 16 == 0", name);
    SQ_REQUIRE(sq::aligned16(W) && sq::aligned16(Wq) && (!s || sq::aligned16(s)), SQ_ERR_ALIGNMENT,
               "%s: W, Wq and s must be 16-byte aligned", name);
    SQ_REQUIRE(per_channel || (workspace && ws_bytes >= sq::kStatusBytes), SQ_ERR_INVALID_ARG,
               "%s: per-tensor quantisation needs a workspace of %zu bytes", name, sq::kStatusBytes);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    if (N == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    int8_t* Q = reinterpret_cast<int8_t*>(Wq);
    if (s)
        return sq::quantize_dt<sq::kMul, sq::kE4M3>(dt, W, N, K, K, s, per_channel, nullptr, Q, qs_w, workspace, st,
                                                   name);
    return sq::quantize_dt<sq::kNoScale, sq::kE4M3>(dt, W, N, K, K, nullptr, per_channel, nullptr, Q, qs_w,
                                                    workspace, st, name);
}

sq_status_t sq_quantize_act_fp8(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx, const float* s,
                                int per_token, const float* static_qs, uint8_t* Xq, float* qs_x, void* workspace,
                                size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_quantize_act_fp8";
    SQ_REQUIRE((X && Xq && qs_x) || M == 0, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(M >= 0 && K > 0 && K % 16 == 0 && ldx >= K && ldx % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: need K > 0, K %% 16 == 0, ldx >= K, ldx %% 8 == 0", name);
    SQ_REQUIRE(sq::aligned16(X) && sq::aligned16(Xq) && (!s || sq::aligned16(s)), SQ_ERR_ALIGNMENT,
               "%s: X, Xq and s must be 16-byte aligned", name);
    SQ_REQUIRE(per_token || static_qs || (workspace && ws_bytes >= sq::kStatusBytes), SQ_ERR_INVALID_ARG,
               "%s: dynamic per-tensor quantisation needs a workspace of %zu bytes", name, sq::kStatusBytes);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    if (M == 0) return SQ_OK;
    cudaStream_t st = sq::as_cuda(stream);
    int8_t* Q = reinterpret_cast<int8_t*>(Xq);
    if (s)
        return sq::quantize_dt<sq::kDiv, sq::kE4M3>(dt, X, M, K, ldx, s, per_token, static_qs, Q, qs_x, workspace,
                                                    st, name);
    return sq::quantize_dt<sq::kNoScale, sq::kE4M3>(dt, X, M, K, ldx, nullptr, per_token, static_qs, Q, qs_x,
                                                    workspace, st, name);
}

sq_status_t sq_scale_from_absmax(const float* absmax, int64_t n, float* qs_out, sq_stream_t stream) {
    SQ_REQUIRE(absmax && qs_out, SQ_ERR_INVALID_ARG, "sq_scale_from_absmax: null pointer");
    SQ_REQUIRE(n > 0, SQ_ERR_UNSUPPORTED_SHAPE, "sq_scale_from_absmax: n must be > 0");
    sq::launch_pdl(sq::scale_from_absmax_kernel<sq::kI8>, dim3(1), dim3(sq::kThreads), 0, sq::as_cuda(stream), absmax, n, qs_out);
    return sq::check_launch("sq_scale_from_absmax");
}

}  // extern "C"

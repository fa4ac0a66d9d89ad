// a5: LayerNorm / RMSNorm with the smoothing folded into gamma' (and beta'),
// fused with int8 quantisation of the result.
//
// "大语言模型量化技术（四）：SmoothQuant", section 融入 LayerNorm: the norm's
// affine parameters absorb 1/s (gamma' = gamma/s, beta' = beta/s), so the
// smoothed activation costs no extra pass; the page writes the LayerNorm
// form y = (x - mu)/sigma * gamma + beta (RMSNorm drops mu and beta). The
// int8 step is the absmax rule of "8位量化：异常值与混合精度分解实战" §2.1,
// per token (row) or with a static per-tensor scale from calibration.
//
// Exactness: every step is one correctly rounded fp32 operation and the two
// row sums use a fixed order, so v, the scales and the codes are bit-equal to
// a CPU evaluation in the same order. The order: 128 lanes (the 128 threads
// of the block); thread t folds its 8-element chunks t, t+128, ... in index
// order with fma; each warp combines its 32 partials by the xor butterfly
// (16, 8, 4, 2, 1), after which every lane holds the same value; the four
// warp totals add as (G0 + G1) + (G2 + G3).
//
// Bandwidth kernels; the row stays in registers:
//   K <= 4096: one warp per row (no block barrier). Lane l holds chunks
//     l, l+32, l+64, ...; chunk c belongs to lane c mod 128 of the order above
//     (its group is (c / 32) mod 4), so the warp keeps four partials, one per
//     group, folds each in increasing chunk order, and runs the four group
//     butterflies itself: bit-identical to the 128-thread order.
//   4096 < K <= 16384: one 128-thread block per row, thread t = lane t.
// The codes are written 8 bytes per chunk, the per-token scale once per row.
#include "sq_common.cuh"

namespace sq {
namespace {

constexpr int kThreads = 128;

struct NormArgs {
    int64_t M, K, ldh;
    const float* gamma;
    const float* beta;
    float eps;
    int per_token;
    const float* static_qs;
    int8_t* Xq;
    float* qs_x;
    float* absmax;  // [K] running max |v|, or null
    void* V;        // [M,K] 16-bit, or null
};

// Fixed-order block sum of one partial per thread (see file comment).
__device__ __forceinline__ float canon_block_sum(float p, float* sh) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sh[warp] = p;
    __syncwarp();
    __syncthreads();
    const float r = __fadd_rn(__fadd_rn(sh[0], sh[1]), __fadd_rn(sh[2], sh[3]));
    __syncwarp();
    __syncthreads();
    return r;
}

__device__ __forceinline__ float block_max4(float v, float* sh) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sh[warp] = v;
    __syncwarp();
    __syncthreads();
    const float r = fmaxf(fmaxf(sh[0], sh[1]), fmaxf(sh[2], sh[3]));
    __syncwarp();
    __syncthreads();
    return r;
}

template <typename T, bool LN, int CMAX>
__global__ void __launch_bounds__(kThreads)
norm_quant_kernel(const T* __restrict__ H, NormArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ float sh[4];
    extern __shared__ float amax_sh[];  // [K] running max |v| (calibration mode)
    const int t = threadIdx.x;
    const int nch = (int)(a.K / 8);
    const float Kf = (float)a.K;
    if (a.absmax)
        for (int j = t; j < a.K; j += kThreads) amax_sh[j] = 0.0f;

    for (int64_t row = blockIdx.x; row < a.M; row += gridDim.x) {
        const T* h = H + row * a.ldh;
        uint4 raw[CMAX];
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
            const int ch = t + c * kThreads;
            if (ch < nch) raw[c] = ldg_nc_v4(h + (int64_t)ch * 8);
        }
        float mu = 0.0f, r;
        if constexpr (LN) {
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                if (t + c * kThreads < nch) {
                    float f[8];
                    unpack<T>(raw[c], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = __fmaf_rn(f[e], 1.0f, acc);
                }
            }
            mu = __fdiv_rn(canon_block_sum(acc, sh), Kf);
            acc = 0.0f;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                if (t + c * kThreads < nch) {
                    float f[8];
                    unpack<T>(raw[c], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float d = __fsub_rn(f[e], mu);
                        acc = __fmaf_rn(d, d, acc);
                    }
                }
            }
            const float var = __fdiv_rn(canon_block_sum(acc, sh), Kf);
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
        } else {
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                if (t + c * kThreads < nch) {
                    float f[8];
                    unpack<T>(raw[c], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = __fmaf_rn(f[e], f[e], acc);
                }
            }
            const float ms = __fdiv_rn(canon_block_sum(acc, sh), Kf);
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
        }

        // v_j, computed identically each time it is needed
        auto compute_v = [&](const uint4& rw, int ch, float* v) {
            float f[8];
            unpack<T>(rw, f);
            const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8));
            const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8 + 4));
            const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            if constexpr (LN) {
                float b[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                const bool hb = a.beta != nullptr;
                if (hb) {
                    const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.beta + ch * 8));
                    const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.beta + ch * 8 + 4));
                    b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
                    b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float u = __fmul_rn(__fmul_rn(__fsub_rn(f[e], mu), r), g[e]);
                    v[e] = hb ? __fadd_rn(u, b[e]) : u;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(__fmul_rn(f[e], r), g[e]);
            }
        };

        float m = 0.0f;
        const bool need_max = a.Xq && a.per_token;
        if (need_max || a.absmax || a.V) {
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                const int ch = t + c * kThreads;
                if (ch < nch) {
                    float v[8];
                    compute_v(raw[c], ch, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
                    if (a.absmax) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) amax_sh[ch * 8 + e] = fmaxf(amax_sh[ch * 8 + e], fabsf(v[e]));
                    }
                    if (a.V) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            o[e] = (uint32_t)to16<T>(v[2 * e]) | ((uint32_t)to16<T>(v[2 * e + 1]) << 16);
                        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.V) + row * a.K + ch * 8) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
        if (a.Xq) {
            float qs;
            if (a.per_token) {
                qs = __fdiv_rn(127.0f, fmaxf(block_max4(m, sh), 1e-8f));
                if (t == 0) a.qs_x[row] = qs;
            } else {
                qs = *a.static_qs;
                if (row == 0 && t == 0) a.qs_x[0] = qs;
            }
            int8_t* q = a.Xq + row * a.K;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                const int ch = t + c * kThreads;
                if (ch < nch) {
                    float v[8];
                    compute_v(raw[c], ch, v);
                    uint32_t b[8];
                    if (a.per_token) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) b[e] = quant_bits_noclip(__fmul_rn(v[e], qs));
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) b[e] = quant_bits_clip(__fmul_rn(v[e], qs));
                    }
                    *reinterpret_cast<uint2*>(q + ch * 8) =
                        make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
                }
            }
        }
    }
    if (a.absmax) {
        __syncwarp();
        __syncthreads();
        // each column was only touched by its owning thread; publish once per block
        for (int j = t; j < a.K; j += kThreads) atomic_max_nonneg(a.absmax + j, amax_sh[j]);
    }
}


// One warp per row (K <= 32 * 8 * CW); see the file comment for the order.
template <typename T, bool LN, int CW>
__global__ void __launch_bounds__(256)
norm_quant_warp_kernel(const T* __restrict__ H, NormArgs a) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float amax_sh[];  // [K] running max |v| of the block (calibration mode)
    const int lane = threadIdx.x & 31;
    const int nch = (int)(a.K / 8);
    const float Kf = (float)a.K;
    if (a.absmax) {
        for (int j = threadIdx.x; j < a.K; j += blockDim.x) amax_sh[j] = 0.0f;
        __syncwarp();
        __syncthreads();
    }
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < a.M; row += nwarps) {
        const T* h = H + row * a.ldh;
        uint4 raw[CW];
#pragma unroll
        for (int i = 0; i < CW; ++i)
            if (lane + 32 * i < nch) raw[i] = ldg_nc_v4(h + (int64_t)(lane + 32 * i) * 8);
        // fixed-order sum of f(x) over the row: four group partials per lane
        auto canon = [&](auto term) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                if (lane + 32 * i < nch) {
                    float f[8];
                    unpack<T>(raw[i], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[i & 3] = term(f[e], acc[i & 3]);
                }
            }
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) acc[w] = __fadd_rn(acc[w], __shfl_xor_sync(0xffffffffu, acc[w], o));
            return __fadd_rn(__fadd_rn(acc[0], acc[1]), __fadd_rn(acc[2], acc[3]));
        };
        float mu = 0.0f, r;
        if constexpr (LN) {
            mu = __fdiv_rn(canon([](float x, float c) { return __fmaf_rn(x, 1.0f, c); }), Kf);
            const float m_ = mu;
            const float var = __fdiv_rn(canon([m_](float x, float c) {
                const float d = __fsub_rn(x, m_);
                return __fmaf_rn(d, d, c);
            }), Kf);
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
        } else {
            const float ms = __fdiv_rn(canon([](float x, float c) { return __fmaf_rn(x, x, c); }), Kf);
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
        }
        auto compute_v = [&](const uint4& rw, int ch, float* v) {
            float f[8];
            unpack<T>(rw, f);
            const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8));
            const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8 + 4));
            const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            if constexpr (LN) {
                if (a.beta) {
                    const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.beta + ch * 8));
                    const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.beta + ch * 8 + 4));
                    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(f[e], mu), r), g[e]), b[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(__fmul_rn(__fsub_rn(f[e], mu), r), g[e]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(__fmul_rn(f[e], r), g[e]);
            }
        };
        float m = 0.0f;
        if ((a.Xq && a.per_token) || a.absmax || a.V) {
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                const int ch = lane + 32 * i;
                if (ch < nch) {
                    float v[8];
                    compute_v(raw[i], ch, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
                    if (a.absmax) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) atomicMax(reinterpret_cast<int*>(amax_sh + ch * 8 + e), __float_as_int(fabsf(v[e])));
                    }
                    if (a.V) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            o[e] = (uint32_t)to16<T>(v[2 * e]) | ((uint32_t)to16<T>(v[2 * e + 1]) << 16);
                        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.V) + row * a.K + ch * 8) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
        if (a.Xq) {
            float qs;
            if (a.per_token) {
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                qs = __fdiv_rn(127.0f, fmaxf(m, 1e-8f));
                if (lane == 0) a.qs_x[row] = qs;
            } else {
                qs = *a.static_qs;
                if (row == 0 && lane == 0) a.qs_x[0] = qs;
            }
            int8_t* q = a.Xq + row * a.K;
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                const int ch = lane + 32 * i;
                if (ch < nch) {
                    float v[8];
                    compute_v(raw[i], ch, v);
                    uint32_t b[8];
                    if (a.per_token) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) b[e] = quant_bits_noclip(__fmul_rn(v[e], qs));
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) b[e] = quant_bits_clip(__fmul_rn(v[e], qs));
                    }
                    *reinterpret_cast<uint2*>(q + ch * 8) =
                        make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
                }
            }
        }
    }
    if (a.absmax) {
        __syncwarp();
        __syncthreads();
        for (int j = threadIdx.x; j < a.K; j += blockDim.x) atomic_max_nonneg(a.absmax + j, amax_sh[j]);
    }
}

template <typename T, bool LN, int CW>
void launch_warp(const void* H, const NormArgs& a, cudaStream_t s) {
    const size_t smem = a.absmax ? (size_t)a.K * sizeof(float) : 0;
    auto kern = norm_quant_warp_kernel<T, LN, CW>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int64_t blocks = (a.M + 7) / 8;  // 8 rows (warps) per block
    const int64_t cap = (int64_t)num_sms() * (a.absmax ? 2 : 8);
    if (blocks > cap) blocks = cap;
    launch_pdl(kern, dim3((unsigned)blocks), dim3(256), smem, s, static_cast<const T*>(H), a);
}

template <typename T, bool LN, int CMAX>
void launch_one(const void* H, const NormArgs& a, cudaStream_t s) {
    const size_t smem = a.absmax ? (size_t)a.K * sizeof(float) : 0;
    auto kern = norm_quant_kernel<T, LN, CMAX>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // up to 16 resident blocks of 128 threads per SM for the small rows
    const int per_sm = CMAX <= 2 ? 16 : (CMAX <= 4 ? 8 : 4);
    int64_t grid = (int64_t)num_sms() * per_sm;
    if (a.absmax) grid = (int64_t)num_sms() * 2;  // fewer blocks: one publish of [K] per block
    if (grid > a.M) grid = a.M;
    launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), smem, s, static_cast<const T*>(H), a);
}

template <typename T, bool LN>
void launch_t(const void* H, const NormArgs& a, cudaStream_t s) {
    const int64_t nch = a.K / 8;
    if (nch <= 32) launch_warp<T, LN, 1>(H, a, s);
    else if (nch <= 64) launch_warp<T, LN, 2>(H, a, s);
    else if (nch <= 128) launch_warp<T, LN, 4>(H, a, s);
    else if (nch <= 256) launch_warp<T, LN, 8>(H, a, s);
    else if (nch <= 512) launch_warp<T, LN, 16>(H, a, s);
    else if (nch <= 1024) launch_one<T, LN, 8>(H, a, s);
    else launch_one<T, LN, 16>(H, a, s);
}

}  // namespace
}  // namespace sq

extern "C" sq_status_t sq_norm_smooth_quant(const void* H, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldh,
                                            sq_norm_t norm, const float* gamma_p, const float* beta_p, float eps,
                                            int per_token, const float* static_qs, int8_t* Xq, float* qs_x,
                                            float* absmax_inout, void* V_out, sq_stream_t stream) {
    const char* name = "sq_norm_smooth_quant";
    SQ_REQUIRE((H || M == 0) && gamma_p, SQ_ERR_INVALID_ARG, "%s: null H or gamma", name);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16, SQ_ERR_INVALID_ARG, "%s: dtype must be F16 or BF16", name);
    SQ_REQUIRE(norm == SQ_LAYERNORM || norm == SQ_RMSNORM, SQ_ERR_INVALID_ARG, "%s: bad norm type", name);
    SQ_REQUIRE(M >= 0 && K >= 8 && K <= 16384 && K % 8 == 0 && ldh >= K && ldh % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: need 8 <= K <= 16384, K %% 8 == 0, ldh >= K, ldh %% 8 == 0", name);
    SQ_REQUIRE(!Xq || qs_x, SQ_ERR_INVALID_ARG, "%s: Xq needs qs_x", name);
    SQ_REQUIRE(!Xq || per_token || static_qs, SQ_ERR_INVALID_ARG, "%s: per-tensor mode needs static_qs", name);
    SQ_REQUIRE(Xq || absmax_inout || V_out, SQ_ERR_INVALID_ARG, "%s: no output requested", name);
    SQ_REQUIRE(sq::aligned16(H) && sq::aligned16(gamma_p) && (!beta_p || sq::aligned16(beta_p)) &&
                   (!Xq || sq::aligned16(Xq)) && (!V_out || sq::aligned16(V_out)),
               SQ_ERR_ALIGNMENT, "%s: H, gamma, beta, Xq and V must be 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    sq::NormArgs a{M, K, ldh, gamma_p, norm == SQ_LAYERNORM ? beta_p : nullptr, eps, per_token, static_qs,
                   Xq, qs_x, absmax_inout, V_out};
    cudaStream_t s = sq::as_cuda(stream);
    const bool ln = norm == SQ_LAYERNORM;
    if (dt == SQ_BF16) {
        if (ln) sq::launch_t<__nv_bfloat16, true>(H, a, s);
        else sq::launch_t<__nv_bfloat16, false>(H, a, s);
    } else {
        if (ln) sq::launch_t<__half, true>(H, a, s);
        else sq::launch_t<__half, false>(H, a, s);
    }
    return sq::check_launch(name);
}

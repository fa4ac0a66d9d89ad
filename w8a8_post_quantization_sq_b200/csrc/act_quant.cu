// The input of down_proj (FC2), act(gate) * up for a SwiGLU MLP, relu(fc1)
// for a ReLU MLP or gelu(fc1) for a GELU MLP, quantised to int8 per token or with a static
// per-tensor scale; optional 16-bit copy of h and a running per-channel max of
// |h| for calibration.
//
// "大语言模型量化技术（四）：SmoothQuant", section 融入前序线性层的权重: the
// smoothing of down_proj's input is folded into up_proj's output channels,
// so h arrives already divided by s and only needs quantising ("8位量化：
// 异常值与混合精度分解实战" §2.1). For a SwiGLU MLP the gate/up projection
// writes one [M, 2I] row per token: gate in columns [0, I), up in [I, 2I).
//
// silu and gelu are fixed sequences of correctly rounded fp32 operations
// (sq_act.cuh), so h, the scales and the codes are bit-equal to a CPU
// evaluation of the same sequence.
//
// One 256-thread block per row, rows strided over the grid. Up to I = 16384
// the thread's h values stay in registers between the absmax and the codes;
// longer rows compute h twice.
#include "sq_act.cuh"
#include "sq_common.cuh"

namespace sq {
namespace {

constexpr int kT = 256;

struct ActArgs {
    int64_t M, I, lda;
    int act;  // SQ_ACT_SWIGLU, SQ_ACT_RELU or SQ_ACT_GELU
    int per_token;
    const float* static_qs;
    int8_t* Xq;
    float* qs_x;
    float* absmax;  // [I] running max |h|, or null
    void* H;        // [M, I] 16-bit copy of h, or null
};

// h of the 8 channels starting at column c of row `row`
template <typename T, int ACT>
__device__ __forceinline__ void act8(const T* __restrict__ A, const ActArgs& a, int64_t row, int64_t c, float* h) {
    const T* r = A + row * a.lda;
    float x[8];
    unpack<T>(ldg_nc_v4(r + c), x);
    if constexpr (ACT == SQ_ACT_SWIGLU) {
        float u[8];
        unpack<T>(ldg_nc_v4(r + a.I + c), u);
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = __fmul_rn(silu_fixed(x[e]), u[e]);
    } else if constexpr (ACT == SQ_ACT_GELU) {
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = gelu_fixed(x[e]);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = x[e] > 0.0f ? x[e] : 0.0f;
    }
}

__device__ __forceinline__ float block_max(float v, float* sh) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sh[warp] = v;
    __syncwarp();
    __syncthreads();
    float r = sh[0];
#pragma unroll
    for (int w = 1; w < kT / 32; ++w) r = fmaxf(r, sh[w]);
    __syncwarp();
    __syncthreads();  // sh is free again for the next row
    return r;
}

__device__ __forceinline__ uint2 codes8(const float* h, float qs, bool clip) {
    uint32_t b[8];
    if (clip) {
#pragma unroll
        for (int e = 0; e < 8; ++e) b[e] = quant_bits_clip(__fmul_rn(h[e], qs));
    } else {
        quant_bits8_noclip(h, qs, b);
    }
    return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
}

// CH > 0: thread t owns chunks t + kT*i (i < CH) and keeps their h in
// registers; CH == 0: any I, h formed again for the codes.
template <typename T, int ACT, int CH>
__global__ void __launch_bounds__(kT)
act_quant_kernel(const T* __restrict__ A, ActArgs a) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float amax_sh[];  // [I] running max |h| of the block (calibration mode)
    __shared__ float sh[kT / 32];
    const int t = threadIdx.x;
    const int nch = (int)(a.I / 8);
    if (a.absmax) {
        for (int j = t; j < a.I; j += kT) amax_sh[j] = 0.0f;
        __syncwarp();
        __syncthreads();
    }
    for (int64_t row = blockIdx.x; row < a.M; row += gridDim.x) {
        float hk[CH > 0 ? CH : 1][8];
        float m = 0.0f;
        auto visit = [&](int ch, const float* h) {
#pragma unroll
            for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(h[e]));
            if (a.absmax) {
#pragma unroll
                for (int e = 0; e < 8; ++e) atomic_max_nonneg(amax_sh + ch * 8 + e, fabsf(h[e]));
            }
            if (a.H) {
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) o[e] = (uint32_t)to16<T>(h[2 * e]) | ((uint32_t)to16<T>(h[2 * e + 1]) << 16);
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.H) + row * a.I + ch * 8) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            }
        };
        if constexpr (CH > 0) {
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int ch = t + kT * i;
                if (ch < nch) {
                    act8<T, ACT>(A, a, row, (int64_t)ch * 8, hk[i]);
                    visit(ch, hk[i]);
                }
            }
        } else {
#pragma unroll 4
            for (int ch = t; ch < nch; ch += kT) {
                float h[8];
                act8<T, ACT>(A, a, row, (int64_t)ch * 8, h);
                visit(ch, h);
            }
        }
        if (!a.Xq) continue;
        float qs;
        if (a.per_token) {
            qs = __fdiv_rn(127.0f, fmaxf(block_max(m, sh), 1e-8f));
            if (t == 0) a.qs_x[row] = qs;
        } else {
            qs = *a.static_qs;
            if (row == 0 && t == 0) a.qs_x[0] = qs;
        }
        int8_t* q = a.Xq + row * a.I;
        if constexpr (CH > 0) {
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int ch = t + kT * i;
                if (ch < nch) *reinterpret_cast<uint2*>(q + ch * 8) = codes8(hk[i], qs, !a.per_token);
            }
        } else {
#pragma unroll 4
            for (int ch = t; ch < nch; ch += kT) {
                float h[8];
                act8<T, ACT>(A, a, row, (int64_t)ch * 8, h);
                *reinterpret_cast<uint2*>(q + ch * 8) = codes8(h, qs, !a.per_token);
            }
        }
    }
    if (a.absmax) {
        __syncwarp();
        __syncthreads();
        for (int j = t; j < a.I; j += kT) atomic_max_nonneg(a.absmax + j, amax_sh[j]);
    }
}

template <typename T, int ACT, int CH>
void launch_k(const void* A, const ActArgs& a, cudaStream_t s) {
    auto kern = act_quant_kernel<T, ACT, CH>;
    const size_t smem = a.absmax ? (size_t)a.I * sizeof(float) : 0;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kT, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    int64_t grid = (int64_t)num_sms() * (a.absmax ? 1 : per_sm);  // calibration: few blocks, few publishes
    if (grid > a.M) grid = a.M;
    launch_pdl(kern, dim3((unsigned)grid), dim3(kT), smem, s, static_cast<const T*>(A), a);
}

template <typename T, int ACT>
void launch_t(const void* A, const ActArgs& a, cudaStream_t s) {
    const int64_t nch = a.I / 8;
    if (nch <= kT) launch_k<T, ACT, 1>(A, a, s);
    else if (nch <= 2 * kT) launch_k<T, ACT, 2>(A, a, s);
    else if (nch <= 4 * kT) launch_k<T, ACT, 4>(A, a, s);
    else if (nch <= 8 * kT) launch_k<T, ACT, 8>(A, a, s);
    else launch_k<T, ACT, 0>(A, a, s);
}

}  // namespace
}  // namespace sq

extern "C" sq_status_t sq_act_quant(const void* A, sq_dtype_t dt, int64_t M, int64_t I, int64_t lda, sq_act_t act,
                                    int per_token, const float* static_qs, int8_t* Xq, float* qs_x,
                                    float* absmax_inout, void* H_out, sq_stream_t stream) {
    const char* name = "sq_act_quant";
    SQ_REQUIRE(A || M == 0, SQ_ERR_INVALID_ARG, "%s: null A", name);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16, SQ_ERR_INVALID_ARG, "%s: dtype must be F16 or BF16", name);
    SQ_REQUIRE(act == SQ_ACT_SWIGLU || act == SQ_ACT_RELU || act == SQ_ACT_GELU, SQ_ERR_INVALID_ARG,
               "%s: bad activation", name);
    const int64_t width = act == SQ_ACT_SWIGLU ? 2 * I : I;
    SQ_REQUIRE(M >= 0 && I > 0 && I % 8 == 0 && lda >= width && lda % 8 == 0 && I <= (int64_t)1 << 24,
               SQ_ERR_UNSUPPORTED_SHAPE, "%s: need I > 0, I %% 8 == 0, lda >= %s, lda %% 8 == 0", name,
               act == SQ_ACT_SWIGLU ? "2I" : "I");
    if (M == 0) return SQ_OK;  // nothing to do; empty tensors may come with null pointers
    SQ_REQUIRE(!Xq || qs_x, SQ_ERR_INVALID_ARG, "%s: Xq needs qs_x", name);
    SQ_REQUIRE(!Xq || per_token || static_qs, SQ_ERR_INVALID_ARG, "%s: per-tensor mode needs static_qs", name);
    SQ_REQUIRE(Xq || absmax_inout || H_out, SQ_ERR_INVALID_ARG, "%s: no output requested", name);
    SQ_REQUIRE(!absmax_inout || I <= 57344, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: calibration mode keeps [I] floats in shared memory (I <= 57344)", name);
    SQ_REQUIRE(sq::aligned16(A) && (!Xq || sq::aligned16(Xq)) && (!H_out || sq::aligned16(H_out)),
               SQ_ERR_ALIGNMENT, "%s: A, Xq and H must be 16-byte aligned", name);
    sq::ActArgs a{M, I, lda, (int)act, per_token, static_qs, Xq, qs_x, absmax_inout, H_out};
    cudaStream_t s = sq::as_cuda(stream);
    if (dt == SQ_BF16) {
        if (act == SQ_ACT_SWIGLU) sq::launch_t<__nv_bfloat16, SQ_ACT_SWIGLU>(A, a, s);
        else if (act == SQ_ACT_GELU) sq::launch_t<__nv_bfloat16, SQ_ACT_GELU>(A, a, s);
        else sq::launch_t<__nv_bfloat16, SQ_ACT_RELU>(A, a, s);
    } else {
        if (act == SQ_ACT_SWIGLU) sq::launch_t<__half, SQ_ACT_SWIGLU>(A, a, s);
        else if (act == SQ_ACT_GELU) sq::launch_t<__half, SQ_ACT_GELU>(A, a, s);
        else sq::launch_t<__half, SQ_ACT_RELU>(A, a, s);
    }
    return sq::check_launch(name);
}

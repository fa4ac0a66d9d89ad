// LayerNorm / RMSNorm with the smoothing folded into gamma' (and beta'),
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
// a CPU evaluation in the same order. The order: 256 lanes; lane t folds its
// 8-element chunks t, t+256, ... in index order with fma; each group of 32
// lanes combines by the xor butterfly (16, 8, 4, 2, 1), after which every lane
// of the group holds the same value; the eight group totals add as
// ((G0 + G1) + (G2 + G3)) + ((G4 + G5) + (G6 + G7)).
//
// Bandwidth kernels; the row stays in registers:
//   K <= 4096: one warp per row (no block barrier). Lane l holds chunks
//     l, l+32, l+64, ...; chunk c belongs to lane c mod 256 of the order above,
//     in group (c / 32) mod 8, so the warp keeps eight partials, one per
//     group, folds each in increasing chunk order and runs the eight group
//     butterflies itself: bit-identical to the 256-lane order.
//   4096 < K <= 16384: one 256-thread block per row, thread t = lane t. Rows
//     reach shared memory through a ring of buffers, one bulk copy (TMA
//     engine, cp.async.bulk) per row issued R rows ahead, so several rows per
//     block are in flight while the block reduces and quantises; gamma' of a
//     thread's chunks lives in its registers for the whole launch, beta' in
//     shared memory.
// The codes are written 8 bytes per chunk, the per-token scale once per row.
#include "sq_common.cuh"

namespace sq {
namespace {

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

__device__ __forceinline__ float butterfly_sum(float p) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
    return p;
}

__device__ __forceinline__ float tree8(const float* g) {
    return __fadd_rn(__fadd_rn(__fadd_rn(g[0], g[1]), __fadd_rn(g[2], g[3])),
                     __fadd_rn(__fadd_rn(g[4], g[5]), __fadd_rn(g[6], g[7])));
}

// Warp maximum of non-negative floats (the row maxima here start at 0 and
// are formed by max operations that drop NaN operands, so they are never
// NaN): their bit patterns order as their values, so one integer redux
// replaces the five-step shuffle tree.
__device__ __forceinline__ float warp_max(float v) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}

// max(a, b, c) in one instruction (exact; the order of a max does not matter)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// max(m, |v_0|, ..., |v_7|)
__device__ __forceinline__ float absmax8(float m, const float* v) {
    const float m0 = max3f(m, fabsf(v[0]), fabsf(v[1]));
    const float m1 = max3f(fabsf(v[2]), fabsf(v[3]), fabsf(v[4]));
    return max3f(max3f(m0, fabsf(v[5]), fabsf(v[6])), m1, fabsf(v[7]));
}

// v_j of one 8-element chunk from d_j = x_j - mu (LayerNorm) or x_j
// (RMSNorm), given r: (d * r) * gamma' (+ beta'). g holds gamma'_j of the
// chunk; b_lo / b_hi point at beta'_j of its first and last four elements
// (null: no shift). v may alias d.
__device__ __forceinline__ void compute_v_d(const float* d, const float4* b_lo, const float4* b_hi, const float* g,
                                            float r, float* v) {
    const uint64_t r2 = pk2(r, r);
    if (b_lo) {
        // the last product feeds an add: the products go as packed pairs, the
        // adds stay scalar (a packed multiply feeding a packed add has been
        // seen fused into one rounding; feeding a scalar add it has not)
        const float4 b0 = *b_lo, b1 = *b_hi;
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float t0, t1;
            upk2(mul2(mul2(pk2(d[e], d[e + 1]), r2), pk2(g[e], g[e + 1])), t0, t1);
            v[e] = __fadd_rn(t0, b[e]);
            v[e + 1] = __fadd_rn(t1, b[e + 1]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; e += 2) upk2(mul2(mul2(pk2(d[e], d[e + 1]), r2), pk2(g[e], g[e + 1])), v[e], v[e + 1]);
    }
}

// d_j = x_j - mu for the eight elements of a chunk, in place
__device__ __forceinline__ void center8(float* f, float mu) {
    const uint64_t nmu2 = pk2(-mu, -mu);  // x + (-mu) is the IEEE x - mu
#pragma unroll
    for (int e = 0; e < 8; e += 2) upk2(add2(pk2(f[e], f[e + 1]), nmu2), f[e], f[e + 1]);
}

// Mixed-precision forms (a 16-bit operand widened exactly, one fp32 rounding):
// acc + x_e in index order over a chunk, and d_e = x_e - mu, straight from the
// packed 16-bit row, with no separate unpack.
template <typename T> struct Mix;
template <> struct Mix<__nv_bfloat16> {
    static __device__ __forceinline__ float add(uint32_t w, float acc) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
            "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %0, hi, %0;\n\t}"
            : "+f"(acc) : "r"(w));
        return acc;
    }
    static __device__ __forceinline__ void sub(uint32_t w, float mu, float& d0, float& d1) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "sub.rn.f32.bf16 %0, lo, %3;\n\tsub.rn.f32.bf16 %1, hi, %3;\n\t}"
            : "=f"(d0), "=f"(d1) : "r"(w), "f"(mu));
    }
};
template <> struct Mix<__half> {
    static __device__ __forceinline__ float add(uint32_t w, float acc) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
            "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %0, hi, %0;\n\t}"
            : "+f"(acc) : "r"(w));
        return acc;
    }
    static __device__ __forceinline__ void sub(uint32_t w, float mu, float& d0, float& d1) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "sub.rn.f32.f16 %0, lo, %3;\n\tsub.rn.f32.f16 %1, hi, %3;\n\t}"
            : "=f"(d0), "=f"(d1) : "r"(w), "f"(mu));
    }
};
template <typename T>
__device__ __forceinline__ float add8_16(const uint4& w, float acc) {
    acc = Mix<T>::add(w.x, acc);
    acc = Mix<T>::add(w.y, acc);
    acc = Mix<T>::add(w.z, acc);
    return Mix<T>::add(w.w, acc);
}
template <typename T>
__device__ __forceinline__ void sub8_16(const uint4& w, float mu, float* d) {
    Mix<T>::sub(w.x, mu, d[0], d[1]);
    Mix<T>::sub(w.y, mu, d[2], d[3]);
    Mix<T>::sub(w.z, mu, d[4], d[5]);
    Mix<T>::sub(w.w, mu, d[6], d[7]);
}

// v_j of one chunk from its fp32 inputs f (v may alias f)
template <bool LN>
__device__ __forceinline__ void compute_v_f(const float* f, const float4* b_lo, const float4* b_hi, const float* g,
                                            float mu, float r, float* v) {
    if constexpr (LN) {
        float d[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = f[e];
        center8(d, mu);
        compute_v_d(d, b_lo, b_hi, g, r, v);
    } else {
        compute_v_d(f, nullptr, nullptr, g, r, v);
    }
}

// the same from the chunk's 16-bit inputs
template <typename T, bool LN>
__device__ __forceinline__ void compute_v_g(const uint4& rw, const float4* b_lo, const float4* b_hi, const float* g,
                                            float mu, float r, float* v) {
    float f[8];
    unpack<T>(rw, f);
    compute_v_f<LN>(f, b_lo, b_hi, g, mu, r, v);
}

__device__ __forceinline__ void load_gamma(const NormArgs& a, int ch, float* g) {
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + ch * 8 + 4));
    g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
    g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
}

// v_j of one 8-element chunk, gamma'_j and beta'_j read from global memory
template <typename T, bool LN>
__device__ __forceinline__ void compute_v(const uint4& rw, int ch, const NormArgs& a, float mu, float r, float* v) {
    float g[8];
    load_gamma(a, ch, g);
    const float4* bl = a.beta ? reinterpret_cast<const float4*>(a.beta) + ch * 2 : nullptr;
    compute_v_g<T, LN>(rw, bl, bl + 1, g, mu, r, v);
}

// Per-chunk parameters staged in shared memory as two planes of float4 (the
// first and last four of every chunk), so a warp reading the chunks of 32
// consecutive lanes touches 512 consecutive bytes per plane: no bank conflicts.
__device__ __forceinline__ void stage_planes(float4* dst, const float* src, int nch, int tid, int nthreads) {
    for (int j = tid; j < nch * 2; j += nthreads)
        dst[(j & 1) * nch + (j >> 1)] = __ldg(reinterpret_cast<const float4*>(src) + j);
}

template <typename T>
__device__ __forceinline__ void store_v16(const NormArgs& a, int64_t row, int ch, const float* v) {
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = (uint32_t)to16<T>(v[2 * e]) | ((uint32_t)to16<T>(v[2 * e + 1]) << 16);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.V) + row * a.K + ch * 8) = make_uint4(o[0], o[1], o[2], o[3]);
}

// int8 codes of eight values. Without a clip the products v * qs go two at a
// time (packed multiply) into the scalar shifter add: a packed multiply feeding
// a scalar add keeps its own rounding (the bit-exact parity tests hit many
// exact ties here), unlike a packed multiply feeding a packed add.
__device__ __forceinline__ uint2 codes8(const float* v, float qs, bool clip) {
    uint32_t b[8];
    if (clip) {
#pragma unroll
        for (int e = 0; e < 8; ++e) b[e] = quant_bits_clip(__fmul_rn(v[e], qs));
    } else {
        const uint64_t q2 = pk2(qs, qs);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float t0, t1;
            upk2(mul2(pk2(v[e], v[e + 1]), q2), t0, t1);
            b[e] = quant_bits_noclip(t0);
            b[e + 1] = quant_bits_noclip(t1);
        }
    }
    return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
}

// ------------------------------------------------------------------ K <= 4096
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
        // fixed-order sum of term(x) over the row: eight group partials per lane
        auto canon = [&](auto term) {
            float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                if (lane + 32 * i < nch) {
                    float f[8];
                    unpack<T>(raw[i], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[i & 7] = term(f[e], acc[i & 7]);
                }
            }
#pragma unroll
            for (int w = 0; w < 8; ++w) acc[w] = butterfly_sum(acc[w]);
            return tree8(acc);
        };
        float mu = 0.0f, r;
        if constexpr (LN) {
            mu = __fdiv_rn(canon([](float x, float c) { return __fmaf_rn(x, 1.0f, c); }), Kf);
            const float m_ = mu;
            const float var = __fdiv_rn(canon([m_](float x, float c) {
                const float d = __fsub_rn(x, m_);
                return __fmaf_rn(d, d, c);
            }), Kf);
            r = __frcp_rn(__fsqrt_rn(__fadd_rn(var, a.eps)));
        } else {
            const float ms = __fdiv_rn(canon([](float x, float c) { return __fmaf_rn(x, x, c); }), Kf);
            r = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, a.eps)));
        }
        float m = 0.0f;
        if ((a.Xq && a.per_token) || a.absmax || a.V) {
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                const int ch = lane + 32 * i;
                if (ch < nch) {
                    float v[8];
                    compute_v<T, LN>(raw[i], ch, a, mu, r, v);
                    m = absmax8(m, v);
                    if (a.absmax) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            atomicMax(reinterpret_cast<int*>(amax_sh + ch * 8 + e), __float_as_int(fabsf(v[e])));
                    }
                    if (a.V) store_v16<T>(a, row, ch, v);
                }
            }
        }
        if (a.Xq) {
            float qs;
            if (a.per_token) {
                qs = __fdiv_rn(127.0f, fmaxf(warp_max(m), 1e-8f));
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
                    compute_v<T, LN>(raw[i], ch, a, mu, r, v);
                    *reinterpret_cast<uint2*>(q + ch * 8) = codes8(v, qs, !a.per_token);
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

// ------------------------------------------------------------------ K > 4096
constexpr int kBlock = 256;
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for a row copy; false after about 2 s.
__device__ __noinline__ bool wait_row_slow(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}
// the common case inline (one try_wait, which itself suspends the thread for
// a while), the bounded loop only when that is not enough
__device__ __forceinline__ bool wait_row(uint32_t bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || wait_row_slow(bar, parity);
}
// One row (bytes, a multiple of 16) from global into shared memory, completing
// on the mbarrier; a plain bulk copy, no multicast.
__device__ __forceinline__ void issue_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Fixed-order block sum of one partial per thread (thread t = lane t).
__device__ __forceinline__ float canon_block_sum(float p, float* sh) {
    p = butterfly_sum(p);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sh[warp] = p;
    __syncwarp();
    __syncthreads();
    return tree8(sh);
}

__device__ __forceinline__ float block_max8(float v, float* sh) {
    v = warp_max(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sh[warp] = v;
    __syncwarp();
    __syncthreads();
    float r = sh[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) r = fmaxf(r, sh[w]);
    return r;
}

// One 256-thread block per row, rows strided over the grid (K <= 256*8*C).
// Thread t always owns chunks t, t+256, ..., so gamma'_j of its chunks is
// loaded once into registers. The rows arrive in a ring of R shared-memory
// buffers, each filled by one bulk copy issued R rows ahead.
//   KEEPV: the sum pass unpacks the thread's chunks into registers, so the
//     row's buffer is refilled right after the first reduction, and v is
//     formed in place and kept there until the codes are written.
//   otherwise (K > 12288): every pass reads the staged row again and the
//     buffer is refilled after the codes.
// CF: every thread owns at least CF chunks (CF == C: K == 2048 * C, no tail
//   test at all; CF == C - 1: only the last chunk is tested, so the first
//   CF chunks' loads and arithmetic are scheduled without branches).
// QONLY: codes and scales only (no V output, no calibration maxima).
// CALIB: calibration maxima only (no codes, no V): a thread owns the same
//   columns in every row, so it keeps their running max |v| in registers and
//   publishes them once, with one atomic max per column, when the block ends.
template <typename T, bool LN, int C, bool KEEPV, int CF, bool QONLY, bool CALIB = false>
__global__ void __launch_bounds__(kBlock, 2)
norm_quant_bulk_kernel(const T* __restrict__ H, NormArgs a, int R) {
    static_assert(!(QONLY && CALIB), "codes-only and calibration-only are exclusive");
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t dsm[];  // R rows, then [K] floats (calibration mode)
    __shared__ __align__(8) uint64_t bars[8];
    __shared__ float sh[3][8];
    const int t = threadIdx.x;
    const int nch = (int)(a.K / 8);
    const float Kf = (float)a.K;
    const uint32_t row_bytes = (uint32_t)(a.K * sizeof(T));
    float* amax_sh = reinterpret_cast<float*>(dsm + (size_t)R * row_bytes);
    // beta' (LayerNorm with a shift) staged once per block after the maxima
    constexpr bool kAmaxSh = !QONLY && !CALIB;  // calibration maxima in shared memory
    float4* beta_sh = (LN && a.beta) ? reinterpret_cast<float4*>(amax_sh + (kAmaxSh && a.absmax ? a.K : 0)) : nullptr;
    float amr[CALIB ? C : 1][8];  // CALIB: this thread's columns' running max |v|
#pragma unroll
    for (int c = 0; c < (CALIB ? C : 1); ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) amr[c][e] = 0.0f;
    auto b_lo = [&](int ch) { return beta_sh ? beta_sh + ch : nullptr; };
    auto b_hi = [&](int ch) { return beta_sh ? beta_sh + nch + ch : nullptr; };
    const int64_t G = gridDim.x;
    constexpr bool FULL = CF == C;
    auto mine = [&](int c) { return c < CF || t + c * kBlock < nch; };
    // the first R rows are requested before anything else, so their DRAM
    // latency overlaps the loads of gamma' and beta' below (the barriers are
    // used by other threads only after the block barrier that follows)
    if (t == 0) {
        for (int i = 0; i < R; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        for (int i = 0; i < R; ++i) {
            const int64_t r = blockIdx.x + i * G;
            if (r < a.M) issue_row(smem_u32(dsm + (size_t)i * row_bytes), H + r * a.ldh, row_bytes, smem_u32(&bars[i]));
        }
    }
    float g[C][8];
#pragma unroll
    for (int c = 0; c < C; ++c)
        if (mine(c)) load_gamma(a, t + c * kBlock, g[c]);
    if (kAmaxSh && a.absmax)
        for (int j = t; j < a.K; j += kBlock) amax_sh[j] = 0.0f;
    if (beta_sh) stage_planes(beta_sh, a.beta, nch, t, kBlock);
    __syncwarp();
    __syncthreads();
    bool aborted = false;
    int64_t abort_row = a.M;  // first row this block did not finish
    int it = 0;
    for (int64_t row = blockIdx.x; row < a.M; row += G, ++it) {
        const int slot = it % R;
        const uint8_t* xs = dsm + (size_t)slot * row_bytes;
        const bool ok = wait_row(smem_u32(&bars[slot]), (uint32_t)((it / R) & 1));
        __syncwarp();
        if (__syncthreads_and(ok) == 0) {  // a copy never landed: give up (not expected)
            aborted = true;
            abort_row = row;
            break;
        }
        auto chunk = [&](int c) { return *reinterpret_cast<const uint4*>(xs + (size_t)(t + c * kBlock) * 16); };
        // every thread is past its last read of the slot: refill it R rows ahead
        auto refill = [&]() {
            if (t == 0) {
                const int64_t nr = row + (int64_t)R * G;
                if (nr < a.M) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    issue_row(smem_u32(dsm + (size_t)slot * row_bytes), H + nr * a.ldh, row_bytes,
                              smem_u32(&bars[slot]));
                }
            }
        };
        float vk[KEEPV ? C : 1][8];
        // pass 1: the sum (LayerNorm: of x; RMSNorm: of x^2) in the lane's order.
        // LayerNorm with the row in registers keeps the packed 16-bit chunks
        // and sums them with mixed-precision adds; d = x - mu is formed from
        // them the same way below.
        // (not for the ragged C = 6 case, nor calibration, whose registers hold the maxima: they would spill)
        constexpr bool kRaw = LN && KEEPV && (FULL || C <= 4) && !CALIB;
        uint4 raw[kRaw ? C : 1];
        float acc = 0.0f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (mine(c)) {
                if constexpr (kRaw) {
                    raw[c] = chunk(c);
                    acc = add8_16<T>(raw[c], acc);
                } else {
                    float fl[8];
                    float* f = KEEPV ? vk[c] : fl;
                    unpack<T>(chunk(c), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = LN ? __fmaf_rn(f[e], 1.0f, acc) : __fmaf_rn(f[e], f[e], acc);
                }
            }
        }
        auto rstd = [&](float s_) { return __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(s_, Kf), a.eps))); };
        float mu = 0.0f, r;
        if constexpr (LN) {
            mu = __fdiv_rn(canon_block_sum(acc, sh[0]), Kf);
            if constexpr (KEEPV) refill();
            acc = 0.0f;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                if (mine(c)) {
                    // d = x - mu, kept in registers from here on when the row is
                    float fl[8];
                    float* d = KEEPV ? vk[c] : fl;
                    if constexpr (kRaw) {
                        sub8_16<T>(raw[c], mu, d);
                    } else {
                        if constexpr (!KEEPV) unpack<T>(chunk(c), fl);
                        center8(d, mu);
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = __fmaf_rn(d[e], d[e], acc);
                }
            }
            r = rstd(canon_block_sum(acc, sh[1]));
        } else {
            r = rstd(canon_block_sum(acc, sh[0]));
            if constexpr (KEEPV) refill();
        }
        // pass 2: v, its absmax, the optional outputs
        float m = 0.0f;
        if (KEEPV || a.per_token || (!QONLY && (a.absmax || a.V))) {
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const int ch = t + c * kBlock;
                if (mine(c)) {
                    float vl[8];
                    float* v = KEEPV ? vk[c] : vl;
                    if constexpr (KEEPV) compute_v_d(vk[c], b_lo(ch), b_hi(ch), g[c], r, v);  // vk holds d
                    else compute_v_g<T, LN>(chunk(c), b_lo(ch), b_hi(ch), g[c], mu, r, v);
                    if constexpr (CALIB) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) amr[c][e] = fmaxf(amr[c][e], fabsf(v[e]));
                    } else {
                        m = absmax8(m, v);
                    }
                    if constexpr (kAmaxSh) {
                        if (a.absmax) {
                            float4* am = reinterpret_cast<float4*>(amax_sh + ch * 8);
                            const float4 o0 = am[0], o1 = am[1];
                            am[0] = make_float4(fmaxf(o0.x, fabsf(v[0])), fmaxf(o0.y, fabsf(v[1])),
                                                fmaxf(o0.z, fabsf(v[2])), fmaxf(o0.w, fabsf(v[3])));
                            am[1] = make_float4(fmaxf(o1.x, fabsf(v[4])), fmaxf(o1.y, fabsf(v[5])),
                                                fmaxf(o1.z, fabsf(v[6])), fmaxf(o1.w, fabsf(v[7])));
                        }
                        if (a.V) store_v16<T>(a, row, ch, v);
                    }
                }
            }
        }
        // pass 3: the codes
        if (!CALIB && (QONLY || a.Xq)) {
            float qs;
            if (a.per_token) {
                qs = __fdiv_rn(127.0f, fmaxf(block_max8(m, sh[2]), 1e-8f));
                if (t == 0) a.qs_x[row] = qs;
            } else {
                qs = *a.static_qs;
                if (row == 0 && t == 0) a.qs_x[0] = qs;
            }
            int8_t* q = a.Xq + row * a.K;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const int ch = t + c * kBlock;
                if (mine(c)) {
                    if constexpr (KEEPV) {
                        *reinterpret_cast<uint2*>(q + ch * 8) = codes8(vk[c], qs, !a.per_token);
                    } else {
                        float v[8];
                        compute_v_g<T, LN>(chunk(c), b_lo(ch), b_hi(ch), g[c], mu, r, v);
                        *reinterpret_cast<uint2*>(q + ch * 8) = codes8(v, qs, !a.per_token);
                    }
                }
            }
        }
        if constexpr (!KEEPV) {
            // the codes read the staged row: refill its buffer once every
            // thread is done with it
            __syncwarp();
            __syncthreads();
            refill();
        }
        // (the shared partials of the reductions are next written after the
        // next row's first barrier, so no barrier is needed here)
    }
    if (aborted && t == 0) {
        // drain copies still in flight before the block's shared memory is released
        for (int i = 0; i < R; ++i) {
            const uint64_t t0 = global_ns();
            for (uint32_t ph = 0; ph < 2; ++ph)
                while (!mbar_try_wait(smem_u32(&bars[i]), ph))
                    if (global_ns() - t0 > kWaitNs / 4) break;
        }
    }
    if (aborted) {
        // the call's results are incomplete: say so in them. The scales of the
        // rows this block did not finish (or the static scale) become NaN, and
        // so do the calibration maxima, so the failure reaches the host in the
        // outputs themselves (there is no workspace to carry a status word)
        const float nan = __int_as_float(0x7fc00000);
        if (a.Xq) {
            if (a.per_token) {
                for (int64_t r = abort_row + (int64_t)t * G; r < a.M; r += (int64_t)kBlock * G) a.qs_x[r] = nan;
            } else if (t == 0) {
                a.qs_x[0] = nan;
            }
        }
        if (kAmaxSh && a.absmax)
            for (int j = t; j < a.K; j += kBlock) amax_sh[j] = nan;  // NaN bits order above every finite value
        if constexpr (CALIB) {
#pragma unroll
            for (int c = 0; c < C; ++c)
#pragma unroll
                for (int e = 0; e < 8; ++e) amr[c][e] = nan;
        }
    }
    if (kAmaxSh && a.absmax) {
        __syncwarp();
        __syncthreads();
        for (int j = t; j < a.K; j += kBlock) atomic_max_nonneg(a.absmax + j, amax_sh[j]);
    }
    if constexpr (CALIB) {
        // each column has one owner per block: one atomic max per column
#pragma unroll
        for (int c = 0; c < C; ++c)
            if (mine(c))
#pragma unroll
                for (int e = 0; e < 8; ++e) atomic_max_nonneg(a.absmax + (t + c * kBlock) * 8 + e, amr[c][e]);
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

template <typename T, bool LN, int C, bool KEEPV, int CF, bool QONLY, bool CALIB = false>
void launch_block_k(const void* H, const NormArgs& a, cudaStream_t s) {
    auto kern = norm_quant_bulk_kernel<T, LN, C, KEEPV, CF, QONLY, CALIB>;
    const size_t row_bytes = (size_t)a.K * sizeof(T);
    const size_t extra = (a.absmax && !CALIB ? (size_t)a.K * sizeof(float) : 0) +
                         (LN && a.beta ? (size_t)a.K * sizeof(float) : 0);
    // about 96 KB of staged rows and beta' (a block per SM with shared-memory maxima: 96 KB of rows)
    int R = (int)((96 * 1024 - (a.absmax && !CALIB ? 0 : extra)) / row_bytes);
    if (R < 2) R = 2;
    if (R > 8) R = 8;
    const size_t smem = (size_t)R * row_bytes + extra;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBlock, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    int64_t grid = (int64_t)num_sms() * per_sm;
    if (a.absmax && !CALIB) grid = (int64_t)num_sms();  // fewer blocks: one publish of [K] per block
    if (grid > a.M) grid = a.M;
    launch_pdl(kern, dim3((unsigned)grid), dim3(kBlock), smem, s, static_cast<const T*>(H), a, R);
}

// The chunks every thread owns: C (full), C - 1 (only the last chunk is
// ragged) or fewer (every chunk tested). Measured on B200, LayerNorm + int8 at
// 8192 x 7168 fp16 (3.5 chunks per thread): every chunk tested 62.8 us.
template <typename T, bool LN, int C, bool KEEPV, bool QONLY, bool CALIB>
void launch_cf(const void* H, const NormArgs& a, cudaStream_t s) {
    const int64_t nch = a.K / 8;
    if (nch == (int64_t)kBlock * C) launch_block_k<T, LN, C, KEEPV, C, QONLY, CALIB>(H, a, s);
    else if (nch > (int64_t)kBlock * (C - 1)) launch_block_k<T, LN, C, KEEPV, C - 1, QONLY, CALIB>(H, a, s);
    else launch_block_k<T, LN, C, KEEPV, 0, QONLY, CALIB>(H, a, s);
}

template <typename T, bool LN, int C, bool KEEPV>
void launch_block(const void* H, const NormArgs& a, cudaStream_t s) {
    const bool qonly = a.Xq && !a.absmax && !a.V;
    // calibration only (up to K = 8192): the running maxima in registers
    if constexpr (KEEPV && C == 4) {
        if (!a.Xq && !a.V && a.absmax) {
            launch_cf<T, LN, C, KEEPV, false, true>(H, a, s);
            return;
        }
    }
    if (qonly) launch_cf<T, LN, C, KEEPV, true, false>(H, a, s);
    else launch_cf<T, LN, C, KEEPV, false, false>(H, a, s);
}

template <typename T, bool LN>
void launch_t(const void* H, const NormArgs& a, cudaStream_t s) {
    const int64_t nch = a.K / 8;
    if (nch <= 32) launch_warp<T, LN, 1>(H, a, s);
    else if (nch <= 64) launch_warp<T, LN, 2>(H, a, s);
    else if (nch <= 128) launch_warp<T, LN, 4>(H, a, s);
    else if (nch <= 256) launch_warp<T, LN, 8>(H, a, s);
    else if (nch <= 512) launch_warp<T, LN, 16>(H, a, s);
    else if (nch <= 1024) launch_block<T, LN, 4, true>(H, a, s);
    else if (nch <= 1536) launch_block<T, LN, 6, true>(H, a, s);
    else launch_block<T, LN, 8, false>(H, a, s);
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

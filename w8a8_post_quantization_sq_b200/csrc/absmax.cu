// Per-input-channel absmax for calibration.
//
// x_j = max_i |X_ij| over the calibration tokens and w_j = max over output
// channels of |W| in input channel j ("大语言模型量化技术（四）：SmoothQuant",
// section 缩放因子; lpnh.cn SmoothQuant article §3.2; "如何通过 SmoothQuant
// 解决激活值离群点难题" §3). With W stored [N,K] both are the same operation: a
// column max over the rows of a row-major matrix, kept as a running max.
//
// Bandwidth kernel. A block of 8 warps covers 32 lanes x four 16-byte vectors
// of columns (1024 columns of a 16-bit matrix, 512 of an fp32 one) and a band
// of rows; warp w reads rows w, w+8, ..., two rows per step, so every warp
// reads 2 KB contiguous segments. Each lane keeps the running max of its
// columns in registers, the warps combine with shared-memory atomics, and one
// atomicMax per column per block publishes the result. max and |.| are exact,
// so the result does not depend on the order. Inputs of 16 MB and more take a
// bulk-staged variant (below) that keeps more bytes in flight per SM.
#include "sq_common.cuh"

namespace sq {
namespace {

constexpr int kWarps = 8;
constexpr int kU = 4;  // 16-byte vectors per lane per row: a warp reads 2 KB of a row

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
col_absmax_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld, int rows_per_block,
                  float* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = Vec<T>::N;
    constexpr int LC = V * kU;     // columns per lane
    constexpr int COLS = 32 * LC;  // columns per block
    __shared__ int red[COLS];      // block maxima as non-negative float bits
    for (int c = threadIdx.x; c < COLS; c += kWarps * 32) red[c] = 0;
    __syncwarp();
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c0 = (int64_t)blockIdx.x * COLS + lane * LC;
    const int64_t r_begin = (int64_t)blockIdx.y * rows_per_block;
    const int64_t r_end = min(M, r_begin + rows_per_block);
    float m[LC];
#pragma unroll
    for (int e = 0; e < LC; ++e) m[e] = 0.0f;
    int nv = 0;  // whole vectors of this lane inside K
    if (c0 < K) nv = (int)min((int64_t)kU, (K - c0) / V);
    if (nv > 0) {
        const T* base = X + c0;
        int64_t r = r_begin + warp;
        for (; r + kWarps < r_end; r += 2 * kWarps) {
            uint4 raw[2][kU];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    if (u < nv) raw[h][u] = ldg_nc_v4(base + (r + h * kWarps) * ld + u * V);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    if (u < nv) {
                        float f[V];
                        unpack<T>(raw[h][u], f);
#pragma unroll
                        for (int e = 0; e < V; ++e) m[u * V + e] = fmaxf(m[u * V + e], fabsf(f[e]));
                    }
        }
        for (; r < r_end; r += kWarps) {
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (u < nv) {
                    float f[V];
                    unpack<T>(ldg_nc_v4(base + r * ld + u * V), f);
#pragma unroll
                    for (int e = 0; e < V; ++e) m[u * V + e] = fmaxf(m[u * V + e], fabsf(f[e]));
                }
        }
    }
    // slot of column lane * LC + e is e * 32 + lane: the 32 lanes of an atomic
    // hit 32 different banks
#pragma unroll
    for (int e = 0; e < LC; ++e)
        if (e / V < nv) atomicMax(&red[e * 32 + lane], __float_as_int(m[e]));
    __syncwarp();
    __syncthreads();
    for (int c = threadIdx.x; c < COLS; c += kWarps * 32) {
        const int64_t col = (int64_t)blockIdx.x * COLS + c;
        if (col < K) atomicMax(reinterpret_cast<int*>(out + col), red[(c % LC) * 32 + c / LC]);
    }
}

// Bulk-staged variant for large inputs. A block owns 1024 columns of a
// 16-bit matrix (512 of fp32), i.e. 2 KB of every row, and a band of rows.
// Thread t owns 8 bytes of each row segment (4 columns of a 16-bit matrix, 2 of
// fp32) for the whole launch, so its running maxima need no combining inside
// the block. One thread streams the band through a ring of kStages stages of
// kStageRows row segments with plain bulk copies (cp.async.bulk, no
// multicast); each stage completes on an mbarrier (bounded wait).
constexpr int kStageRows = 16;
constexpr int kStages = 3;
constexpr int kSegBytes = 2048;
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
__device__ __noinline__ bool wait_stage_slow(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}
// the common case inline (one try_wait, which itself suspends the thread for
// a while), the bounded loop only when that is not enough
__device__ __forceinline__ bool wait_stage(uint32_t bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || wait_stage_slow(bar, parity);
}

template <typename T>
__device__ __forceinline__ void max8b(uint2 w, float* m);
template <>
__device__ __forceinline__ void max8b<__nv_bfloat16>(uint2 w, float* m) {
    m[0] = fmaxf(m[0], fabsf(__uint_as_float(w.x << 16)));
    m[1] = fmaxf(m[1], fabsf(__uint_as_float(w.x & 0xffff0000u)));
    m[2] = fmaxf(m[2], fabsf(__uint_as_float(w.y << 16)));
    m[3] = fmaxf(m[3], fabsf(__uint_as_float(w.y & 0xffff0000u)));
}
template <>
__device__ __forceinline__ void max8b<__half>(uint2 w, float* m) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    m[0] = fmaxf(m[0], fabsf(a.x));
    m[1] = fmaxf(m[1], fabsf(a.y));
    m[2] = fmaxf(m[2], fabsf(b.x));
    m[3] = fmaxf(m[3], fabsf(b.y));
}
template <>
__device__ __forceinline__ void max8b<float>(uint2 w, float* m) {
    m[0] = fmaxf(m[0], fabsf(__uint_as_float(w.x)));
    m[1] = fmaxf(m[1], fabsf(__uint_as_float(w.y)));
}

template <typename T>
__global__ void __launch_bounds__(256)
col_absmax_bulk_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld, int rows_per_block,
                       float* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    constexpr int EB = (int)sizeof(T);
    constexpr int COLS = kSegBytes / EB;  // columns per block
    constexpr int TC = 8 / EB;            // columns per thread
    extern __shared__ __align__(128) uint8_t ring_raw[];  // [kStages][kStageRows][kSegBytes]
    auto ring = reinterpret_cast<uint8_t(*)[kStageRows][kSegBytes]>(ring_raw);
    __shared__ __align__(8) uint64_t bars[kStages];
    const int t = threadIdx.x;
    const int64_t c0 = (int64_t)blockIdx.x * COLS;
    const uint32_t seg = (uint32_t)(min((int64_t)COLS, K - c0) * EB);  // bytes of each row segment
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_block;
    const int64_t r1 = min(M, r0 + rows_per_block);
    const int nst = (int)((r1 - r0 + kStageRows - 1) / kStageRows);
    auto issue = [&](int s) {  // stage s of the band into slot s % kStages (thread 0)
        const int slot = s % kStages;
        const int64_t rs = r0 + (int64_t)s * kStageRows;
        const int n = (int)min((int64_t)kStageRows, r1 - rs);
        const uint32_t bar = smem_u32(&bars[slot]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(seg * n) : "memory");
        for (int i = 0; i < n; ++i)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(smem_u32(&ring[slot][i][0])), "l"(X + (rs + i) * ld + c0), "r"(seg), "r"(bar)
                         : "memory");
    };
    if (t == 0) {
        for (int i = 0; i < kStages; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        for (int s = 0; s < kStages && s < nst; ++s) issue(s);
    }
    __syncwarp();
    __syncthreads();
    const bool active = (uint32_t)t * 8u < seg;  // this thread's columns exist
    float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    bool aborted = false;
    for (int s = 0; s < nst; ++s) {
        const int slot = s % kStages;
        const bool ok = wait_stage(smem_u32(&bars[slot]), (uint32_t)((s / kStages) & 1));
        __syncwarp();
        if (__syncthreads_and(ok) == 0) {  // a copy never landed: give up (not expected)
            aborted = true;
            break;
        }
        const int n = (int)min((int64_t)kStageRows, r1 - (r0 + (int64_t)s * kStageRows));
        if (active) {
#pragma unroll 4
            for (int i = 0; i < n; ++i) max8b<T>(*reinterpret_cast<const uint2*>(&ring[slot][i][t * 8]), m);
        }
        __syncwarp();
        __syncthreads();  // every thread is done with the slot
        if (t == 0 && s + kStages < nst) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(s + kStages);
        }
    }
    if (aborted && t == 0) {
        // drain copies still in flight before the block's shared memory is released
        for (int i = 0; i < kStages; ++i) {
            const uint64_t t0 = global_ns();
            for (uint32_t ph = 0; ph < 2; ++ph)
                while (!mbar_try_wait(smem_u32(&bars[i]), ph))
                    if (global_ns() - t0 > kWaitNs / 4) break;
        }
    }
    if (active) {
        // a band that gave up (not expected) publishes NaN for its columns:
        // NaN's bits order above every finite value, so the maxima the host
        // reads carry the failure
#pragma unroll
        for (int e = 0; e < TC; ++e)
            atomic_max_nonneg(out + c0 + t * TC + e, aborted ? __int_as_float(0x7fc00000) : m[e]);
    }
}

template <typename T>
sq_status_t launch(const void* X, int64_t M, int64_t K, int64_t ld, float* out, cudaStream_t s,
                   const char* name) {
    if ((double)M * (double)K * sizeof(T) >= 16.0 * (1 << 20)) {
        // large input: bulk-staged kernel, as many row bands as resident blocks allow
        constexpr int COLS = kSegBytes / (int)sizeof(T);
        const int64_t col_blocks = (K + COLS - 1) / COLS;
        const size_t smem = (size_t)kStages * kStageRows * kSegBytes;
        auto kern = col_absmax_bulk_kernel<T>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        int64_t bands = (int64_t)num_sms() * per_sm / col_blocks;
        if (bands < 1) bands = 1;
        int64_t rpb = (M + bands - 1) / bands;
        if (rpb < kStageRows) rpb = kStageRows;
        const int64_t row_blocks = (M + rpb - 1) / rpb;
        SQ_REQUIRE(row_blocks <= 65535 && rpb <= INT32_MAX, SQ_ERR_UNSUPPORTED_SHAPE, "%s: too many rows (M=%lld)",
                   name, (long long)M);
        launch_pdl(kern, dim3((unsigned)col_blocks, (unsigned)row_blocks), dim3(256), smem, s,
                   static_cast<const T*>(X), M, K, ld, (int)rpb, out);
        return check_launch(name);
    }
    constexpr int COLS = 32 * Vec<T>::N * kU;
    const int64_t col_blocks = (K + COLS - 1) / COLS;
    // one full wave of resident blocks: as many row bands as fit beside the
    // column blocks; rows per band a multiple of the warp count
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, col_absmax_kernel<T>, kWarps * 32, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t target = (int64_t)num_sms() * per_sm;
    int64_t bands = target / col_blocks;
    if (bands < 1) bands = 1;
    int64_t rpb = (M + bands - 1) / bands;
    rpb = ((rpb + kWarps - 1) / kWarps) * kWarps;
    if (rpb < 2 * kWarps) rpb = 2 * kWarps;
    const int64_t row_blocks = (M + rpb - 1) / rpb;
    SQ_REQUIRE(row_blocks <= 65535, SQ_ERR_UNSUPPORTED_SHAPE, "%s: too many rows (M=%lld)", name, (long long)M);
    dim3 grid((unsigned)col_blocks, (unsigned)row_blocks);
    launch_pdl(col_absmax_kernel<T>, dim3(grid), dim3(kWarps * 32), 0, s, static_cast<const T*>(X), M, K, ld,
               (int)rpb, out);
    return check_launch(name);
}

sq_status_t col_absmax(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ld, float* out,
                       sq_stream_t stream, const char* name) {
    SQ_REQUIRE((X || M == 0) && out, SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(M >= 0 && K > 0 && ld >= K, SQ_ERR_UNSUPPORTED_SHAPE, "%s: bad sizes M=%lld K=%lld ld=%lld",
               name, (long long)M, (long long)K, (long long)ld);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16 || dt == SQ_F32, SQ_ERR_INVALID_ARG, "%s: dtype must be F16, BF16 or F32",
               name);
    const int v = dt == SQ_F32 ? 4 : 8;
    SQ_REQUIRE(K % v == 0 && ld % v == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K and ld must be multiples of %d", name, v);
    SQ_REQUIRE(aligned16(X), SQ_ERR_ALIGNMENT, "%s: input not 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    cudaStream_t s = as_cuda(stream);
    switch (dt) {
        case SQ_F16: return launch<__half>(X, M, K, ld, out, s, name);
        case SQ_BF16: return launch<__nv_bfloat16>(X, M, K, ld, out, s, name);
        default: return launch<float>(X, M, K, ld, out, s, name);
    }
}

}  // namespace
}  // namespace sq

extern "C" {

sq_status_t sq_calib_absmax(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                            float* xmax_inout, sq_stream_t stream) {
    return sq::col_absmax(X, dt, M, K, ldx, xmax_inout, stream, "sq_calib_absmax");
}

sq_status_t sq_weight_absmax(const void* W, sq_dtype_t dt, int64_t N, int64_t K, int64_t ldw,
                             float* wmax_inout, sq_stream_t stream) {
    return sq::col_absmax(W, dt, N, K, ldw, wmax_inout, stream, "sq_weight_absmax");
}

}  // extern "C"

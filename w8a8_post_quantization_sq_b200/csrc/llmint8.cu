// The LLM.int8() mixed-precision decomposition
// ("8位量化：异常值与混合精度分解实战" §2.2 split_outliers / mixed_precision_matmul,
// §2.3 threshold 6.0, §4.1 any value over the threshold marks its dimension).
//
//   O = { j : count_i(|X_ij| > threshold) / M > min_ratio }, ascending;
//   the columns of X in O take a 16-bit product with the matching input
//   channels of W; the other columns take the vector-wise int8 path (row
//   scales for X, per-output-channel scales for W over the channels not in O);
//   the two results are summed.
//
// Kernels:
//   detect_kernel     one pass over X; a block owns 256 columns x 128 rows and
//                     writes its per-column counts to its own slot of the
//                     workspace. The last block of each 256-column group to
//                     finish (an atomic count per group) adds the group's
//                     slots, applies the ratio test in fp64 and writes the
//                     group's 256-bit outlier mask; the last group to finish
//                     writes O in ascending order with a block-wide prefix sum
//                     over the masks, and compares O with the set the cached
//                     int8 weight was built for, updating that record. Each
//                     block that completes a count sets it back to zero, so
//                     the counters are zero between calls;
//   masked_quant_kernel  row-wise absmax int8 over the columns not in O (used
//                     for the rows of X and for the output channels of W; the
//                     weight pass returns at once when O is unchanged);
//   the tcgen05 GEMM, whose epilogue adds the 16-bit outlier term.
// Nothing here synchronises with the host, so a whole call can be captured in
// a CUDA graph.
#include <cuda.h>

#include <mutex>
#include <type_traits>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {

static size_t r256(size_t b) { return (b + 255) / 256 * 256; }

// Detection scratch: the 256-byte header (word 0 status, word 1 "O changed",
// word 2 the count of finished column groups), one arrival counter per
// 256-column group, the groups' outlier masks (8 words each), then the
// per-band column counts [row bands, K]. The arrival counters take room for
// the widest rows any call takes (K <= 2^20: 4096 groups), so they sit at the
// same bytes whatever K a call has: a call that leaves them at zero leaves a
// workspace ready for any later call, while the masks and counts a call
// leaves behind (written before they are read) never land where a later
// call with more columns expects a zero counter.
constexpr int64_t kMaxDetectK = int64_t(1) << 20;
static int64_t col_groups(int64_t K) { return (K + 255) / 256; }
static size_t detect_done_off() { return kStatusBytes; }
static size_t detect_mask_off(int64_t) { return detect_done_off() + (size_t)col_groups(kMaxDetectK) * 4; }
static size_t detect_count_off(int64_t K) { return detect_mask_off(K) + r256((size_t)col_groups(K) * 32); }

size_t detect_workspace_bytes(int64_t M, int64_t K) {
    const int64_t rb = (M + kDetectRows - 1) / kDetectRows;
    const size_t counts = (size_t)(rb > 0 ? rb : 1) * (size_t)K * sizeof(int32_t);
    return detect_count_off(K) + r256(counts);
}
static int64_t wo_ld_of(int64_t N) { return (N + 255) / 256 * 256; }

// header + counts | Xq [M,K] int8 | qs_x [M] fp32 | X_O [cap, M] fp32 (o-major) | W_O [cap, N256] fp32
size_t llmint8_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    return detect_workspace_bytes(M, K) + r256((size_t)M * (size_t)K) + r256((size_t)M * 4) +
           r256((size_t)M * kOutlierCap * 4) + r256((size_t)kOutlierCap * (size_t)wo_ld_of(N) * 4);
}

namespace {

constexpr int kWarps = 8;

// Per-column counts of |x| > thr over a 128-row band, then (in the last block
// of each column group, and of the grid) the outlier set. `done` holds one
// arrival counter per column group, `gdone` the count of finished groups;
// both are zero when the kernel starts and when it ends.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
detect_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t ld, float thr, double min_ratio,
              int32_t* __restrict__ partial, uint32_t* __restrict__ done, uint32_t* __restrict__ masks,
              uint32_t* __restrict__ gdone, int32_t* __restrict__ idx, int32_t* __restrict__ n_out,
              int32_t* __restrict__ cached_idx, int32_t* __restrict__ cached_n, int32_t* __restrict__ changed) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t red[kWarps][256];
    __shared__ int32_t warp_tot[kWarps];
    __shared__ int32_t flag_sh;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t rb = gridDim.y;
    const int64_t c0 = (int64_t)blockIdx.x * 256 + lane * 8;
    const int64_t r0 = (int64_t)blockIdx.y * kDetectRows;
    const int64_t r1 = min(M, r0 + kDetectRows);
    int32_t cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c0 < K) {
        // the warp's rows of the band (kDetectRows / kWarps of them), all
        // loads issued before any is used
        constexpr int RW = kDetectRows / kWarps;
        uint4 v[RW];
#pragma unroll
        for (int u = 0; u < RW; ++u) {
            const int64_t r = r0 + warp + (int64_t)u * kWarps;
            if (r < r1) v[u] = ldg_nc_v4(X + r * ld + c0);
        }
#pragma unroll
        for (int u = 0; u < RW; ++u) {
            const int64_t r = r0 + warp + (int64_t)u * kWarps;
            if (r < r1) {
                float f[8];
                unpack<T>(v[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) cnt[e] += fabsf(f[e]) > thr ? 1 : 0;
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = cnt[e];
    __syncwarp();  // lanes may have diverged above; bar.sync needs whole warps
    __syncthreads();
    const int64_t col = (int64_t)blockIdx.x * 256 + t;  // kWarps * 32 == 256: one column per thread
    {
        int32_t s = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][t];
        if (col < K) partial[(int64_t)blockIdx.y * K + col] = s;
    }
    // the last band of this column group to arrive adds the group's counts
    __threadfence();
    __syncthreads();
    if (t == 0) flag_sh = atomicAdd(done + blockIdx.x, 1u) == (uint32_t)(rb - 1);
    __syncthreads();
    if (!flag_sh) return;
    __threadfence();
    bool flag = false;
    if (col < K) {
        // the band counts of this column, eight loads in flight at a time
        int64_t total = 0;
        int64_t b = 0;
        for (; b + 8 <= rb; b += 8) {
            int32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldcg(partial + (b + u) * K + col);
#pragma unroll
            for (int u = 0; u < 8; ++u) total += v[u];
        }
        for (; b < rb; ++b) total += __ldcg(partial + b * K + col);
        // an empty column has ratio 0, never above min_ratio >= 0
        if (total > 0) {
            const double ratio = M > 0 ? __ddiv_rn((double)total, (double)M) : 0.0;
            flag = ratio > min_ratio;
        }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) masks[blockIdx.x * 8 + warp] = bal;
    if (t == 0) done[blockIdx.x] = 0u;  // ready for the next call
    // the last column group to finish writes O
    __threadfence();
    __syncthreads();
    if (t == 0) flag_sh = atomicAdd(gdone, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!flag_sh) return;
    __threadfence();
    const int64_t words = (int64_t)gridDim.x * 8;
    int base = 0;
    for (int64_t w0 = 0; w0 < words; w0 += 256) {
        const int64_t w = w0 + t;
        const uint32_t bits = w < words ? __ldcg(masks + w) : 0u;
        const int c = __popc(bits);
        // exclusive prefix of c over the block, in word order
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncwarp();
        __syncthreads();
        int before = base + incl - c;
        int total = 0;
#pragma unroll
        for (int q = 0; q < kWarps; ++q) {
            if (q < warp) before += warp_tot[q];
            total += warp_tot[q];
        }
        uint32_t rest = bits;
        while (rest) {
            const int bpos = __ffs(rest) - 1;
            idx[before++] = (int32_t)(w * 32 + bpos);
            rest &= rest - 1u;
        }
        base += total;
        __syncwarp();
        __syncthreads();
    }
    const int n = base;
    if (t == 0) {
        *n_out = n;
        *gdone = 0u;  // ready for the next call
    }
    if (cached_n) {
        __threadfence_block();
        if (t == 0) flag_sh = *cached_n != n;
        __syncthreads();
        if (!flag_sh)
            for (int o = t; o < n; o += kWarps * 32)
                if (cached_idx[o] != idx[o]) flag_sh = 1;
        __syncwarp();
        __syncthreads();
        const int d = flag_sh;
        if (d) {
            for (int o = t; o < n; o += kWarps * 32) cached_idx[o] = idx[o];
            if (t == 0) *cached_n = n;
        }
        if (t == 0) *changed = d;
    }
}

// One row-quantisation job of the masked kernels: row-wise int8 over the
// columns not in O (zeros in O) of a [rows, K] 16-bit matrix, with the fp32
// copy of its outlier columns (o-major, xo[o * xo_ld + row]) when xo is
// given. When only_if is given and *only_if == 0 the job does nothing.
struct MQJob {
    const void* X;
    int64_t rows, ld;
    int8_t* Q;
    float* qs;
    float* xo;
    int64_t xo_ld;
    const int32_t* only_if;
};

// A launch runs up to two jobs (the rows of X and the weight's output
// channels of one LLM.int8 call): blocks [0, split) take job 0, the rest job
// 1. Builds the outlier bit mask in shared memory; returns false when the
// block's job has nothing to do.
__device__ __forceinline__ bool mq_setup(const MQJob& j0, const MQJob& j1, int split, int64_t K,
                                         const int32_t* __restrict__ idx, const int32_t* __restrict__ n_idx,
                                         uint32_t* mask, MQJob& job, int64_t& b0, int64_t& nb, int& n) {
    const bool second = (int)blockIdx.x >= split;
    job = second ? j1 : j0;
    b0 = second ? (int64_t)blockIdx.x - split : (int64_t)blockIdx.x;
    nb = second ? (int64_t)gridDim.x - split : (int64_t)split;
    if (job.only_if && *job.only_if == 0) return false;  // block-uniform
    const int64_t words = (K + 31) / 32;
    for (int64_t w = threadIdx.x; w < words; w += blockDim.x) mask[w] = 0u;
    __syncwarp();
    __syncthreads();
    n = *n_idx;
    for (int o = threadIdx.x; o < n; o += blockDim.x) {
        const int j = idx[o];
        atomicOr(&mask[j >> 5], 1u << (j & 31));
    }
    __syncwarp();
    __syncthreads();
    return true;
}

template <typename T>
__device__ __forceinline__ void write_xo(const MQJob& job, const T* x, int64_t row, const int32_t* idx, int n,
                                         int lane) {
    if (job.xo)  // fp32 copy of the outlier columns of this row, for the GEMM epilogue
        for (int o = lane; o < n && o < kOutlierCap; o += 32) {
            const uint16_t u = reinterpret_cast<const uint16_t*>(x)[idx[o]];
            float f[8];
            unpack<T>(make_uint4(u, 0, 0, 0), f);
            job.xo[(int64_t)o * job.xo_ld + row] = f[0];
        }
}

// One warp per row, the row read twice (any K).
template <typename T>
__global__ void __launch_bounds__(256)
masked_quant_kernel(MQJob j0, MQJob j1, int split, int64_t K, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ n_idx) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];  // K bits
    MQJob job;
    int64_t b0, nb;
    int n = 0;
    if (!mq_setup(j0, j1, split, K, idx, n_idx, mask, job, b0, nb, n)) return;
    const T* X = static_cast<const T*>(job.X);
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = nb * (blockDim.x >> 5);
    for (int64_t row = (b0 * blockDim.x + threadIdx.x) >> 5; row < job.rows; row += nwarps) {
        const T* x = X + row * job.ld;
        float m = 0.0f;
#pragma unroll 4
        for (int64_t k0 = lane * 8; k0 < K; k0 += 256) {
            float f[8];
            unpack<T>(ldg_v4(x + k0), f);
            const uint32_t bits = (mask[k0 >> 5] >> (k0 & 31)) & 0xffu;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (!((bits >> e) & 1u)) m = fmaxf(m, fabsf(f[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float qs = __fdiv_rn(127.0f, fmaxf(m, 1e-8f));
        if (lane == 0) job.qs[row] = qs;
        write_xo<T>(job, x, row, idx, n, lane);
        int8_t* q = job.Q + row * K;
#pragma unroll 4
        for (int64_t k0 = lane * 8; k0 < K; k0 += 256) {
            float f[8];
            unpack<T>(ldg_v4(x + k0), f);
            const uint32_t bits = (mask[k0 >> 5] >> (k0 & 31)) & 0xffu;
            uint32_t c[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) c[e] = ((bits >> e) & 1u) ? 0u : quant_bits_noclip(__fmul_rn(f[e], qs));
            *reinterpret_cast<uint2*>(q + k0) =
                make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]), pack_low_bytes(c[4], c[5], c[6], c[7]));
        }
    }
}

// The same with the row in registers (K <= 256 * CH): one read of X. Lane l
// holds chunks l, l + 32, ... of 8 columns.
template <typename T, int CH>
__global__ void __launch_bounds__(256)
masked_quant_reg_kernel(MQJob j0, MQJob j1, int split, int64_t K, const int32_t* __restrict__ idx,
                        const int32_t* __restrict__ n_idx) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];  // K bits
    MQJob job;
    int64_t b0, nb;
    int n = 0;
    if (!mq_setup(j0, j1, split, K, idx, n_idx, mask, job, b0, nb, n)) return;
    const T* X = static_cast<const T*>(job.X);
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = nb * (blockDim.x >> 5);
    for (int64_t row = (b0 * blockDim.x + threadIdx.x) >> 5; row < job.rows; row += nwarps) {
        const T* x = X + row * job.ld;
        uint4 raw[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int64_t k0 = (int64_t)lane * 8 + 256 * i;
            if (k0 < K) raw[i] = ldg_nc_v4(x + k0);
        }
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int64_t k0 = (int64_t)lane * 8 + 256 * i;
            if (k0 < K) {
                float f[8];
                unpack<T>(raw[i], f);
                const uint32_t bits = (mask[k0 >> 5] >> (k0 & 31)) & 0xffu;
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, ((bits >> e) & 1u) ? 0.0f : fabsf(f[e]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float qs = __fdiv_rn(127.0f, fmaxf(m, 1e-8f));
        if (lane == 0) job.qs[row] = qs;
        write_xo<T>(job, x, row, idx, n, lane);
        int8_t* q = job.Q + row * K;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int64_t k0 = (int64_t)lane * 8 + 256 * i;
            if (k0 < K) {
                float f[8];
                unpack<T>(raw[i], f);
                const uint32_t bits = (mask[k0 >> 5] >> (k0 & 31)) & 0xffu;
                uint32_t c[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    c[e] = ((bits >> e) & 1u) ? 0u : quant_bits_noclip(__fmul_rn(f[e], qs));
                *reinterpret_cast<uint2*>(q + k0) =
                    make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]), pack_low_bytes(c[4], c[5], c[6], c[7]));
            }
        }
    }
}

// W_O[o, j] = W[j, idx[o]] for o < min(n, cap), j < N; zero for N <= j < ld.
// When `only_if` is given and *only_if == 0 the kernel does nothing.
template <typename T>
__global__ void gather_wo_kernel(const T* __restrict__ W, int64_t N, int64_t K, const int32_t* __restrict__ idx,
                                 const int32_t* __restrict__ n_idx, const int32_t* __restrict__ only_if,
                                 float* __restrict__ wo, int64_t ld) {
    pdl_wait();
    pdl_trigger();
    if (only_if && *only_if == 0) return;
    const int n = min(*n_idx, kOutlierCap);
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < ld; j += (int64_t)gridDim.x * blockDim.x)
        for (int o = 0; o < n; ++o) {
            float v = 0.0f;
            if (j < N) {
                const uint16_t u = reinterpret_cast<const uint16_t*>(W)[j * K + idx[o]];
                float f[8];
                unpack<T>(make_uint4(u, 0, 0, 0), f);
                v = f[0];
            }
            wo[(int64_t)o * ld + j] = v;
        }
}

sq_status_t launch_detect(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx, float thr,
                          double min_ratio, int32_t* idx, int32_t* n_out, int32_t* cached_idx, int32_t* cached_n,
                          void* ws, cudaStream_t s) {
    char* wsb = static_cast<char*>(ws);
    int32_t* changed = reinterpret_cast<int32_t*>(wsb + 4);
    uint32_t* gdone = reinterpret_cast<uint32_t*>(wsb + 8);
    uint32_t* done = reinterpret_cast<uint32_t*>(wsb + detect_done_off());
    uint32_t* masks = reinterpret_cast<uint32_t*>(wsb + detect_mask_off(K));
    int32_t* partial = reinterpret_cast<int32_t*>(wsb + detect_count_off(K));
    int64_t rb = (M + kDetectRows - 1) / kDetectRows;
    if (rb < 1) rb = 1;  // M == 0: one band with no rows, so O is empty
    SQ_REQUIRE(rb <= 65535, SQ_ERR_UNSUPPORTED_SHAPE, "sq_llmint8_detect: M too large");
    SQ_REQUIRE(K <= kMaxDetectK, SQ_ERR_UNSUPPORTED_SHAPE, "sq_llmint8_detect: K too large");
    dim3 grid((unsigned)col_groups(K), (unsigned)rb);
    if (dt == SQ_BF16)
        launch_pdl(detect_kernel<__nv_bfloat16>, grid, dim3(kWarps * 32), 0, s, static_cast<const __nv_bfloat16*>(X), M,
                   K, ldx, thr, min_ratio, partial, done, masks, gdone, idx, n_out, cached_idx, cached_n, changed);
    else
        launch_pdl(detect_kernel<__half>, grid, dim3(kWarps * 32), 0, s, static_cast<const __half*>(X), M, K, ldx, thr,
                   min_ratio, partial, done, masks, gdone, idx, n_out, cached_idx, cached_n, changed);
    return check_launch("sq_llmint8_detect");
}

// Blocks for one job: one warp per row, 8 warps per block, capped; a
// conditional (weight-side) job usually returns at once, so it gets fewer.
int64_t mq_blocks(const MQJob& j) {
    int64_t grid = (j.rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * (j.only_if ? 2 : 8);
    return grid > cap ? cap : grid;
}

// Launch the masked row quantisation for one job, or two in one launch.
sq_status_t launch_masked_quant(sq_dtype_t dt, int64_t K, const int32_t* idx, const int32_t* n_idx, const MQJob& j0,
                                const MQJob* j1, cudaStream_t s, const char* name) {
    const size_t smem = (size_t)((K + 31) / 32) * 4;
    const int64_t g0 = j0.rows > 0 ? mq_blocks(j0) : 0;
    const int64_t g1 = (j1 && j1->rows > 0) ? mq_blocks(*j1) : 0;
    if (g0 + g1 < 1) return SQ_OK;
    const MQJob second = (j1 && j1->rows > 0) ? *j1 : j0;
    auto go = [&](auto k) {
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(k, dim3((unsigned)(g0 + g1)), dim3(256), smem, s, j0, second, (int)g0, K, idx, n_idx);
    };
    auto pick = [&](auto* tag) {
        using T = std::remove_pointer_t<decltype(tag)>;
        if (K <= 256) go(masked_quant_reg_kernel<T, 1>);
        else if (K <= 512) go(masked_quant_reg_kernel<T, 2>);
        else if (K <= 1024) go(masked_quant_reg_kernel<T, 4>);
        else if (K <= 2048) go(masked_quant_reg_kernel<T, 8>);
        else if (K <= 4096) go(masked_quant_reg_kernel<T, 16>);
        else go(masked_quant_kernel<T>);
    };
    if (dt == SQ_BF16) pick(static_cast<__nv_bfloat16*>(nullptr));
    else pick(static_cast<__half*>(nullptr));
    return check_launch(name);
}

MQJob mq_job(const void* X, int64_t rows, int64_t ld, int8_t* Q, float* qs, float* xo = nullptr, int64_t xo_ld = 0,
             const int32_t* only_if = nullptr) {
    return MQJob{X, rows, ld, Q, qs, xo, xo_ld, only_if};
}

sq_status_t check_x(const char* name, const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx) {
    SQ_REQUIRE(X || M == 0, SQ_ERR_INVALID_ARG, "%s: null input", name);
    SQ_REQUIRE(dt == SQ_F16 || dt == SQ_BF16, SQ_ERR_INVALID_ARG, "%s: dtype must be F16 or BF16", name);
    SQ_REQUIRE(M >= 0 && K > 0 && ldx >= K && K % 8 == 0 && ldx % 8 == 0, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: need K > 0, K %% 8 == 0, ldx >= K, ldx %% 8 == 0", name);
    SQ_REQUIRE(K <= kMaxDetectK, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K too large", name);
    SQ_REQUIRE(aligned16(X), SQ_ERR_ALIGNMENT, "%s: input not 16-byte aligned", name);
    return SQ_OK;
}

}  // namespace
}  // namespace sq

extern "C" {

sq_status_t sq_llmint8_detect(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx, float threshold,
                              double min_ratio, int32_t* outlier_idx, int32_t* n_outliers, void* workspace,
                              size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_llmint8_detect";
    sq_status_t st = sq::check_x(name, X, dt, M, K, ldx);
    if (st != SQ_OK) return st;
    SQ_REQUIRE(outlier_idx && n_outliers, SQ_ERR_INVALID_ARG, "%s: null output", name);
    SQ_REQUIRE(min_ratio >= 0.0 && threshold >= 0.0f, SQ_ERR_INVALID_ARG, "%s: threshold and min_ratio must be >= 0",
               name);
    SQ_REQUIRE(workspace && ws_bytes >= sq::detect_workspace_bytes(M, K), SQ_ERR_INVALID_ARG,
               "%s: needs a workspace of %zu bytes", name, sq::detect_workspace_bytes(M, K));
    return sq::launch_detect(X, dt, M, K, ldx, threshold, min_ratio, outlier_idx, n_outliers, nullptr, nullptr,
                             workspace, sq::as_cuda(stream));
}

sq_status_t sq_llmint8_quant_rows(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                                  const int32_t* idx, const int32_t* n_idx, int8_t* Xq, float* qs_x,
                                  sq_stream_t stream) {
    const char* name = "sq_llmint8_quant_rows";
    sq_status_t st = sq::check_x(name, X, dt, M, K, ldx);
    if (st != SQ_OK) return st;
    SQ_REQUIRE(idx && n_idx && ((Xq && qs_x) || M == 0), SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(sq::aligned16(Xq), SQ_ERR_ALIGNMENT, "%s: Xq not 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    return sq::launch_masked_quant(dt, K, idx, n_idx, sq::mq_job(X, M, ldx, Xq, qs_x), nullptr, sq::as_cuda(stream),
                                   name);
}

sq_status_t sq_llmint8_quant_weight(const void* W, sq_dtype_t dt, int64_t N, int64_t K, const int32_t* idx,
                                    const int32_t* n_idx, int8_t* Wq, float* qs_w, sq_stream_t stream) {
    const char* name = "sq_llmint8_quant_weight";
    sq_status_t st = sq::check_x(name, W, dt, N, K, K);
    if (st != SQ_OK) return st;
    SQ_REQUIRE(idx && n_idx && ((Wq && qs_w) || N == 0), SQ_ERR_INVALID_ARG, "%s: null pointer", name);
    SQ_REQUIRE(sq::aligned16(Wq), SQ_ERR_ALIGNMENT, "%s: Wq not 16-byte aligned", name);
    if (N == 0) return SQ_OK;
    return sq::launch_masked_quant(dt, K, idx, n_idx, sq::mq_job(W, N, K, Wq, qs_w), nullptr, sq::as_cuda(stream),
                                   name);
}

sq_status_t sq_llmint8_matmul(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                              const sq_llmint8_weight_t* w, float threshold, double min_ratio, void* Y, int64_t ldy,
                              int32_t* idx_out, int32_t* n_out, void* workspace, size_t ws_bytes,
                              sq_stream_t stream) {
    const char* name = "sq_llmint8_matmul";
    sq_status_t st = sq::check_x(name, X, dt, M, K, ldx);
    if (st != SQ_OK) return st;
    SQ_REQUIRE(w && w->W && w->Wq && w->qs_w && w->cached_idx && w->cached_n, SQ_ERR_INVALID_ARG,
               "%s: incomplete weight state", name);
    SQ_REQUIRE((Y || M == 0) && idx_out && n_out, SQ_ERR_INVALID_ARG, "%s: null output", name);
    SQ_REQUIRE(w->N > 0 && ldy >= w->N, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need N > 0 and ldy >= N", name);
    SQ_REQUIRE(K % 16 == 0 && K <= 133144, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be a multiple of 16, <= 133144",
               name);
    SQ_REQUIRE(M < (1ll << 31) && w->N < (1ll << 31), SQ_ERR_UNSUPPORTED_SHAPE, "%s: M and N must be < 2^31", name);
    SQ_REQUIRE(sq::aligned16(w->W) && sq::aligned16(w->Wq), SQ_ERR_ALIGNMENT, "%s: weights not 16-byte aligned", name);
    const size_t need = sq::llmint8_workspace_bytes(M, w->N, K);
    SQ_REQUIRE(workspace && ws_bytes >= need, SQ_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes", name, need);
    cudaStream_t s = sq::as_cuda(stream);
    char* wsb = static_cast<char*>(workspace);
    const size_t det = sq::detect_workspace_bytes(M, K);
    size_t off = det;
    int8_t* Xq = reinterpret_cast<int8_t*>(wsb + off);
    off += sq::r256((size_t)M * K);
    float* qs_x = reinterpret_cast<float*>(wsb + off);
    off += sq::r256((size_t)M * 4);
    float* xo = reinterpret_cast<float*>(wsb + off);
    off += sq::r256((size_t)M * sq::kOutlierCap * 4);
    float* wo = reinterpret_cast<float*>(wsb + off);
    const int64_t wo_ld = sq::wo_ld_of(w->N);
    int32_t* changed = reinterpret_cast<int32_t*>(wsb + 4);
    // the outlier set O, and whether the cached int8 weight was built for it
    st = sq::launch_detect(X, dt, M, K, ldx, threshold, min_ratio, idx_out, n_out, w->cached_idx, w->cached_n, workspace,
                           s);
    if (st != SQ_OK) return st;
    // one launch: the row quantisation outside O (and the fp32 copy of the
    // outlier columns of X), and the weight side for O, whose blocks return
    // at once when O is unchanged; with a W_O buffer in the weight state the
    // weight side refreshes it too (wo[o, n] is W[n, O_o], o-major like X_O)
    const sq::MQJob wjob = sq::mq_job(w->W, w->N, K, w->Wq, w->qs_w, w->wo, wo_ld, changed);
    st = sq::launch_masked_quant(dt, K, idx_out, n_out, sq::mq_job(X, M, ldx, Xq, qs_x, xo, M), &wjob, s, name);
    if (st != SQ_OK) return st;
    if (M == 0) return SQ_OK;
    // without a W_O buffer in the weight state: gather W_O into the workspace
    if (w->wo) {
        wo = w->wo;
    } else {
        const int32_t* only_if = nullptr;
        int64_t blocks = (wo_ld + 255) / 256;
        if (blocks > (int64_t)sq::num_sms() * 4) blocks = (int64_t)sq::num_sms() * 4;
        if (dt == SQ_BF16)
            sq::launch_pdl(sq::gather_wo_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(256), 0, s,
                           static_cast<const __nv_bfloat16*>(w->W), w->N, K, idx_out, n_out, only_if, wo, wo_ld);
        else
            sq::launch_pdl(sq::gather_wo_kernel<__half>, dim3((unsigned)blocks), dim3(256), 0, s,
                           static_cast<const __half*>(w->W), w->N, K, idx_out, n_out, only_if, wo, wo_ld);
        st = sq::check_launch(name);
        if (st != SQ_OK) return st;
    }
    // int8 GEMM + 16-bit outlier term in the epilogue
    sq::GemmEpilogue ep;
    ep.qs_x = qs_x;
    ep.x_per_token = 1;
    ep.qs_w = w->qs_w;
    ep.w_per_channel = 1;
    ep.out_dt = dt;
    ep.Y = Y;
    ep.ldy = ldy;
    ep.x16 = X;
    ep.ldx16 = ldx;
    ep.w16 = w->W;
    ep.idx = idx_out;
    ep.n_out = n_out;
    ep.in16_bf16 = dt == SQ_BF16;
    ep.xo = xo;
    ep.wo = wo;
    ep.wo_ld = wo_ld;
    // the workspace past its header holds the decomposition's own buffers: no stream-K scratch
    return sq::launch_gemm_w8a8(Xq, w->Wq, M, w->N, K, ep, static_cast<int*>(workspace), sq::kStatusBytes, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// sq_llmint8_detect_noalloc: the same detection for callers that cannot hand
// the library any scratch memory. Its scratch (the 256-byte header plus the
// per-band column counts) is this file-scope device array; each device that
// loads the library holds one copy until the process exits.
namespace sq {
namespace {

constexpr size_t kDetectScratchBytes = size_t(4) << 20;  // 4 MiB
__device__ __align__(256) unsigned char g_detect_scratch[kDetectScratchBytes];

// Device addresses of g_detect_scratch, one per CUDA context: the array's
// name is only a host-side stand-in, and each context that loads the
// library's module has its own copy of it. Keyed by the context's unique id
// (cuCtxGetId), which a context created later never reuses, even when it
// gets the same handle (the primary context after cudaDeviceReset).
constexpr int kMaxContexts = 64;
std::mutex g_scratch_mu;
unsigned long long g_scratch_ctx[kMaxContexts] = {};
void* g_scratch_addr[kMaxContexts] = {};
int g_scratch_n = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}

sq_status_t detect_scratch(void** out) {
    static CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_cur || !get_id)
        return set_error(SQ_ERR_CUDA, "sq_llmint8_detect_noalloc: cuCtxGetCurrent / cuCtxGetId unavailable");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    void* p = nullptr;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) {
        // no context current on this thread yet: the symbol lookup
        // initialises the runtime's (primary) context and makes it current
        const cudaError_t e = cudaGetSymbolAddress(&p, g_detect_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(SQ_ERR_CUDA, "sq_llmint8_detect_noalloc: cudaGetSymbolAddress: %s",
                             cudaGetErrorString(e));
        if (get_cur(&ctx) != CUDA_SUCCESS || !ctx)
            return set_error(SQ_ERR_CUDA, "sq_llmint8_detect_noalloc: no current CUDA context");
    }
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS)
        return set_error(SQ_ERR_CUDA, "sq_llmint8_detect_noalloc: cannot identify the current CUDA context");
    for (int i = 0; i < g_scratch_n; ++i)
        if (g_scratch_ctx[i] == id) {
            *out = g_scratch_addr[i];
            return SQ_OK;
        }
    if (!p) {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_detect_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(SQ_ERR_CUDA, "sq_llmint8_detect_noalloc: cudaGetSymbolAddress: %s",
                             cudaGetErrorString(e));
    }
    // a full table forgets the oldest context (it only costs a new lookup)
    const int slot = g_scratch_n < kMaxContexts ? g_scratch_n++ : (int)(id % kMaxContexts);
    g_scratch_ctx[slot] = id;
    g_scratch_addr[slot] = p;
    *out = p;
    return SQ_OK;
}

}  // namespace
}  // namespace sq

extern "C" sq_status_t sq_llmint8_detect_noalloc(const void* X, sq_dtype_t dt, int64_t M, int64_t K, int64_t ldx,
                                                 float threshold, double min_ratio, int32_t* outlier_idx,
                                                 int32_t* n_outliers, sq_stream_t stream) {
    const char* name = "sq_llmint8_detect_noalloc";
    sq_status_t st = sq::check_x(name, X, dt, M, K, ldx);
    if (st != SQ_OK) return st;
    SQ_REQUIRE(outlier_idx && n_outliers, SQ_ERR_INVALID_ARG, "%s: null output", name);
    SQ_REQUIRE(min_ratio >= 0.0 && threshold >= 0.0f, SQ_ERR_INVALID_ARG, "%s: threshold and min_ratio must be >= 0",
               name);
    const size_t need = sq::detect_workspace_bytes(M, K);
    SQ_REQUIRE(need <= sq::kDetectScratchBytes, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: ceil(M/%d) * K = %lld counts need %zu bytes of scratch, more than its fixed %zu bytes; "
               "use sq_llmint8_detect with a workspace",
               name, sq::kDetectRows, (long long)(((M + sq::kDetectRows - 1) / sq::kDetectRows) * K), need,
               sq::kDetectScratchBytes);
    void* scratch = nullptr;
    st = sq::detect_scratch(&scratch);
    if (st != SQ_OK) return st;
    // the arrival counters must start at zero: a completed call leaves them
    // at zero, and they are cleared here too (a memset, no allocation); the
    // counts and masks are written before they are read
    if (cudaMemsetAsync(scratch, 0, sq::detect_mask_off(K), sq::as_cuda(stream)) != cudaSuccess)
        return sq::check_launch("sq_llmint8_detect_noalloc: clearing the counters");
    return sq::launch_detect(X, dt, M, K, ldx, threshold, min_ratio, outlier_idx, n_outliers, nullptr, nullptr,
                             scratch, sq::as_cuda(stream));
}

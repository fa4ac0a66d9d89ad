// INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor cores with a
// dequantising epilogue, and the LLM.int8 16-bit outlier term fused into
// the same epilogue.
//
// What it computes ("8位量化：异常值与混合精度分解实战" §2.1; "大语言模型量化技术
// （四）：SmoothQuant", 为什么激活不能用逐通道量化):
//   acc[i,j] = sum_k Xq[i,k] * Wq[j,k]            exact in int32
//   Y[i,j]   = acc * ((1/qs_x[i]) * (1/qs_w[j])) (+ h[i,j]) (+ bias[j])
// where h is the outlier term sum_{o in O} X16[i,o] * W16[j,o] of §2.2,
// added to the dequantised value by fp32 fma in ascending o (the 16-bit
// products are exact in fp32).
//
// Design (sm_100a):
//   - persistent: one 320-thread CTA per SM loops over 128 x BN output tiles
//     in a grouped raster (the CTAs running together share Xq rows and weight
//     tiles in L2); when the last wave of whole tiles would be mostly idle,
//     that wave's tiles are cut by k-blocks into one range per CTA, run
//     before the whole tiles (stream-K, see plan_gemm);
//   - warp 0 (one lane) issues TMA loads of 128 x 128 int8 tiles of Xq and
//     BN x 128 tiles of Wq (128-byte swizzle) into a 4-stage shared-memory
//     ring guarded by mbarriers;
//   - warp 1 (one lane) issues tcgen05.mma.cta_group::1.kind::i8 (M=128,
//     N=BN, K=32 each, four per stage) into a double-buffered int32
//     accumulator in tensor memory (2 x BN of the 512 columns), and frees
//     ring stages and accumulator buffers with tcgen05.commit;
//   - warps 2..9 read the accumulator with tcgen05.ld (warp w owns TMEM lanes
//     32*(w%4)..+31 = tile rows, and half of the columns), double-buffering
//     the loads, dequantise in fp32, stage 32 x 32 chunks in shared memory
//     and write them out while the next tile's MMAs run in the other
//     accumulator buffer; the buffer is released right after its last load.
//     16-bit outputs with 16-byte aligned rows leave by TMA store (one
//     cp.async.bulk.tensor per chunk from a 64-byte-swizzled staging box,
//     rows and columns past the edge clipped by the copy engine); the
//     others by whole row segments of plain stores.
// Batched variant (lpnh.cn SmoothQuant practice article §2.2: the QK^T and PV
// products of attention can run in int8): problem b of a [batch, M, K] x
// [batch, N, K] pair through 3-D tensor maps, its own row scales (one per
// (head, token) or (head, channel)), Y[b] = Y + b * M * ldy.
// FP8 variant ("SmoothQuant" (newton wiki), 技術原理與特性: INT8 or FP8
// units): the same kernel with tcgen05.mma kind::f8f6f4 on E4M3 operands and
// an fp32 accumulator; the epilogue reads the fp32 sums instead of int32.
// Every wait is bounded (about 2 s of %globaltimer); on expiry the kernel
// records code 0x6E1 + role in the status word, drains its own TMA copies and
// MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "sq_act.cuh"
#include "sq_common.cuh"
#include "sq_internal.h"
#include "sq_wait.cuh"

namespace sq {
namespace {

constexpr int BM = 128;
constexpr int BK = 128;  // one 128-byte swizzle row of int8
constexpr int UMMA_K = 32;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, each on half the tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint64_t kTimeoutNs = 2000000000ull;
// staging: 32 rows x 64 B of data (32 16-bit or 16 32-bit values) + 16 B pad
// for the plain stores; the TMA-store box uses the first 2 KB of the same
// slot unpadded (64-byte swizzle), so slots start on 512-byte boundaries.
// (Two boxes per warp, one filled while the other is read out, measured no
// faster on B200 and need a pair's sixth ring stage.)
constexpr int kStgRow = 80;
constexpr int kStgWarpBytes = 32 * kStgRow;
static_assert(kStgWarpBytes % 512 == 0, "staging slots must keep the 64-byte swizzle's 512-byte alignment");
enum OutKind { kOutBF16 = 0, kOutF16 = 1, kOutF32 = 2, kOutI32 = 3 };
// activation applied to the 16-bit output in the epilogue (sq_gemm_w8a8_act):
// none, or the sq_act_t value (SwiGLU on interleaved gate/up columns, ReLU, GELU)
constexpr int kActNone = -1;
// operand formats: int8 x int8 -> int32, or FP8 E4M3 x E4M3 -> fp32
enum MmaKind { kKindI8 = 0, kKindF8 = 1 };

// CG = 1: one CTA computes a 128 x BN tile with cta_group::1 MMAs.
// CG = 2: a cluster of two CTAs computes a 256 x BN tile with cta_group::2
// MMAs issued by CTA 0: each CTA loads its own 128 rows of Xq and its own
// BN/2 rows of the weight tile, and holds its 128 rows x BN of the
// accumulator, so each SM streams half as many weight bytes per MMA.
template <int BN, int CG>
struct Cfg {
    static constexpr int STAGES = CG == 2 ? 6 : 4;
    static constexpr uint32_t A_BYTES = BM * BK;         // this CTA's 128 rows of Xq
    static constexpr uint32_t B_BYTES = (BN / CG) * BK;  // this CTA's rows of the weight tile
    static constexpr uint32_t A_OFF = 0;
    static constexpr uint32_t B_OFF = STAGES * A_BYTES;
    static constexpr uint32_t BAR_OFF = B_OFF + STAGES * B_BYTES;
    // full[S], empty[S], tfull[2], tempty[2], drain
    static constexpr uint32_t NBAR = 2 * STAGES + 5;
    static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base, abort flag
    // per epilogue warp: 1/qs_w and bias of the tile's columns
    static constexpr uint32_t RW_OFF = (MISC_OFF + 16 + 15) / 16 * 16;
    static constexpr uint32_t RW_BYTES = kEpiWarps * 2 * (BN / 2) * 4;
    // per epilogue warp: a 32 x 32 output chunk (rows padded to avoid bank conflicts)
    static constexpr uint32_t STG_OFF = (RW_OFF + RW_BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t STG_BYTES = kEpiWarps * kStgWarpBytes;
    static constexpr uint32_t SMEM = STG_OFF + STG_BYTES;
    static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // slack to align the base to 1024
    static_assert(SMEM_ALLOC <= 232448, "over the 227 KB of shared memory a block may use");
    static constexpr uint32_t TMEM_COLS = 2 * BN;
    // kind::i8: D = s32 (bits 4-5 = 2), A = B = signed 8-bit (bits 7-9, 10-12 = 1);
    // kind::f8f6f4: D = f32 (bits 4-5 = 1), A = B = E4M3 (format 0);
    // both K-major, N >> 3 at bit 17, M >> 4 at bit 24 (M = 256 for a CTA pair)
    static constexpr uint32_t idesc(int kind) {
        return (kind == kKindF8 ? (1u << 4) : ((2u << 4) | (1u << 7) | (1u << 10))) |
               ((uint32_t)(BN >> 3) << 17) | ((uint32_t)((BM * CG) >> 4) << 24);
    }
};

struct Params {
    int M, N, K;
    int batch;          // independent problems (heads); 1 for a plain GEMM
    int64_t y_bstride;  // elements between the batches of Y
    int num_m, num_n, num_kb;
    int group_m;    // m-blocks per raster group
    int vec_store;  // Y rows start on 16-byte boundaries
    int tma_store;  // 16-bit Y written by TMA store through the Y tensor map
    GemmEpilogue ep;
    int* status;
    // Stream-K (one problem only): the first dp_tiles tiles in raster order
    // run whole, the CTAs taking them in turn; the k-blocks of the remaining
    // sk_tiles tiles, sk_iters in all, are cut into one contiguous range per
    // CTA.
    int dp_tiles, sk_tiles, sk_iters;
    int sk_units;      // the units the split ranges are dealt to: CTAs, or CTA pairs (grid / CG)
    int sk_cnt_bytes;  // size of the counter region, recorded in header word 3 for sq_workspace_status
    int* sk_cnt;   // [sk_tiles][CG][kEpiWarps] k-blocks counted in per tile region (zero between launches)
    int* sk_part;  // [grid][2][kEpiWarps][NCH][8][32] int4: parked int32 partial sums
};

// First k-iteration of unit c's stream-K range (a unit is a CTA, or a CTA
// pair, which splits as one; every unit gets at least one: sk_iters >= units).
__device__ __forceinline__ int sk_start(int c, const Params& p) {
    return (int)((int64_t)c * p.sk_iters / (int64_t)p.sk_units);
}
// The unit whose range holds k-iteration x.
__device__ __forceinline__ int sk_owner(int x, const Params& p) {
    return (int)((((int64_t)x + 1) * (int64_t)p.sk_units + p.sk_iters - 1) / p.sk_iters - 1);
}

// This CTA's work, the same sequence for its three roles: the pieces of its
// stream-K range first (a piece is the part of the range inside one tile),
// then its whole tiles, so the parking of partial sums and the fix-up
// epilogues overlap the whole tiles' MMAs instead of trailing the launch.
// slot = -1 for a whole tile; a piece is the CTA's first (slot 0) or last
// (slot 1) piece: a range spans at most one whole tile between them. A CTA
// pair (CG = 2) walks the tiles as one unit: both CTAs see the same sequence.
template <bool SK, int CG>
struct Segments {
    int tile_dp, it, end;
    bool first;
    __device__ explicit Segments(const Params& p) {
        tile_dp = blockIdx.x / CG;
        it = SK ? sk_start(blockIdx.x / CG, p) : 0;
        end = SK ? sk_start(blockIdx.x / CG + 1, p) : 0;
        first = true;
    }
    __device__ bool next(const Params& p, int num_tiles, int& tile, int& k0, int& k1, int& slot) {
        if (SK && it < end) {
            const int u = it / p.num_kb;
            k0 = it - u * p.num_kb;
            k1 = min(p.num_kb, k0 + (end - it));
            tile = p.dp_tiles + u;
            slot = (k0 == 0 && k1 == p.num_kb) ? -1 : (first ? 0 : 1);
            first = false;
            it += k1 - k0;
            return true;
        }
        tile = tile_dp;
        k0 = 0;
        k1 = p.num_kb;
        slot = -1;
        tile_dp += gridDim.x / CG;
        return tile < (SK ? p.dp_tiles : num_tiles);
    }
};

// Raster: groups of group_m m-blocks; inside a group, n-major then m. The
// CTAs running together then share the group's rows of Xq (kept in L2) and a
// few weight tiles, and each weight tile is fetched once per group.
__device__ __forceinline__ void tile_coords(int tile, const Params& p, int bm, int bn, int& m0, int& n0) {
    const int per_group = p.group_m * p.num_n;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int gm0 = g * p.group_m;
    const int gsize = min(p.group_m, p.num_m - gm0);
    const int nb = r / gsize;
    m0 = (gm0 + (r - nb * gsize)) * bm;
    n0 = nb * bn;
}

// Batched problems: tile t of problem b = t / (num_m * num_n).
__device__ __forceinline__ void tile_coords_b(int tile, const Params& p, int bm, int bn, int& b, int& m0, int& n0) {
    const int tpb = p.num_m * p.num_n;
    b = tile / tpb;
    tile_coords(tile - b * tpb, p, bm, bn, m0, n0);
}

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// Wait for the phase of `parity` to complete, giving up after kTimeoutNs or
// when another role has aborted (the shared bounded wait of sq_wait.cuh).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                             int code) {
    return wait_bounded_ns(bar, parity, abort_flag, status, code, kTimeoutNs);
}

// The same with the common case inline: one try_wait (which itself suspends
// the thread for a while if the phase is not complete), and the call into the
// bounded loop only when that is not enough. The producer and the MMA issuer
// wait once per k-block; a call per wait sat on their critical path.
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                         int code) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded(bar, parity, abort_flag, status, code);
}

// Short bounded wait used while draining after an abort (ignores the flag).
__device__ __noinline__ void wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kTimeoutNs / 4) return;
}

// Tile (x = k, y = row) of problem z of a 3-D [batch, rows, K] int8 tensor
// into this CTA's shared memory. CG = 2: the completion is counted on the
// mbarrier `bar` names in the shared::cluster window, which may be the other
// CTA's of the pair (no multicast: each CTA loads only its own tile).
template <int CG>
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
    if constexpr (CG == 2) {
        asm volatile(
            "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
            "[%0], [%1, {%3, %4, %5}], [%2];"
            ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
            : "memory");
    } else {
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
            "[%0], [%1, {%3, %4, %5}], [%2];"
            ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
            : "memory");
    }
}


// Store a 32 x 32 box of 16-bit outputs (x = column, y = row, z = problem)
// from this CTA's shared memory; elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// this thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// this thread's bulk stores have completed
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------- CTA pairs
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared::cluster address of this CTA's shared-memory location `a` in
// CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// Every thread of both CTAs arrives, then waits (aligned: whole warps).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (possibly the
// other CTA's), with the arrive's default semantics. It hands an accumulator
// buffer back to the pair's MMA issuer: the tensor-memory reads it orders
// have completed (tcgen05.wait::ld) and are fenced by
// tcgen05.fence::before_thread_sync, and the issuer's wait is followed by
// tcgen05.fence::after_thread_sync. A release at cluster scope would first
// order every earlier memory access of this thread at that scope, a fence per
// tile that showed up as membar stalls (measured on B200: the int8 QK^T
// product at 96 x 2048 x 2048 x 128 took 302 us with it, 264 us without).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// UMMA shared-memory descriptor, K-major operand with 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (SBO), version 1, layout 2.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

template <int KIND, int CG>
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (CG == 2 && KIND == kKindF8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    } else if constexpr (CG == 2) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    } else if constexpr (KIND == kKindF8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    }
}
// Arrive on `bar` once every MMA this thread has issued completes. CG = 2:
// on the mbarrier at the same shared-memory offset in each CTA of `mask`.
template <int CG>
__device__ __forceinline__ void umma_commit(uint32_t bar, uint16_t mask = 3) {
    if constexpr (CG == 2) {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
            ::"r"(bar), "h"(mask)
            : "memory");
    } else {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
    }
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Issue a 32-column TMEM load without waiting; tmem_wait(r) completes it. The
// wait names the destination registers so no use of them moves above it.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait(uint32_t* r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// A 32-column TMEM load and its wait in one asm statement: the destination
// registers are defined only after the wait, so the compiler cannot spill or
// reuse them while the load is in flight.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ float load16(const void* base, int64_t idx, int bf16) {
    const uint16_t u = static_cast<const uint16_t*>(base)[idx];
    if (bf16) return __uint_as_float((uint32_t)u << 16);
    return __half2float(__ushort_as_half(u));
}

template <int OUT>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    if constexpr (OUT == kOutBF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}


// One 32-column chunk of one warp's 32 rows: dequantise (and add the outlier
// term and bias), stage the chunk in shared memory, then write it out as
// whole 64-byte row segments (four lanes per row for 16-bit outputs; 32-bit
// outputs go out in two 16-column halves).
template <typename T16>
__device__ __forceinline__ float round16(float v) {
    if constexpr (std::is_same<T16, __nv_bfloat16>::value) return __bfloat162float(__float2bfloat16_rn(v));
    else return __half2float(__float2half_rn(v));
}

template <int OUT, bool OUTL, int KIND, int ACT = kActNone>
__device__ __forceinline__ void epi_chunk(const Params& p, const uint32_t* r, int cw, int col0, int row0, int64_t row,
                                          bool row_ok, float rx, const float* rw_w, const float* bias_w, uint8_t* stg,
                                          int lane, int n_out, bool compact, int prob, const CUtensorMap* tmap_y) {
    const GemmEpilogue& ep = p.ep;
    float y[32];
    if constexpr (OUT == kOutI32) {
#pragma unroll
        for (int e = 0; e < 32; ++e) y[e] = __int_as_float((int)r[e]);  // raw bits, stored unchanged
    } else {
        // y = acc * (rx * rw), each product one fp32 rounding, two lanes per op
        const float4* rw4 = reinterpret_cast<const float4*>(rw_w + cw);
        const uint64_t rx2 = pk2(rx, rx);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 w = rw4[e];
            const uint64_t d01 = mul2(rx2, pk2(w.x, w.y));
            const uint64_t d23 = mul2(rx2, pk2(w.z, w.w));
            float a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                a[i] = KIND == kKindF8 ? __uint_as_float(r[4 * e + i]) : (float)(int)r[4 * e + i];
            upk2(mul2(pk2(a[0], a[1]), d01), y[4 * e + 0], y[4 * e + 1]);
            upk2(mul2(pk2(a[2], a[3]), d23), y[4 * e + 2], y[4 * e + 3]);
        }
        if constexpr (OUTL) {
            // the 16-bit outlier term, added term by term in ascending o with
            // fma (the 16-bit products are exact in fp32)
            if (compact) {
                // X_O is o-major (a warp's 32 rows read 128 contiguous bytes);
                // two outliers per step so their loads are in flight together,
                // the fmas still in ascending o
                auto term = [&](float xo, const float4* w4) {
                    const uint64_t x2 = pk2(xo, xo);  // fmas two columns at a time
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 w = __ldg(w4 + e);
                        upk2(fma2(x2, pk2(w.x, w.y), pk2(y[4 * e + 0], y[4 * e + 1])), y[4 * e + 0], y[4 * e + 1]);
                        upk2(fma2(x2, pk2(w.z, w.w), pk2(y[4 * e + 2], y[4 * e + 3])), y[4 * e + 2], y[4 * e + 3]);
                    }
                };
                int o = 0;
                for (; o + 1 < n_out; o += 2) {
                    const float xa = row_ok ? __ldg(ep.xo + (int64_t)o * p.M + row) : 0.0f;
                    const float xb = row_ok ? __ldg(ep.xo + (int64_t)(o + 1) * p.M + row) : 0.0f;
                    term(xa, reinterpret_cast<const float4*>(ep.wo + (int64_t)o * ep.wo_ld + col0));
                    term(xb, reinterpret_cast<const float4*>(ep.wo + (int64_t)(o + 1) * ep.wo_ld + col0));
                }
                if (o < n_out) {
                    const float xa = row_ok ? __ldg(ep.xo + (int64_t)o * p.M + row) : 0.0f;
                    term(xa, reinterpret_cast<const float4*>(ep.wo + (int64_t)o * ep.wo_ld + col0));
                }
            } else {
                for (int o = 0; o < n_out; ++o) {
                    const int ko = ep.idx[o];
                    const float xo = row_ok ? load16(ep.x16, row * ep.ldx16 + ko, ep.in16_bf16) : 0.0f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = min(col0 + e, p.N - 1);
                        y[e] = __fmaf_rn(xo, load16(ep.w16, (int64_t)col * p.K + ko, ep.in16_bf16), y[e]);
                    }
                }
            }
        }
        if (ep.bias) {
            const float4* b4 = reinterpret_cast<const float4*>(bias_w + cw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 b = b4[e];
                y[4 * e + 0] = __fadd_rn(y[4 * e + 0], b.x);
                y[4 * e + 1] = __fadd_rn(y[4 * e + 1], b.y);
                y[4 * e + 2] = __fadd_rn(y[4 * e + 2], b.z);
                y[4 * e + 3] = __fadd_rn(y[4 * e + 3], b.w);
            }
        }
    }
    if constexpr (ACT != kActNone) {
        // the MLP activation on the 16-bit outputs Y this GEMM would write:
        // SwiGLU on interleaved (gate, up) column pairs -> 16 values h for the
        // chunk's 32 columns, ReLU or GELU -> 32 values; each h one rounding
        using T16 = typename std::conditional<OUT == kOutBF16, __nv_bfloat16, __half>::type;
#pragma unroll
        for (int e = 0; e < 32; ++e) y[e] = round16<T16>(y[e]);
        constexpr int NH = ACT == SQ_ACT_SWIGLU ? 16 : 32;  // activation values of the chunk
        if constexpr (ACT == SQ_ACT_SWIGLU) {
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(silu_fixed(y[2 * e]), y[2 * e + 1]);
        } else if constexpr (ACT == SQ_ACT_RELU) {
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] = y[e] > 0.0f ? y[e] : 0.0f;
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] = gelu_fixed(y[e]);
        }
        if (ep.act_qs) {
            // static per-tensor scale: the int8 codes of h, clipped, straight
            // from the registers (each lane writes its row's NH bytes)
            const float qs = *ep.act_qs;
            uint32_t w[NH / 4];
#pragma unroll
            for (int e = 0; e < NH / 4; ++e)
                w[e] = pack_low_bytes(quant_bits_clip(__fmul_rn(y[4 * e], qs)),
                                      quant_bits_clip(__fmul_rn(y[4 * e + 1], qs)),
                                      quant_bits_clip(__fmul_rn(y[4 * e + 2], qs)),
                                      quant_bits_clip(__fmul_rn(y[4 * e + 3], qs)));
            const int64_t nh = ACT == SQ_ACT_SWIGLU ? p.N / 2 : p.N;
            const int64_t col = ACT == SQ_ACT_SWIGLU ? (int64_t)col0 / 2 : (int64_t)col0;
            if (row_ok && col < nh) {
                uint8_t* out = static_cast<uint8_t*>(ep.Y) + prob * p.y_bstride + row * ep.ldy + col;
                if (p.vec_store && col + NH <= nh) {
#pragma unroll
                    for (int e = 0; e < NH / 16; ++e)
                        reinterpret_cast<uint4*>(out)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                } else {
#pragma unroll
                    for (int e = 0; e < NH; ++e)
                        if (col + e < nh) out[e] = (uint8_t)(w[e >> 2] >> (8 * (e & 3)));
                }
            }
            return;
        }
        if constexpr (ACT == SQ_ACT_SWIGLU) {
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = round16<T16>(y[e]);
            uint4* dst = reinterpret_cast<uint4*>(stg + lane * kStgRow);
#pragma unroll
            for (int e = 0; e < 2; ++e)
                dst[e] = make_uint4(pack2<OUT>(y[8 * e], y[8 * e + 1]), pack2<OUT>(y[8 * e + 2], y[8 * e + 3]),
                                    pack2<OUT>(y[8 * e + 4], y[8 * e + 5]), pack2<OUT>(y[8 * e + 6], y[8 * e + 7]));
            __syncwarp();
            // 32 rows x 32 bytes: two lanes per row segment
            const int part = lane & 1;
            const int64_t nh = p.N / 2;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int rr = it * 16 + (lane >> 1);
                const int64_t grow = (int64_t)row0 + rr;
                const int64_t col = (int64_t)col0 / 2 + part * 8;
                const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStgRow + part * 16);
                if (grow < p.M && col < nh) {
                    uint16_t* out = static_cast<uint16_t*>(ep.Y) + prob * p.y_bstride + grow * ep.ldy + col;
                    if (p.vec_store && col + 8 <= nh) {
                        *reinterpret_cast<uint4*>(out) = v;
                    } else {
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (col + e < nh) out[e] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
                    }
                }
            }
            __syncwarp();
            return;
        }
    }
    if constexpr (OUT == kOutBF16 || OUT == kOutF16) {
        if (p.tma_store) {
            // the previous chunk's store has read the box; refill it with
            // this lane's row (16-byte unit e of row r at unit e ^ ((r >> 1) & 3),
            // the 64-byte swizzle: the eight rows of each quarter-warp store
            // cover all 32 banks), then one lane hands the box to the copy engine
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            uint8_t* rowp = stg + lane * 64;
            const int sw = (lane >> 1) & 3;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                *reinterpret_cast<uint4*>(rowp + ((e ^ sw) << 4)) =
                    make_uint4(pack2<OUT>(y[8 * e], y[8 * e + 1]), pack2<OUT>(y[8 * e + 2], y[8 * e + 3]),
                               pack2<OUT>(y[8 * e + 4], y[8 * e + 5]), pack2<OUT>(y[8 * e + 6], y[8 * e + 7]));
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) tma_store_3d(tmap_y, smem_u32(stg), col0, row0, prob);
            return;
        }
        uint4* dst = reinterpret_cast<uint4*>(stg + lane * kStgRow);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack2<OUT>(y[8 * e], y[8 * e + 1]), pack2<OUT>(y[8 * e + 2], y[8 * e + 3]),
                                pack2<OUT>(y[8 * e + 4], y[8 * e + 5]), pack2<OUT>(y[8 * e + 6], y[8 * e + 7]));
        __syncwarp();
        const int part = lane & 3;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int rr = it * 8 + (lane >> 2);
            const int64_t grow = (int64_t)row0 + rr;
            const int col = col0 + part * 8;
            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStgRow + part * 16);
            if (grow < p.M && col < p.N) {
                uint16_t* out = static_cast<uint16_t*>(ep.Y) + prob * p.y_bstride + grow * ep.ldy + col;
                if (p.vec_store && col + 8 <= p.N) {
                    *reinterpret_cast<uint4*>(out) = v;
                } else {
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (col + e < p.N) out[e] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
                }
            }
        }
        __syncwarp();
    } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint4* dst = reinterpret_cast<uint4*>(stg + lane * kStgRow);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(__float_as_uint(y[16 * hh + 4 * e]), __float_as_uint(y[16 * hh + 4 * e + 1]),
                                    __float_as_uint(y[16 * hh + 4 * e + 2]), __float_as_uint(y[16 * hh + 4 * e + 3]));
            __syncwarp();
            const int part = lane & 3;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int rr = it * 8 + (lane >> 2);
                const int64_t grow = (int64_t)row0 + rr;
                const int col = col0 + 16 * hh + part * 4;
                const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStgRow + part * 16);
                if (grow < p.M && col < p.N) {
                    uint32_t* out = static_cast<uint32_t*>(ep.Y) + prob * p.y_bstride + grow * ep.ldy + col;
                    if (p.vec_store && col + 4 <= p.N) {
                        *reinterpret_cast<uint4*>(out) = v;
                    } else {
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (col + e < p.N) out[e] = w[e];
                    }
                }
            }
            __syncwarp();
        }
    }
}

template <int BN, int OUT, bool OUTL, int KIND, bool SK, int CG, int ACT = kActNone>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_y, const Params p) {
    using C = Cfg<BN, CG>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + C::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
    float* rw_s = reinterpret_cast<float*>(smem + C::RW_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA pair: CTA 0 issues the MMAs for both; its stage-full and
    // accumulator-empty barriers count both CTAs' loads and epilogue warps
    const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), kEpiWarps * CG);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        // a CTA pair allocates the same columns in both CTAs (one warp of each)
        if constexpr (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_holder)), "r"(C::TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_holder)), "r"(C::TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
        if (p.tma_store) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_y)) : "memory");
    }
    // bar.sync is an aligned barrier: every warp must reach it converged
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    // a pair: neither CTA signals the other's barriers before both are initialised
    if constexpr (CG == 2) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // the set-up above touches only this CTA's shared and tensor memory; wait
    // here for the previous kernel in the stream before any global access
    pdl_wait();
    pdl_trigger();
    // where this launch keeps its stream-K counters: if a bounded wait gives
    // up, sq_workspace_status clears that region with the status word
    if (SK && blockIdx.x == 0 && threadIdx.x == 0) p.status[3] = p.sk_cnt_bytes;

    const int num_tiles = p.batch * p.num_m * p.num_n;
    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_phase[s] = 0;
            bool ok = true;
            Segments<SK, CG> seg(p);
            int tile, k0, k1, slot;
            while (ok && seg.next(p, num_tiles, tile, k0, k1, slot)) {
                int b, m0, n0;
                tile_coords_b(tile, p, BM * CG, BN, b, m0, n0);
                // this CTA's rows: of a pair, CTA r loads Xq rows m0 + 128 r and
                // weight rows n0 + (BN / 2) r
                m0 += (int)rank * BM;
                n0 += (int)rank * (BN / CG);
                for (int kb = k0; kb < k1; ++kb) {
                    if (!wait_fast(empty_bar(stage), phase ^ 1u, abort_flag, p.status, 0x6E1)) {
                        ok = false;
                        break;
                    }
                    // the pair's loads all count on CTA 0's barrier, which expects both
                    const uint32_t fb = CG == 2 ? map_to_rank(full_bar(stage), 0) : full_bar(stage);
                    if (rank == 0) mbar_expect_tx(full_bar(stage), CG * (C::A_BYTES + C::B_BYTES));
                    // (no L2 eviction hints: marking the weight tiles evict-first made the
                    // other m-blocks of the group fetch them again, 2.8 -> 7.9 GB of DRAM
                    // reads at 4096 x 12288 x 49152, and the step 8 % slower on B200)
                    tma_load_3d<CG>(sbase + C::A_OFF + stage * C::A_BYTES, &tmap_a, fb, kb * BK, m0, b);
                    tma_load_3d<CG>(sbase + C::B_OFF + stage * C::B_BYTES, &tmap_b, fb, kb * BK, n0, b);
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES) stage = 0, phase ^= 1u;
                }
            }
            if (!ok && rank == 0) {
                // make sure no copy still lands in shared memory after we leave
                // (of a pair, CTA 0's barriers count both CTAs' copies, and both
                // CTAs stay resident until the pair's closing cluster barrier)
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s]) wait_drain(full_bar(s), issued_phase[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            Segments<SK, CG> seg(p);
            int tile, k0, k1, slot;
            for (; ok && seg.next(p, num_tiles, tile, k0, k1, slot); ++local) {
                const int acc = local & 1;
                const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
                if (!wait_fast(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status, 0x6E2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = k0; kb < k1; ++kb) {
                    if (!wait_fast(full_bar(stage), phase, abort_flag, p.status, 0x6E3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + C::A_OFF + stage * C::A_BYTES;
                    const uint32_t b_addr = sbase + C::B_OFF + stage * C::B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        umma<KIND, CG>(d_tmem, sdesc(a_addr + k * UMMA_K), sdesc(b_addr + k * UMMA_K),
                                       C::idesc(KIND), (kb != k0 || k != 0) ? 1u : 0u);
                    umma_commit<CG>(empty_bar(stage));  // both CTAs' stage is free
                    if (++stage == STAGES) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                umma_commit<CG>(tfull_bar(acc));  // both CTAs' epilogues may read
            }
            // all MMAs issued by this thread complete before tensor memory is freed
            umma_commit<CG>(drain_bar, 1);
            wait_drain(drain_bar, 0);
        }
    } else {
        // -------------------------------------------------------- epilogue
        // Eight warps: warp w reads TMEM lanes 32*(w%4)..+31 (its tile rows)
        // and half h = (w-2)/4 of the tile's columns. No block-level barrier
        // is used here: an abort can make one warp leave early, so each warp
        // stages its own column factors and output chunks and decides
        // collectively (all lanes) whether to go on.
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        constexpr int HC = BN / 2;        // columns per warp
        constexpr int NCH = HC / 32;      // 32-column chunks per warp
        const GemmEpilogue& ep = p.ep;
        const int n_out = OUTL ? *ep.n_out : 0;
        const bool compact = n_out <= kOutlierCap;
        float* rw_w = rw_s + (warp - 2) * 2 * HC;  // this warp's 1/qs_w and bias
        float* bias_w = rw_w + HC;
        uint8_t* stg = smem + C::STG_OFF + (warp - 2) * kStgWarpBytes;
        int local = 0;
        Segments<SK, CG> seg(p);
        int tile, k0, k1, slot;
        // the accumulator buffer is released on CTA 0's barrier for a pair
        auto release_acc = [&](int a) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2) mbar_arrive_remote(map_to_rank(tempty_bar(a), 0));
                else mbar_arrive(tempty_bar(a));
            }
        };
        for (; seg.next(p, num_tiles, tile, k0, k1, slot); ++local) {
            int b, m0, n0;
            tile_coords_b(tile, p, BM * CG, BN, b, m0, n0);
            m0 += (int)rank * BM;  // this CTA's 128 rows of the pair's tile
            const int c_base = n0 + half * HC;  // first column of this warp
            const int row0 = m0 + q * 32;  // first row of this warp
            const int64_t row = (int64_t)row0 + lane;
            const bool row_ok = row < p.M;
            // the tile's scales: every load issued before the first is used
            // (and the row scale before the wait for the accumulator), so a
            // short k-loop does not wait on them one after another
            float qxv = 1.0f;
            if constexpr (OUT != kOutI32) {
                constexpr int NL = HC / 32;
                float qv[NL], bv[NL];
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    const int col = c_base + lane + 32 * i;
                    qv[i] = 0.0f;
                    bv[i] = 0.0f;
                    if (col < p.N) {
                        qv[i] = ep.w_per_channel ? ep.qs_w[(int64_t)b * p.N + col] : ep.qs_w[b];
                        if (ep.bias) bv[i] = ep.bias[col];
                    }
                }
                if (row_ok) qxv = ep.x_per_token ? ep.qs_x[(int64_t)b * p.M + row] : ep.qs_x[b];
                __syncwarp();
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    rw_w[lane + 32 * i] = c_base + lane + 32 * i < p.N ? __frcp_rn(qv[i]) : 0.0f;
                    bias_w[lane + 32 * i] = bv[i];
                }
                __syncwarp();
            }
            const int acc = local & 1;
            const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
            if constexpr (OUTL) {
                // while this tile's MMAs run: bring its X_O rows and W_O
                // columns into L1, so the outlier term's loads do not wait on L2
                if (compact && row0 < p.M && c_base < p.N) {
                    for (int o = 0; o < n_out; ++o)
                        if (row_ok)
                            asm volatile("prefetch.global.L1 [%0];" ::"l"(ep.xo + (int64_t)o * p.M + row));
                    for (int i = lane; i < n_out * NCH; i += 32) {
                        const int o = i / NCH, l = i - o * NCH;
                        asm volatile("prefetch.global.L1 [%0];" ::"l"(ep.wo + (int64_t)o * ep.wo_ld + c_base + 32 * l));
                    }
                }
            }
            const bool ok = wait_fast(tfull_bar(acc), acc_phase, abort_flag, p.status, 0x6E4);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            float rx = 0.0f;
            if constexpr (OUT != kOutI32)
                if (row_ok) rx = __frcp_rn(qxv);
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + half * HC);
            // chunks that hold at least one valid column; none when the rows are past M
            int nch = 0;
            if (row0 < p.M && c_base < p.N) nch = min(NCH, (p.N - c_base + 31) / 32);
            // Double-buffered TMEM loads only where the variant keeps every
            // value in registers (no spill may sit between a load and its wait).
            // (the single-CTA GELU instance spills a few bytes, so it loads synchronously)
            constexpr bool kPipe = !OUTL && OUT != kOutF32 && !SK && !(ACT == SQ_ACT_GELU && CG == 1);
            uint32_t ra[32];
            if constexpr (SK) {
                if (slot >= 0) {
                    // a piece of a split tile: park this warp region's partial
                    // sums (each warp store writes 512 contiguous bytes),
                    // release the accumulator, count the piece's k-blocks in;
                    // the piece that completes the count adds every piece up
                    // (int32: exact in any order) and runs the epilogue
                    const int wr = warp - 2;
                    int4* mine = reinterpret_cast<int4*>(p.sk_part) +
                                 ((size_t)(blockIdx.x * 2 + slot) * kEpiWarps + wr) * (NCH * 8 * 32);
                    for (int c = 0; c < NCH; ++c) {
                        tmem_ld32(t_row + (uint32_t)(c * 32), ra);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            mine[(c * 8 + e) * 32 + lane] = make_int4((int)ra[4 * e], (int)ra[4 * e + 1],
                                                                      (int)ra[4 * e + 2], (int)ra[4 * e + 3]);
                    }
                    release_acc(acc);  // accumulator read in full
                    __threadfence();
                    __syncwarp();
                    const int u = tile - p.dp_tiles;
                    int before = 0;
                    // (of a pair, each CTA counts its own half of the tile)
                    int* cnt = p.sk_cnt + ((size_t)u * CG + rank) * kEpiWarps + wr;
                    if (lane == 0) before = atomicAdd(cnt, k1 - k0);
                    before = __shfl_sync(0xffffffffu, before, 0);
                    if (before + (k1 - k0) == p.num_kb) {
                        __threadfence();
                        const int x0 = u * p.num_kb;
                        const int c_lo = sk_owner(x0, p), c_hi = sk_owner(x0 + p.num_kb - 1, p);
                        for (int c = 0; c < nch; ++c) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) ra[e] = 0u;
                            for (int cc = c_lo; cc <= c_hi; ++cc) {
                                const int sl = sk_start(cc, p) >= x0 ? 0 : 1;
                                const int4* src = reinterpret_cast<const int4*>(p.sk_part) +
                                                  ((size_t)((cc * CG + (int)rank) * 2 + sl) * kEpiWarps + wr) *
                                                      (NCH * 8 * 32);
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const int4 v = __ldcg(src + (c * 8 + e) * 32 + lane);
                                    ra[4 * e] += (uint32_t)v.x;
                                    ra[4 * e + 1] += (uint32_t)v.y;
                                    ra[4 * e + 2] += (uint32_t)v.z;
                                    ra[4 * e + 3] += (uint32_t)v.w;
                                }
                            }
                            epi_chunk<OUT, OUTL, KIND, ACT>(p, ra, c * 32, c_base + c * 32, row0, row, row_ok, rx, rw_w,
                                                       bias_w, stg, lane, n_out, compact, b, &tmap_y);
                        }
                        if (lane == 0) *cnt = 0;  // ready for the next launch
                    }
                    continue;
                }
            }
            if constexpr (kPipe) {
                uint32_t rb[32];
                if (nch > 0) {
                    tmem_ld32_async(t_row, ra);
                    tmem_wait(ra);
                }
                for (int c = 0; c < nch; c += 2) {
                    // chunk c is in ra; fetch chunk c+1 into rb while ra is used
                    const bool more = c + 1 < nch;
                    if (more) tmem_ld32_async(t_row + (uint32_t)((c + 1) * 32), rb);
                    else {
                        release_acc(acc);  // accumulator read in full
                    }
                    epi_chunk<OUT, OUTL, KIND, ACT>(p, ra, c * 32, c_base + c * 32, row0, row, row_ok, rx, rw_w, bias_w, stg,
                                         lane, n_out, compact, b, &tmap_y);
                    if (!more) break;
                    tmem_wait(rb);
                    const bool more2 = c + 2 < nch;
                    if (more2) tmem_ld32_async(t_row + (uint32_t)((c + 2) * 32), ra);
                    else {
                        release_acc(acc);
                    }
                    epi_chunk<OUT, OUTL, KIND, ACT>(p, rb, (c + 1) * 32, c_base + (c + 1) * 32, row0, row, row_ok, rx, rw_w,
                                         bias_w, stg, lane, n_out, compact, b, &tmap_y);
                    if (more2) tmem_wait(ra);
                }
            } else {
                for (int c = 0; c < nch; ++c) {
                    tmem_ld32(t_row + (uint32_t)(c * 32), ra);
                    if (c + 1 == nch) {
                        release_acc(acc);  // accumulator read in full
                    }
                    epi_chunk<OUT, OUTL, KIND, ACT>(p, ra, c * 32, c_base + c * 32, row0, row, row_ok, rx, rw_w, bias_w, stg,
                                         lane, n_out, compact, b, &tmap_y);
                }
            }
            if (nch == 0) {
                release_acc(acc);
            }
        }
        // the output boxes handed to the copy engine are written before the
        // grid completes (and before the staging memory is released)
        if (p.tma_store && lane == 0) bulk_wait_all();
    }

    // Lanes 1..31 of warps 0 and 1 reach this point long before their lane 0
    // finishes its role loop; reconverge each warp first, because bar.sync is
    // an aligned barrier and must be executed by whole warps. Only then is
    // every MMA drained and every TMEM read done before the dealloc.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    // a pair: CTA 0's MMAs write both CTAs' tensor memory, so neither frees it
    // before both have finished (CTA 0's issuer waited for its last MMA)
    if constexpr (CG == 2) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D int8 tensor [batch, rows, K] (rows of each problem contiguous, problems
// rows * K bytes apart), box BK x box_rows x 1, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows, int64_t batch) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)batch};
    cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)(rows * K)};
    cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D 16-bit output [batch, M, ldy] (problems y_bstride elements apart), box
// 32 columns x 32 rows x 1, 64-byte swizzle (the staging layout of a chunk).
bool make_map_y(CUtensorMap* m, void* Y, int64_t M, int64_t N, int64_t ldy, int64_t batch, int64_t y_bstride,
                bool bf16) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)batch};
    cuuint64_t strides[2] = {(cuuint64_t)(ldy * 2), (cuuint64_t)(y_bstride * 2)};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const Params);

template <int BN, bool SK, int CG>
KernelFn pick_kernel_sk(sq_dtype_t out_dt, bool outl, int kind) {
    if (kind == kKindF8) {
        switch (out_dt) {
            case SQ_BF16: return gemm_w8a8_kernel<BN, kOutBF16, false, kKindF8, SK, CG>;
            case SQ_F16: return gemm_w8a8_kernel<BN, kOutF16, false, kKindF8, SK, CG>;
            default: return gemm_w8a8_kernel<BN, kOutF32, false, kKindF8, SK, CG>;
        }
    }
    switch (out_dt) {
        case SQ_BF16:
            return outl ? gemm_w8a8_kernel<BN, kOutBF16, true, kKindI8, SK, CG>
                        : gemm_w8a8_kernel<BN, kOutBF16, false, kKindI8, SK, CG>;
        case SQ_F16:
            return outl ? gemm_w8a8_kernel<BN, kOutF16, true, kKindI8, SK, CG>
                        : gemm_w8a8_kernel<BN, kOutF16, false, kKindI8, SK, CG>;
        case SQ_F32: return gemm_w8a8_kernel<BN, kOutF32, false, kKindI8, SK, CG>;
        default: return gemm_w8a8_kernel<BN, kOutI32, false, kKindI8, SK, CG>;
    }
}

// the fused-activation variants: 16-bit outputs, int8 operands, no outlier term
template <int BN, bool SK, int CG>
KernelFn pick_kernel_act(sq_dtype_t out_dt, int act) {
    const bool bf = out_dt == SQ_BF16;
    switch (act) {
        case SQ_ACT_SWIGLU:
            return bf ? gemm_w8a8_kernel<BN, kOutBF16, false, kKindI8, SK, CG, SQ_ACT_SWIGLU>
                      : gemm_w8a8_kernel<BN, kOutF16, false, kKindI8, SK, CG, SQ_ACT_SWIGLU>;
        case SQ_ACT_RELU:
            return bf ? gemm_w8a8_kernel<BN, kOutBF16, false, kKindI8, SK, CG, SQ_ACT_RELU>
                      : gemm_w8a8_kernel<BN, kOutF16, false, kKindI8, SK, CG, SQ_ACT_RELU>;
        default:
            return bf ? gemm_w8a8_kernel<BN, kOutBF16, false, kKindI8, SK, CG, SQ_ACT_GELU>
                      : gemm_w8a8_kernel<BN, kOutF16, false, kKindI8, SK, CG, SQ_ACT_GELU>;
    }
}

template <int BN, int CG>
KernelFn pick_kernel(sq_dtype_t out_dt, bool outl, int kind, bool sk, int act) {
    if (act != kActNone) return sk ? pick_kernel_act<BN, true, CG>(out_dt, act) : pick_kernel_act<BN, false, CG>(out_dt, act);
    return sk ? pick_kernel_sk<BN, true, CG>(out_dt, outl, kind) : pick_kernel_sk<BN, false, CG>(out_dt, outl, kind);
}

// CTA pairs of the pair kernel that can be resident at once on the current
// device (0 if the device cannot run it), cached per device.
int max_resident_pairs() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    if (cache[dev] == 0) {
        using C = Cfg<256, 2>;
        KernelFn fn = gemm_w8a8_kernel<256, kOutBF16, false, kKindI8, false, 2>;
        int n = 0;
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM_ALLOC) ==
            cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * num_sms());
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = C::SMEM_ALLOC;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();
        cache[dev] = n > 0 ? n : -1;
    }
    return cache[dev] > 0 ? cache[dev] : 0;
}

// SQ_GEMM_CTA_PAIRS: 0 never uses CTA pairs, 1 uses them wherever the plan
// allows (256-wide tiles); unset leaves the choice to plan_gemm. Read on
// every call (a few hundred nanoseconds), so a process can switch it.
int pairs_mode() {
    const char* e = getenv("SQ_GEMM_CTA_PAIRS");
    return (e && e[0] == '0') ? 0 : (e && e[0] == '1') ? 1 : -1;
}

template <int BN, int CG>
sq_status_t launch_bn(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K, const GemmEpilogue& ep,
                      const GemmPlan& plan, int* status, void* sk_ws, cudaStream_t stream) {
    using C = Cfg<BN, CG>;
    CUtensorMap ta, tb;
    // each CTA loads 128 rows of Xq and BN / CG rows of the weight per stage
    if (!make_map(&ta, Xq, M, K, BM, ep.batch) || !make_map(&tb, Wq, N, K, BN / CG, ep.batch))
        return set_error(SQ_ERR_CUDA, "sq_gemm_w8a8: cuTensorMapEncodeTiled failed");
    const bool outl = ep.idx != nullptr;
    if (outl && ep.out_dt != SQ_BF16 && ep.out_dt != SQ_F16)
        return set_error(SQ_ERR_INVALID_ARG, "sq_gemm_w8a8: the outlier term needs a 16-bit output");
    const bool sk = plan.sk_tiles > 0 && sk_ws != nullptr;
    KernelFn fn = pick_kernel<BN, CG>(ep.out_dt, outl, ep.kind, sk, ep.act);
    // the shared-memory opt-in is per kernel and per device; it is cheap, so set it every time
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM_ALLOC) != cudaSuccess)
        return check_launch("sq_gemm_w8a8: set shared memory size");
    Params p;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.batch = (int)ep.batch;
    p.y_bstride = ep.y_bstride;
    p.num_m = (int)((M + BM * CG - 1) / (BM * CG));
    p.num_n = (int)((N + BN - 1) / BN);
    p.num_kb = (int)((K + BK - 1) / BK);
    // rows of Xq per raster group kept within about 96 MB of L2
    // (SQ_GEMM_GROUP_MB overrides the 96). Measured on B200 at 4096 x 12288 x
    // 49152 (single CTAs, K-panels of 6.3 MB): 48 MB groups read 3.68 GB from
    // DRAM in 1769 us, 96 MB groups 2.87 GB in 1715 us, 16 MB groups 7.25 GB
    // in 2049 us; 4096 x 36864 x 12288 (pairs) is the same from 48 MB up.
    const int64_t per_mblock = (int64_t)BM * CG * K;
    int64_t budget = 96;
    if (const char* e = getenv("SQ_GEMM_GROUP_MB")) {
        const long v = strtol(e, nullptr, 10);
        if (v > 0 && v < 4096) budget = v;
    }
    int64_t g = (budget << 20) / per_mblock;
    p.group_m = (int)(g < 1 ? 1 : (g > p.num_m ? p.num_m : g));
    // bytes per output element: int8 codes from a fused activation with a
    // static scale, else the output dtype's
    const int eb = ep.act_qs ? 1 : (ep.out_dt == SQ_BF16 || ep.out_dt == SQ_F16) ? 2 : 4;
    p.vec_store = ((reinterpret_cast<uintptr_t>(ep.Y) & 15u) == 0) && ((ep.ldy * eb) % 16 == 0);
    // 16-bit outputs of the plain, ReLU and GELU epilogues go out by TMA
    // store (row and problem strides multiples of 16 bytes, within the
    // tensor map's limits); SwiGLU's half-width rows keep the plain stores
    CUtensorMap ty;
    memset(&ty, 0, sizeof(ty));
    p.tma_store = 0;
    const int64_t ybs = ep.batch > 1 ? ep.y_bstride : M * ep.ldy;  // one problem: any stride past its rows
    if (p.vec_store && eb == 2 && ep.act != SQ_ACT_SWIGLU && (ybs * 2) % 16 == 0 && ybs * 2 < (1ll << 40))
        p.tma_store = make_map_y(&ty, ep.Y, M, N, ep.ldy, ep.batch, ybs, ep.out_dt == SQ_BF16) ? 1 : 0;
    p.ep = ep;
    p.status = status;
    p.dp_tiles = sk ? plan.tiles - plan.sk_tiles : plan.tiles;
    p.sk_tiles = sk ? plan.sk_tiles : 0;
    p.sk_iters = sk ? plan.sk_tiles * p.num_kb : 0;
    p.sk_units = plan.grid / CG;
    p.sk_cnt = sk ? static_cast<int*>(sk_ws) : nullptr;
    p.sk_cnt_bytes = sk ? (int)plan.sk_cnt_bytes : 0;
    p.sk_part = sk ? reinterpret_cast<int*>(static_cast<uint8_t*>(sk_ws) + plan.sk_cnt_bytes) : nullptr;
    const int grid = plan.grid;
    if constexpr (CG == 2)
        launch_pdl_cluster(fn, dim3(grid), dim3(kThreads), C::SMEM_ALLOC, stream, 2, ta, tb, ty, p);
    else
        launch_pdl(fn, dim3(grid), dim3(kThreads), C::SMEM_ALLOC, stream, ta, tb, ty, p);
    return check_launch("sq_gemm_w8a8");
}

}  // namespace

// Arrival counters of a split: one per warp region of each CTA's part of a
// tile, in a region of one size for every shape (room for kSkMaxParts CTA
// parts of tiles; a split covers less than one wave, so fewer parts than
// SMs). The counters thus sit at the same bytes whatever the shape: a call
// that leaves them at zero leaves the workspace ready for a call of any other
// shape it is large enough for, and the partial sums one shape parks after
// its counters are never read as another shape's counters.
constexpr int64_t kSkMaxParts = 256;
static size_t sk_counter_bytes() { return (size_t)kSkMaxParts * kEpiWarps * sizeof(int); }
static_assert((kSkMaxParts * kEpiWarps * sizeof(int)) % 256 == 0, "the parked sums start 256-byte aligned");

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int64_t batch) {
    GemmPlan pl;
    const int sms = num_sms();
    const int64_t num_m = (M + BM - 1) / BM;
    // narrow N tiles when wide ones would leave most SMs idle
    const int64_t tiles256 = batch * num_m * ((N + 255) / 256);
    pl.bn = (tiles256 < (int64_t)sms && N > 128) ? 128 : 256;
    const int64_t tiles = batch * num_m * ((N + pl.bn - 1) / pl.bn);
    pl.tiles = (int)tiles;
    pl.grid = (int)(tiles < sms ? tiles : sms);
    // Stream-K for the remainder: when the last wave of whole tiles would be
    // at most three quarters full (and the waves average under 90 % busy),
    // its tiles are cut by k-blocks into one range per CTA, which every CTA
    // runs before its whole tiles. Measured on B200: 1024 x 7168 x 7168
    // (56 k-blocks) 54.1 -> 51.4 us, 1024 x 7168 x 28672 176 -> 174 us. Each
    // CTA's range must hold 8 k-blocks or more, and the k-loop 32 or more,
    // or the parking of partial sums costs more than the idle tail. Waves
    // between 90 and 95 % busy are cut only for k-loops of 64 blocks or more
    // (4096 x 12288 x 49152: 1832 -> 1792 us; 1024 x 21504 x 7168 gains nothing).
    const int64_t kb = (K + BK - 1) / BK;
    const int64_t rem = tiles % pl.grid;
    const double eff = (double)tiles / (double)(((tiles + pl.grid - 1) / pl.grid) * pl.grid);
    if (batch == 1 && pl.grid == sms && tiles > pl.grid && kb >= 32 && rem > 0 && 4 * rem <= 3 * (int64_t)pl.grid &&
        (eff < 0.9 || (eff < 0.95 && kb >= 64)) && rem * kb >= 8ll * pl.grid && rem * kb < (1ll << 31) &&
        rem <= kSkMaxParts) {
        pl.sk_tiles = (int)rem;
        pl.sk_cnt_bytes = sk_counter_bytes();
        pl.sk_bytes = pl.sk_cnt_bytes + (size_t)pl.grid * 2 * BM * pl.bn * sizeof(int);
    }
    // CTA pairs (256 x 256 tiles, cta_group::2: each SM streams half the
    // weight bytes per MMA) where there are two waves of them or more, with or
    // without a stream-K split in the single-CTA plan. Measured on B200 (us,
    // single CTA -> pairs): 4096 x 36864 x 12288 1285 -> 1252 (and 1178 with
    // the inline waits), 4096 x 12288 x 12288 419 (stream-K) -> 386,
    // 4096 x 12288 x 49152 1713 (stream-K) -> 1625; shapes with fewer pair
    // tiles keep single CTAs and their split (1024 x 7168 x 28672: 158).
    if (pl.bn == 256 && pairs_mode() != 0) {
        const int pairs = max_resident_pairs();
        const int64_t ptiles = batch * ((M + 2 * BM - 1) / (2 * BM)) * ((N + 255) / 256);
        if (pairs > 0 && ptiles < (1ll << 31) && (pairs_mode() == 1 || ptiles >= 2ll * pairs)) {
            GemmPlan pp;
            pp.bn = 256;
            pp.cg = 2;
            pp.tiles = (int)ptiles;
            const int units = (int)(ptiles < pairs ? ptiles : pairs);
            pp.grid = 2 * units;
            // the stream-K rule over pairs: the ragged last wave of pair tiles
            // cut into one k-range per pair, for k-loops of 64 to 128 blocks.
            // Measured on B200 (us, whole pair tiles -> split): 4096 x 12288 x
            // 12288 (96 k-blocks, 10.4 waves of 74 pairs) 382 -> 368; longer or
            // shorter k-loops lost: 4096 x 12288 x 49152 1713 -> 1734,
            // 2048 x 6144 x 4096 45.2 -> 47.1
            const int64_t prem = ptiles % units;
            const double peff = (double)ptiles / (double)(((ptiles + units - 1) / units) * units);
            if (batch == 1 && units == pairs && ptiles > units && kb >= 64 && kb <= 128 && prem > 0 &&
                4 * prem <= 3 * (int64_t)units && peff < 0.95 && prem * kb >= 8ll * units && prem * kb < (1ll << 31) &&
                2 * prem <= kSkMaxParts) {
                pp.sk_tiles = (int)prem;
                pp.sk_cnt_bytes = sk_counter_bytes();
                pp.sk_bytes = pp.sk_cnt_bytes + (size_t)pp.grid * 2 * BM * pp.bn * sizeof(int);
            }
            return pp;
        }
    }
    return pl;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0) return kStatusBytes;
    return kStatusBytes + plan_gemm(M, N, K, 1).sk_bytes;
}

sq_status_t launch_gemm_w8a8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                             const GemmEpilogue& ep, int* status_word, size_t ws_bytes, cudaStream_t stream) {
    const GemmPlan pl = plan_gemm(M, N, K, ep.batch);
    // a workspace without room for the split runs whole tiles only
    void* sk_ws = (pl.sk_tiles > 0 && ws_bytes >= kStatusBytes + pl.sk_bytes)
                      ? static_cast<void*>(reinterpret_cast<uint8_t*>(status_word) + kStatusBytes)
                      : nullptr;
    if (pl.cg == 2) return launch_bn<256, 2>(Xq, Wq, M, N, K, ep, pl, status_word, sk_ws, stream);
    if (pl.bn == 128) return launch_bn<128, 1>(Xq, Wq, M, N, K, ep, pl, status_word, sk_ws, stream);
    return launch_bn<256, 1>(Xq, Wq, M, N, K, ep, pl, status_word, sk_ws, stream);
}

}  // namespace sq

extern "C" sq_status_t sq_gemm_fp8(const uint8_t* Xq, const uint8_t* Wq, int64_t M, int64_t N, int64_t K,
                                   const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                                   const float* bias, sq_dtype_t out_dt, void* Y, int64_t ldy, void* workspace,
                                   size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_gemm_fp8";
    SQ_REQUIRE((Xq || M == 0) && Wq && (Y || M == 0) && qs_x && qs_w, SQ_ERR_INVALID_ARG,
               "%s: null Xq, Wq, Y or scales", name);
    SQ_REQUIRE(out_dt == SQ_F32 || out_dt == SQ_F16 || out_dt == SQ_BF16, SQ_ERR_INVALID_ARG,
               "%s: out dtype must be F32, F16 or BF16", name);
    SQ_REQUIRE(workspace && ws_bytes >= sq::kStatusBytes, SQ_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes",
               name, sq::kStatusBytes);
    SQ_REQUIRE(M >= 0 && N > 0 && K > 0 && ldy >= N, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need N > 0, K > 0, ldy >= N", name);
    SQ_REQUIRE(K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be a multiple of 16 (TMA row stride)", name);
    SQ_REQUIRE(M < (1ll << 31) && N < (1ll << 31), SQ_ERR_UNSUPPORTED_SHAPE, "%s: M and N must be < 2^31", name);
    SQ_REQUIRE(sq::aligned16(Xq) && sq::aligned16(Wq), SQ_ERR_ALIGNMENT, "%s: Xq and Wq must be 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    sq::GemmEpilogue ep;
    ep.qs_x = qs_x;
    ep.x_per_token = x_per_token;
    ep.qs_w = qs_w;
    ep.w_per_channel = w_per_channel;
    ep.bias = bias;
    ep.out_dt = out_dt;
    ep.Y = Y;
    ep.ldy = ldy;
    ep.kind = 1;
    return sq::launch_gemm_w8a8(reinterpret_cast<const int8_t*>(Xq), reinterpret_cast<const int8_t*>(Wq), M, N, K, ep,
                                static_cast<int*>(workspace), ws_bytes, sq::as_cuda(stream));
}

extern "C" sq_status_t sq_bmm_w8a8(const int8_t* Aq, const int8_t* Bq, int64_t batch, int64_t M, int64_t N,
                                   int64_t K, const float* qs_a, int a_per_row, const float* qs_b, int b_per_row,
                                   sq_dtype_t out_dt, void* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                                   sq_stream_t stream) {
    const char* name = "sq_bmm_w8a8";
    SQ_REQUIRE(batch >= 0 && M >= 0 && N > 0 && K > 0 && ldy >= N, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: need batch, M >= 0, N, K > 0, ldy >= N", name);
    if (batch == 0 || M == 0) return SQ_OK;
    SQ_REQUIRE(Aq && Bq && Y, SQ_ERR_INVALID_ARG, "%s: null Aq, Bq or Y", name);
    SQ_REQUIRE(out_dt == SQ_I32 || (qs_a && qs_b), SQ_ERR_INVALID_ARG, "%s: dequantising output needs qs_a and qs_b",
               name);
    SQ_REQUIRE(out_dt == SQ_I32 || out_dt == SQ_F32 || out_dt == SQ_F16 || out_dt == SQ_BF16, SQ_ERR_INVALID_ARG,
               "%s: out dtype must be I32, F32, F16 or BF16", name);
    SQ_REQUIRE(workspace && ws_bytes >= sq::kStatusBytes, SQ_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes",
               name, sq::kStatusBytes);
    SQ_REQUIRE(K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be a multiple of 16 (TMA row stride)", name);
    SQ_REQUIRE(K <= 133144, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K > 133144 could overflow the int32 accumulator", name);
    SQ_REQUIRE(batch * ((M + 127) / 128) * ((N + 127) / 128) < (1ll << 31) && M < (1ll << 31) && N < (1ll << 31),
               SQ_ERR_UNSUPPORTED_SHAPE, "%s: too many tiles", name);
    SQ_REQUIRE(sq::aligned16(Aq) && sq::aligned16(Bq), SQ_ERR_ALIGNMENT, "%s: Aq and Bq must be 16-byte aligned", name);
    sq::GemmEpilogue ep;
    ep.qs_x = qs_a;
    ep.x_per_token = a_per_row;
    ep.qs_w = qs_b;
    ep.w_per_channel = b_per_row;
    ep.out_dt = out_dt;
    ep.Y = Y;
    ep.ldy = ldy;
    ep.batch = batch;
    ep.y_bstride = M * ldy;
    return sq::launch_gemm_w8a8(Aq, Bq, M, N, K, ep, static_cast<int*>(workspace), ws_bytes, sq::as_cuda(stream));
}

extern "C" sq_status_t sq_gemm_w8a8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                                    const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                                    const float* bias, sq_dtype_t out_dt, void* Y, int64_t ldy, void* workspace,
                                    size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_gemm_w8a8";
    SQ_REQUIRE((Xq || M == 0) && Wq && (Y || M == 0), SQ_ERR_INVALID_ARG, "%s: null Xq, Wq or Y", name);
    SQ_REQUIRE(out_dt == SQ_I32 || (qs_x && qs_w), SQ_ERR_INVALID_ARG, "%s: dequantising output needs qs_x and qs_w",
               name);
    SQ_REQUIRE(out_dt == SQ_I32 || out_dt == SQ_F32 || out_dt == SQ_F16 || out_dt == SQ_BF16, SQ_ERR_INVALID_ARG,
               "%s: out dtype must be I32, F32, F16 or BF16", name);
    SQ_REQUIRE(workspace && ws_bytes >= sq::kStatusBytes, SQ_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes",
               name, sq::kStatusBytes);
    SQ_REQUIRE(M >= 0 && N > 0 && K > 0 && ldy >= N, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need N > 0, K > 0, ldy >= N", name);
    SQ_REQUIRE(K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be a multiple of 16 (TMA row stride)", name);
    SQ_REQUIRE(K <= 133144, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K > 133144 could overflow the int32 accumulator", name);
    SQ_REQUIRE(M < (1ll << 31) && N < (1ll << 31), SQ_ERR_UNSUPPORTED_SHAPE, "%s: M and N must be < 2^31", name);
    SQ_REQUIRE(sq::aligned16(Xq) && sq::aligned16(Wq), SQ_ERR_ALIGNMENT, "%s: Xq and Wq must be 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    sq::GemmEpilogue ep;
    ep.qs_x = qs_x;
    ep.x_per_token = x_per_token;
    ep.qs_w = qs_w;
    ep.w_per_channel = w_per_channel;
    ep.bias = bias;
    ep.out_dt = out_dt;
    ep.Y = Y;
    ep.ldy = ldy;
    return sq::launch_gemm_w8a8(Xq, Wq, M, N, K, ep, static_cast<int*>(workspace), ws_bytes, sq::as_cuda(stream));
}

extern "C" sq_status_t sq_gemm_w8a8_act(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                                        const float* qs_x, int x_per_token, const float* qs_w, int w_per_channel,
                                        const float* bias, sq_act_t act, const float* static_qs, sq_dtype_t out_dt,
                                        void* H, int64_t ldh, void* workspace, size_t ws_bytes, sq_stream_t stream) {
    const char* name = "sq_gemm_w8a8_act";
    SQ_REQUIRE((Xq || M == 0) && Wq && (H || M == 0) && qs_x && qs_w, SQ_ERR_INVALID_ARG,
               "%s: null Xq, Wq, H or scales", name);
    SQ_REQUIRE(act == SQ_ACT_SWIGLU || act == SQ_ACT_RELU || act == SQ_ACT_GELU, SQ_ERR_INVALID_ARG,
               "%s: bad activation", name);
    SQ_REQUIRE(out_dt == SQ_F16 || out_dt == SQ_BF16, SQ_ERR_INVALID_ARG, "%s: out dtype must be F16 or BF16", name);
    SQ_REQUIRE(workspace && ws_bytes >= sq::kStatusBytes, SQ_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes",
               name, sq::kStatusBytes);
    const int64_t width = act == SQ_ACT_SWIGLU ? N / 2 : N;
    SQ_REQUIRE(M >= 0 && N > 0 && K > 0 && ldh >= width, SQ_ERR_UNSUPPORTED_SHAPE, "%s: need N > 0, K > 0, ldh >= %s",
               name, act == SQ_ACT_SWIGLU ? "N/2" : "N");
    SQ_REQUIRE(act != SQ_ACT_SWIGLU || N % 2 == 0, SQ_ERR_UNSUPPORTED_SHAPE,
               "%s: SwiGLU needs an even N (interleaved gate/up channel pairs)", name);
    SQ_REQUIRE(K % 16 == 0, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K must be a multiple of 16 (TMA row stride)", name);
    SQ_REQUIRE(K <= 133144, SQ_ERR_UNSUPPORTED_SHAPE, "%s: K > 133144 could overflow the int32 accumulator", name);
    SQ_REQUIRE(M < (1ll << 31) && N < (1ll << 31), SQ_ERR_UNSUPPORTED_SHAPE, "%s: M and N must be < 2^31", name);
    SQ_REQUIRE(sq::aligned16(Xq) && sq::aligned16(Wq), SQ_ERR_ALIGNMENT, "%s: Xq and Wq must be 16-byte aligned", name);
    if (M == 0) return SQ_OK;
    sq::GemmEpilogue ep;
    ep.qs_x = qs_x;
    ep.x_per_token = x_per_token;
    ep.qs_w = qs_w;
    ep.w_per_channel = w_per_channel;
    ep.bias = bias;
    ep.out_dt = out_dt;
    ep.Y = H;
    ep.ldy = ldh;
    ep.act = (int)act;
    ep.act_qs = static_qs;
    return sq::launch_gemm_w8a8(Xq, Wq, M, N, K, ep, static_cast<int*>(workspace), ws_bytes, sq::as_cuda(stream));
}

// Declarations shared between the library's translation units (not public).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sq_api.h"

namespace sq {

// Every workspace-taking operation keeps a 256-byte header; word 0 is the
// status word written by bounded device waits (0 = fine).
constexpr size_t kStatusBytes = 256;

// Rows per block of the outlier-count pass of sq_llmint8_detect.
constexpr int kDetectRows = 128;
size_t detect_workspace_bytes(int64_t M, int64_t K);
size_t llmint8_workspace_bytes(int64_t M, int64_t N, int64_t K);

// Outlier counts up to this size use compact fp32 copies of the outlier
// columns (X_O [M, cap], W_O [cap, N padded to 256]) built in the workspace;
// larger sets read the 16-bit operands directly in the epilogue.
constexpr int kOutlierCap = 32;

// Epilogue description of the int8 GEMM.
struct GemmEpilogue {
    const float* qs_x = nullptr;
    int x_per_token = 0;
    const float* qs_w = nullptr;
    int w_per_channel = 0;
    const float* bias = nullptr;
    sq_dtype_t out_dt = SQ_BF16;
    void* Y = nullptr;
    int64_t ldy = 0;
    // LLM.int8 16-bit outlier term: sum over o < *n_out of
    // X16[i, idx[o]] * W16[j, idx[o]] (null idx = no outlier term).
    const void* x16 = nullptr;
    int64_t ldx16 = 0;
    const void* w16 = nullptr;
    const int32_t* idx = nullptr;
    const int32_t* n_out = nullptr;
    int in16_bf16 = 0;
    const float* xo = nullptr;  // [kOutlierCap, M] fp32 copies of X[:, O] (o-major)
    const float* wo = nullptr;  // [kOutlierCap, wo_ld] fp32 copies of W[:, O]^T
    int64_t wo_ld = 0;          // multiple of 256, >= N
    int kind = 0;               // 0: int8 operands, int32 sums; 1: FP8 E4M3 operands, fp32 sums
    int act = -1;               // sq_act_t applied to the 16-bit output (sq_gemm_w8a8_act), -1: none
    const float* act_qs = nullptr;  // with act: a static per-tensor scale, Y then holds the int8 codes of h
    int64_t batch = 1;          // independent problems; operands [batch, rows, K], scales [batch, rows]
    int64_t y_bstride = 0;      // elements between the batches of Y
};

// How the GEMM covers a problem: tile width, grid, and how many trailing
// tiles are cut by k-blocks (stream-K), with the scratch that needs.
struct GemmPlan {
    int bn = 256;
    int cg = 1;  // 2: tiles of 256 rows on CTA pairs (cta_group::2), grid = 2 x pairs
    int tiles = 0;
    int grid = 0;
    int sk_tiles = 0;
    size_t sk_cnt_bytes = 0;  // arrival counters per tile region (zero between launches)
    size_t sk_bytes = 0;      // counters + parked partial sums
};
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int64_t batch);
// Workspace of sq_gemm_w8a8 / sq_gemm_fp8: the status header plus the
// stream-K scratch of the plan.
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

// status_word: the caller's workspace (ws_bytes); the stream-K scratch, if
// the plan has one and it fits, follows the 256-byte header.
sq_status_t launch_gemm_w8a8(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                             const GemmEpilogue& ep, int* status_word, size_t ws_bytes, cudaStream_t stream);

}  // namespace sq

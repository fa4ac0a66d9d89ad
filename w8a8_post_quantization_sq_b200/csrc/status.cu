// Host-side status handling, workspace sizing and device queries.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {

static thread_local std::string g_last_error;

sq_status_t set_error(sq_status_t st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

sq_status_t check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(SQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return SQ_OK;
}

bool pdl_enabled() {
    static const bool on = [] {
        const char* e = getenv("SQ_DISABLE_PDL");
        return !(e && e[0] == '1');
    }();
    return on;
}

int num_sms() {
    // one entry per device, filled on first use; host threads may race to
    // fill it, and every one of them stores the same value
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace sq

extern "C" {

const char* sq_last_error_string(void) { return sq::g_last_error.c_str(); }

int sq_version(void) { return 100; }

size_t sq_workspace_size(sq_op_t op, int64_t M, int64_t N, int64_t K) {
    switch (op) {
        case SQ_OP_GEMM: return sq::gemm_workspace_bytes(M, N, K);
        case SQ_OP_QUANT_ACT: return sq::kStatusBytes;
        case SQ_OP_QUANT_WEIGHT: return sq::kStatusBytes;
        case SQ_OP_LLMINT8_DETECT: return sq::detect_workspace_bytes(M, K);
        case SQ_OP_LLMINT8: return sq::llmint8_workspace_bytes(M, N, K);
    }
    return 0;
}

sq_status_t sq_workspace_status(void* workspace, sq_stream_t stream) {
    SQ_REQUIRE(workspace != nullptr, SQ_ERR_INVALID_ARG, "sq_workspace_status: null workspace");
    cudaStream_t s = sq::as_cuda(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return sq::set_error(SQ_ERR_CUDA, "sq_workspace_status: %s",
                             cudaGetErrorString(cudaGetLastError()));
    // word 0: the status word; word 3: the size of the stream-K counter
    // region that follows the header, as the last stream-K GEMM recorded it
    int words[4] = {0, 0, 0, 0};
    if (cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess)
        return sq::set_error(SQ_ERR_CUDA, "sq_workspace_status: copy failed");
    if (words[0] != 0) {
        // a call gave up part-way: its stream-K counters may be left counted
        // in; clear them with the status word, so the next call starts clean
        if (words[3] > 0 && words[3] <= (1 << 26))
            cudaMemset(static_cast<char*>(workspace) + sq::kStatusBytes, 0, (size_t)words[3]);
        const int zero = 0;
        cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice);
        cudaMemcpy(static_cast<int*>(workspace) + 3, &zero, sizeof(int), cudaMemcpyHostToDevice);
        return sq::set_error(SQ_ERR_TIMEOUT,
                             "a bounded device wait timed out (code %d); results of that call are invalid",
                             words[0]);
    }
    return SQ_OK;
}

}  // extern "C"

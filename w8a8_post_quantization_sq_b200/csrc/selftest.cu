// Check of the failure path of the bounded waits: one block waits on an
// mbarrier that nothing completes, with the same bounded wait the GEMM roles
// use, gives up after timeout_ns, records its code in the workspace status
// word and returns; the host sees SQ_ERR_TIMEOUT from sq_workspace_status and
// the context stays usable. No fault, trap or hang is involved.
#include "sq_common.cuh"
#include "sq_internal.h"
#include "sq_wait.cuh"

namespace sq {
namespace {

__global__ void wait_timeout_kernel(int* status, uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
        mbar_init(b, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // phase 0 never completes: no thread arrives
        wait_bounded_ns(b, 0, &abort_flag, status, 0x6E5, timeout_ns);
    }
}

}  // namespace
}  // namespace sq

extern "C" sq_status_t sq_selftest_wait_timeout(void* workspace, size_t ws_bytes, uint64_t timeout_ns,
                                                sq_stream_t stream) {
    SQ_REQUIRE(workspace && ws_bytes >= sq::kStatusBytes, SQ_ERR_INVALID_ARG,
               "sq_selftest_wait_timeout: needs a workspace of %zu bytes", sq::kStatusBytes);
    SQ_REQUIRE(timeout_ns > 0 && timeout_ns <= 2000000000ull, SQ_ERR_INVALID_ARG,
               "sq_selftest_wait_timeout: timeout must be in (0, 2 s]");
    sq::wait_timeout_kernel<<<1, 32, 0, sq::as_cuda(stream)>>>(static_cast<int*>(workspace), timeout_ns);
    return sq::check_launch("sq_selftest_wait_timeout");
}

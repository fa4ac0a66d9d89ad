// mbarrier helpers and the bounded wait shared by the kernels that wait on
// asynchronous copies or on other roles of their block.
#pragma once

#include <stdint.h>

namespace sq {

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Wait for the phase of `parity` to complete. Gives up when another role has
// set *abort_flag, or after timeout_ns of %globaltimer, when it sets the flag
// and records `code` in the status word (read on the host by
// sq_workspace_status). Never traps: the caller drains its own work and
// returns.
static __device__ __noinline__ bool wait_bounded_ns(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                             int code, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((n & 31u) == 0 && global_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            atomicExch(status, code);
            return false;
        }
    }
}

}  // namespace sq

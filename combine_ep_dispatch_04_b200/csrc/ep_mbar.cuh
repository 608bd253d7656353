// ep_mbar.cuh -- shared-memory barriers (mbarrier) with bounded waits, as
// the tensor-core kernels use them: every wait gives up after kWaitLimitNs of
// %globaltimer and reports it, so that no kernel can wait for ever.
#pragma once

#include <cstdint>

namespace ep {

constexpr uint32_t kDevTimeout = 0x4u;               // status bit: a bounded wait gave up
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s

__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// true once the phase of parity `parity` has completed; false after 2 s
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = gtimer();
#pragma unroll 1
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (gtimer() - t0 > kWaitLimitNs) return false;
    }
}

}  // namespace ep

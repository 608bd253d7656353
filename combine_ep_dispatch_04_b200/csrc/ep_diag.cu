// ep_diag.cu -- a check of the bounded waits of the tensor-core kernels.
//
// ep_wait_probe launches one block whose thread waits, with the same helper
// the GEMM kernels use (mbar_wait), on a shared-memory barrier that nothing
// completes: the wait must give up after kWaitLimitNs and set kDevTimeout in
// the status word, and the kernel must return, leaving the context usable.
// This is the failure path of every mbarrier wait, exercised without a fault.
#include <cuda_runtime.h>

#include "ep.h"
#include "ep_mbar.cuh"

namespace ep {

__global__ void wait_probe_kernel(uint32_t *status) {
    __shared__ uint64_t bar;
    const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);  // one arrival completes the phase; none comes
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(b, 0)) atomicOr(status, kDevTimeout);
}

}  // namespace ep

extern "C" ep_status_t ep_wait_probe(uint32_t *dev_status, ep_stream_t stream) {
    if (!dev_status) return EP_ERR_INVALID_ARG;
    ep::wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev_status);
    return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

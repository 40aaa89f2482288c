// selftest.cu -- failure-detection self test of the bounded pipeline waits.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits for
// it with the same bounded wait the GEMV/GEMM pipelines use, but with a short
// caller-chosen limit.  The wait gives up, raises WQ_DEVFLAG_TIMEOUT in the
// status word and the kernel returns normally: no trap, no hang, the context
// stays usable.
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

__global__ void bounded_wait_selftest_kernel(uint32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0u, status, limit_ns);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(uint32_t* status, uint32_t limit_us, cudaStream_t stream) {
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, (uint64_t)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace wq

// selftest.cu -- the bounded wait of the library's kernels, exercised on its own: one CTA waits on
// an mbarrier that nothing arrives at, with the same helper the kernels use on their copies, gives
// up after the cap and records the timeout in the status word.
#include "../../include/stq.h"
#include "stq_internal.cuh"

namespace stq {
namespace {

__global__ void wait_timeout_kernel(int32_t *status)
{
    __shared__ unsigned long long bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    // phase 0 never completes: no thread arrives and no copy is in flight
    const bool got = mbar_wait_bounded(smem_u32(&bar), 0u);
    if (!got && threadIdx.x == 0) flag(status, kFlagTimeout);
}

}  // namespace
}  // namespace stq

extern "C" stq_status stq_selftest_wait_timeout(int32_t *dev_status, void *stream)
{
    if (!dev_status) return STQ_ERR_INVALID_ARG;
    stq::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status);
    return cudaGetLastError() == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

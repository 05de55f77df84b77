// selftest.cu -- a device wait that never completes, for the failure-detection
// test: every mbarrier wait of the tcgen05 kernels goes through the bounded
// mbar_wait, which gives up after kWaitLimitNs, records MOE_ERR_TIMEOUT in
// the status word and raises the CTA's abort flag instead of hanging.  Here
// nothing ever arrives on the barrier, so the wait must run out.
#include <cuda.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void wait_selftest_kernel(int32_t *status)
{
    pdl_enter();
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, status);
}

}  // namespace
}  // namespace moe

extern "C" MOE_API moe_status moe_selftest_wait_timeout(int32_t *dev_status, moe_stream_t stream)
{
    if (!dev_status) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t err = moe::launch_k(moe::wait_selftest_kernel, dim3(1), dim3(32), 0, s, dev_status);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// selftest.cu -- the kernels' failure path, exercised without a real failure.
//
// Every wait in the kernels is bounded: after WAIT_NS of polling the waiting thread records
// ERR_TIMEOUT in the layout's device error word and gives up (sm100.cuh), so a stalled pipeline
// ends its kernel instead of hanging the GPU, and the host learns of it from st_layout_check.
// st_selftest_wait_timeout launches one warp whose only wait is on an mbarrier that nothing
// completes: that wait runs out exactly as a stalled pipeline's would.
#include "layout.h"
#include "sm100.cuh"

namespace st {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int32_t *err)
{
    __shared__ uint64_t bar;
    __shared__ int32_t abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival completes phase 0; none is ever made
        abort = 0;
        fence_barrier_init();
        mbar_wait(&bar, 0, &abort, err);  // gives up after WAIT_NS and records ERR_TIMEOUT
    }
}

}  // namespace
}  // namespace st

extern "C" st_status_t st_selftest_wait_timeout(st_layout_t *layout, st_stream_t stream)
{
    if (!layout) return ST_ERR_INVALID_ARG;
    if (!layout->uploaded) return ST_ERR_NOT_UPLOADED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (dev != layout->device) return ST_ERR_INVALID_ARG;
    st::wait_timeout_kernel<<<1, 32, 0, stream>>>(layout->d_err);
    return cudaGetLastError() == cudaSuccess ? ST_OK : ST_ERR_CUDA;
}

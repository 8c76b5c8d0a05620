// pa_selftest.cu -- a kernel whose bounded waits can never succeed, for the
// test of the library's failure path: every mbarrier wait in the kernels
// gives up after a fixed limit (2 s), flags PA_DEV_TIMEOUT in the caller's
// status word and lets the kernel return, so that a lost arrival ends as a
// status bit and the CUDA context stays usable.  Here nothing ever arrives
// on the barrier, so each of the three wait forms the kernels use (the
// unrolled poll, the rolled poll, the warp-collective one) must time out.
#include <cuda_runtime.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

__global__ void __launch_bounds__(96) wait_timeout_selftest_kernel(int32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Phase 0 of a fresh barrier completes only after one arrival: none comes.
    bool ok = true;
    if (warp == 0) {
        if (lane == 0) ok = mbar_wait(&bar, 0);
    } else if (warp == 1) {
        if (lane == 0) ok = mbar_wait_lean(&bar, 0);
    } else {
        ok = mbar_wait_warp(&bar, 0);
    }
    if (!ok && lane == 0) flag_status(status, PA_DEV_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int32_t* status, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 96, 0, stream>>>(status);
    return cudaGetLastError();
}

}  // namespace pa

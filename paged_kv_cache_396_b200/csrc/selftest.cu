// selftest.cu -- the device-side failure path, exercised without a GPU fault.
//
// Every pipeline wait of the kernels is bounded: ptx::mbar_wait gives up after ~2 s
// of globaltimer time, the kernel records PA_DEV_TIMEOUT and returns, and the CUDA
// context stays usable.  This kernel runs that wait on a phase nothing completes.
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"
#include "selftest.h"

namespace pkv {

namespace {

__global__ void wait_timeout_kernel(int32_t *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);   // one arrival completes phase 0; none comes
        ptx::fence_mbar_init();
    }
    __syncthreads();
    const bool done = ptx::mbar_wait(&bar, 0);
    if (!done && threadIdx.x == 0) raise_flag(err, PA_DEV_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(int32_t *err, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(err);
    return cudaGetLastError();
}

}  // namespace pkv

// selftest.h -- launcher of the device failure-path self-test (selftest.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

// One CTA whose bounded mbarrier wait (the pipelines' ptx::mbar_wait) waits on a phase
// nothing completes; after ~2 s it sets PA_DEV_TIMEOUT in *err and returns.
cudaError_t launch_selftest_wait_timeout(int32_t *err, cudaStream_t stream);

}  // namespace pkv

// A self-test of the library's failure path: every pipeline wait in the kernels is bounded, and a
// wait that runs out records JCA_STATUS_TIMEOUT, stops its CTA and returns, leaving the context
// usable. This kernel runs that same bounded wait on a barrier that nothing ever completes (a
// flag that nothing sets), so a test can check the status and the context afterwards without
// faulting or hanging the GPU.
#include <cstdint>

#include <cuda_runtime.h>

#include "jca_device.cuh"
#include "jca_internal.h"

namespace jca {
namespace {

__global__ void wait_timeout_selftest_kernel(int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Phase 0 never completes: no thread arrives and no copy is pending.
    mbar_wait(smem_u32(&bar), 0, &abort_flag, status);
  }
  __syncthreads();
}

}  // namespace
}  // namespace jca

extern "C" int jca_selftest_wait_timeout(int32_t* status, jca_stream_t stream) {
  if (!status) return JCA_ERR_NULL;
  int dev = 0, sms = 0;
  const int rc = jca::current_device(&dev, &sms);
  if (rc) return rc;
  jca::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

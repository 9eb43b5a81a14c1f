// selftest.cu -- diagnostic entry point for the device-side failure path.
//
// Every kernel of the library waits on mbarriers with a bounded wait
// (mbar_wait in cr_device.cuh: %globaltimer limit CR_WAIT_TIMEOUT_NS, then the
// CTA records CR_ERR_TIMEOUT in the workspace status word and winds down).
// cr_selftest_wait_timeout runs that same wait on a barrier that nothing ever
// completes, so that a test can check that the wait gives up, that the status
// word records the timeout, and that the context stays usable -- without any
// fault, trap or unbounded wait.

#include <cuda_runtime.h>

#include <cstdint>

#include "cr_device.cuh"
#include "cr_internal.h"

namespace cr {
namespace {

__global__ void wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // one arrival expected; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0u, &abort_flag)) record_status(status, CR_ERR_TIMEOUT);
}

}  // namespace
}  // namespace cr

extern "C" cr_status cr_selftest_wait_timeout(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < 256) return CR_ERR_WORKSPACE;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return CR_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return CR_ERR_UNSUPPORTED_ARCH;
  int* status = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + cr::kWsStatusOff);
  cr::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
  return cudaGetLastError() == cudaSuccess ? CR_OK : CR_ERR_CUDA;
}

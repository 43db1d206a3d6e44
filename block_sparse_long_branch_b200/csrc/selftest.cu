// selftest.cu -- msa_selftest_wait_timeout: drives the kernels' failure path
// (a bounded wait that runs out, an error code in the workspace, the kernel
// returning normally) without faulting or hanging the GPU.
//
// One warp waits, with the same mbar_wait_for every kernel of the library
// uses, on an mbarrier that nothing ever arrives on.  The wait gives up after
// the caller's limit, records kDevSelfTest and the kernel exits; the caller
// reads the code back with msa_get_device_error.
#include <stdint.h>

#include "../../include/msa.h"
#include "sm100.cuh"

namespace msa {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // no thread or copy ever arrives on `bar`: the phase-0 wait can only run out
  mbar_wait_for(&bar, 0, &abort_s, err, kDevSelfTest, limit_ns);
  __syncwarp();
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_selftest_wait_timeout(void* ws, uint64_t limit_ns,
                                                  msa_stream_t stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u) || limit_ns < 1000 ||
      limit_ns > 1000000000ull)
    return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  msa::wait_timeout_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

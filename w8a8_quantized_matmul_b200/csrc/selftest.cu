// Self-test of the bounded device-side wait that every kernel of the library
// uses: one CTA waits on an mbarrier phase that nothing completes. The wait
// gives up after its time limit and the CTA records I8MM_ERR_TIMEOUT in a status
// word, exactly as the kernels do when a wait runs out, and leaves normally.
// No fault, trap or endless loop is involved; the GPU context stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "int8mm.h"
#include "ptx.cuh"

namespace i8mm {
namespace {

__global__ void wait_timeout_kernel(int32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival expected; none ever comes
    fence_mbarrier_init();
  }
  __syncthreads();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0));
  if (!ok && threadIdx.x == 0) atomicCAS(status, 0, -5 /* I8MM_ERR_TIMEOUT */);
}

}  // namespace
}  // namespace i8mm

extern "C" int int8_selftest_wait_timeout(int32_t* status, i8mm_stream_t stream) {
  if (!status) return I8MM_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return I8MM_ERR_CUDA;
  i8mm::wait_timeout_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError() == cudaSuccess ? I8MM_OK : I8MM_ERR_CUDA;
}

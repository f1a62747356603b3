// int8_mixed_matmul_noalloc: the full LLM.int8() matmul without a caller
// workspace. Its scratch (outlier bitmap and list, codes, scales, outlier
// panels, control words) lives in one statically sized device array of this
// library, so neither the caller nor the library allocates device memory when
// it runs. Meant for callers that cannot hand the library a workspace: code
// whose host framework owns every device allocation and gives it no
// allocator, or code that must not grow device memory use at call time.
//
// Costs and limits:
//   * every GPU that loads the library holds kNoAllocScratchBytes (64 MiB) of
//     device memory for this array until the process exits;
//   * problems whose workspace (int8_mixed_matmul_workspace_size) exceeds that
//     are rejected with I8MM_ERR_WORKSPACE;
//   * all calls on a device share the one array and it keeps the contents of
//     the last call; calls that may overlap on the GPU (other streams, other
//     host threads) race on it and must be serialised by the caller.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "int8mm.h"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
// Offset of the status word in the scratch: the array is carved exactly like a
// caller workspace, whose second int32 is the status word.
constexpr size_t kStatusOffset = 4;

// The scratch itself. In host code this name is only a stand-in for the device
// object: its device address must be obtained with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached. The device is checked first:
// on anything but sm_100 the module holding the array does not load, and the
// lookup would fail with an unrelated CUDA error.
int scratch_address(void** out) {
  const int st = i8mm::abi_check_device();
  if (st != I8MM_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return i8mm::abi_cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return I8MM_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      // Record why, and clear the error so that the caller's next
      // cudaGetLastError does not blame an unrelated launch for it.
      (void)cudaGetLastError();
      return i8mm::abi_cuda_fail("cudaGetSymbolAddress of the built-in scratch",
                                 e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return I8MM_OK;
}

}  // namespace

static_assert(kNoAllocScratchBytes == I8MM_NOALLOC_SCRATCH_BYTES, "header and array disagree");

extern "C" {

int int8_mixed_matmul_noalloc(const void* X, const int8_t* Wq, const float* w_scale,
                              const void* Wt_fp16, int M, int N, int K, float threshold,
                              void* Y, i8mm_stream_t stream) {
  if (M == 0 || N == 0) {
    // Same empty-problem rule as int8_mixed_matmul, without touching the device.
    return int8_mixed_matmul(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, nullptr, 0, stream);
  }
  const size_t need = int8_mixed_matmul_workspace_size(M, N, K);
  if (need == 0) {
    // Invalid sizes: let the regular entry point report which check failed.
    return int8_mixed_matmul(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) return I8MM_ERR_WORKSPACE;   // too large for the array
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != I8MM_OK) return st;
  // The regular path clears the control words it needs (count, status, barrier
  // counter, bitmap) at the start of every call, so the previous call's
  // contents of the array do not matter.
  return int8_mixed_matmul(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, scratch,
                           kNoAllocScratchBytes, stream);
}

int int8_noalloc_device_status(i8mm_stream_t stream) {
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != I8MM_OK) return st;
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, static_cast<const uint8_t*>(scratch) + kStatusOffset, 4,
                                  cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return i8mm::abi_cuda_fail("status read", e);
  return h == 0 ? I8MM_OK : (h == I8MM_ERR_TIMEOUT ? I8MM_ERR_TIMEOUT : I8MM_ERR_CUDA);
}

}  // extern "C"

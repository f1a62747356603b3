// Top-k outlier selection ([AIInfra] "05Quantization01", LLM.int8() section,
// training notes: keep the top 1% or 2% largest-magnitude feature dimensions in
// FP16): the outlier set is the k columns with the largest max |x| over the
// tokens, ties to the lower column index.
//
// One CTA: radix select of the k-th largest key over the column maxima (fp32
// >= 0, whose bit patterns order like the values), four passes of 8-bit digits
// with a shared-memory histogram; then every key above it is selected, and of
// the keys equal to it the ones with the lowest column indices, by an
// index-ordered block scan. The result is an outlier bitmap.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxWords = 65536 / 32;

__global__ void __launch_bounds__(kThreads) topk_select_kernel(const float* __restrict__ colmax,
                                                               int K, int k,
                                                               uint32_t* __restrict__ bitmap) {
  __shared__ unsigned int hist[256];
  __shared__ uint32_t words[kMaxWords];
  __shared__ unsigned int s_prefix, s_remaining, s_taken;
  __shared__ unsigned int warp_cnt[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (K + 31) / 32;
  for (int w = tid; w < nw; w += kThreads) words[w] = 0u;
  __syncthreads();
  if (k >= K) {
    for (int j = tid; j < K; j += kThreads) atomicOr(&words[j >> 5], 1u << (j & 31));
  } else if (k > 0) {
    unsigned int prefix = 0u, mask = 0u, remaining = static_cast<unsigned int>(k);
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += kThreads) hist[i] = 0u;
      __syncthreads();
      for (int j = tid; j < K; j += kThreads) {
        const unsigned int key = __float_as_uint(colmax[j]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        unsigned int cum = 0u;
        for (int d = 255; d >= 0; --d) {
          if (cum + hist[d] >= remaining) {
            s_prefix = prefix | (static_cast<unsigned int>(d) << shift);
            s_remaining = remaining - cum;
            break;
          }
          cum += hist[d];
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      mask |= 0xFFu << shift;
      __syncthreads();
    }
    // prefix is the k-th largest key; `remaining` keys equal to it are taken.
    if (tid == 0) s_taken = 0u;
    __syncthreads();
    for (int base = 0; base < K; base += kThreads) {
      const int j = base + tid;
      const unsigned int key = (j < K) ? __float_as_uint(colmax[j]) : 0u;
      const bool eq = (j < K) && key == prefix;
      const unsigned int ball = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) warp_cnt[warp] = __popc(ball);
      __syncthreads();
      unsigned int before = s_taken;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w];
      before += __popc(ball & ((1u << lane) - 1u));
      const bool take = (j < K) && (key > prefix || (eq && before < remaining));
      if (take) atomicOr(&words[j >> 5], 1u << (j & 31));
      __syncthreads();
      if (tid == 0) {
        unsigned int tot = 0u;
        for (int w = 0; w < kThreads / 32; ++w) tot += warp_cnt[w];
        s_taken += tot;
      }
      __syncthreads();
    }
  }
  __syncthreads();
  for (int w = tid; w < nw; w += kThreads) bitmap[w] = words[w];
}

}  // namespace

cudaError_t launch_topk_select(const float* colmax, int K, int k, uint32_t* bitmap,
                               cudaStream_t s) {
  if (K <= 0 || K > 65536) return cudaErrorInvalidValue;
  topk_select_kernel<<<1, kThreads, 0, s>>>(colmax, K, k, bitmap);
  return cudaGetLastError();
}

}  // namespace i8mm

// Top-k outlier selection ([AIInfra] "05Quantization01", LLM.int8() section,
// training notes: keep the top 1% or 2% largest-magnitude feature dimensions in
// FP16): the outlier set is the k columns with the largest max |x| over the
// tokens, ties to the lower column index.
//
// Up to 8192 columns each column is ranked against all others across the grid
// and selected when its rank is below k. Beyond, one CTA runs a radix select
// of the k-th largest key over the column maxima (fp32 >= 0, whose bit
// patterns order like the values), held in registers; four
// passes of 8-bit digits, each a shared-memory histogram (one atomic per
// distinct digit per warp) and a warp scan of its 256 bins; then every key
// above the k-th is selected, and of the keys equal to it the ones with the
// lowest column indices, by an index-ordered block scan. The result is an
// outlier bitmap.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxWords = 65536 / 32;

// The digit d of the current pass such that the keys with that digit (and the
// prefix so far) hold the `remaining`-th largest: suffix sums of the histogram
// from digit 255 down, by warp 0 (eight bins per lane, then a warp scan).
__device__ __forceinline__ void pick_digit(const unsigned int* hist, unsigned int remaining,
                                           unsigned int* s_digit, unsigned int* s_above) {
  const int lane = threadIdx.x & 31;
  // lane l owns bins 255 - 8l - i, i = 0..7 (highest digits first)
  unsigned int c[8], tot = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hist[255 - 8 * lane - i];
    tot += c[i];
  }
  unsigned int incl = tot;   // inclusive prefix over lanes 0..lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  unsigned int before = incl - tot;   // keys in higher digits than this lane's bins
  // the lane whose range contains the remaining-th key
  const bool mine = before < remaining && incl >= remaining;
  if (mine) {
    unsigned int cum = before;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (cum + c[i] >= remaining) {
        *s_digit = static_cast<unsigned int>(255 - 8 * lane - i);
        *s_above = cum;
        break;
      }
      cum += c[i];
    }
  }
}

// KPT keys per thread (keys t + i * kThreads) held in registers, K <= KPT *
// kThreads; KPT = 64 reads them from global memory (L2) in every pass instead.
template <int KPT>
__global__ void __launch_bounds__(kThreads) topk_select_kernel(const float* __restrict__ colmax,
                                                               int K, int k,
                                                               uint32_t* __restrict__ bitmap) {
  constexpr bool kRegs = KPT <= 16;
  constexpr int kMaxKeys = KPT;
  __shared__ unsigned int hist[256];
  __shared__ uint32_t words[kMaxWords];
  __shared__ unsigned int s_digit, s_above;
  __shared__ unsigned int warp_cnt[kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (K + 31) / 32;
  const int per = (K + kThreads - 1) / kThreads;
  // Thread t holds keys j = t + i * kThreads (coalesced loads, once).
  unsigned int kr[kRegs ? KPT : 1];
#pragma unroll
  for (int i = 0; i < (kRegs ? KPT : 1); ++i) {
    const int j = tid + i * kThreads;
    kr[i] = (kRegs && i < per && j < K) ? __float_as_uint(__ldg(colmax + j)) : 0u;
  }
  auto key_of = [&](int i) -> unsigned int {
    if constexpr (kRegs) {
      return kr[i];
    } else {
      const int j = tid + i * kThreads;
      return j < K ? __float_as_uint(__ldg(colmax + j)) : 0u;
    }
  };
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
#pragma unroll
      for (int i = 0; i < kMaxKeys; ++i) {
        const int j = tid + i * kThreads;
        if (i < per) {
          const unsigned int ki = key_of(i);
          const bool in = j < K && (ki & mask) == prefix;
          const unsigned int d = (ki >> shift) & 255u;
          // one atomic per distinct digit among the warp's matching lanes
          const unsigned int act = __ballot_sync(0xffffffffu, in);
          if (in) {
            const unsigned int peers = __match_any_sync(act, d);
            if (lane == __ffs(peers) - 1) atomicAdd(&hist[d], __popc(peers));
          }
        }
      }
      __syncthreads();
      if (warp == 0) pick_digit(hist, remaining, &s_digit, &s_above);
      __syncthreads();
      prefix |= s_digit << shift;
      remaining -= s_above;
      mask |= 0xFFu << shift;
    }
    // prefix is the k-th largest key; `remaining` keys equal to it are taken,
    // the ones with the lowest column indices.
    unsigned int taken = 0u;
#pragma unroll
    for (int i = 0; i < kMaxKeys; ++i) {
      if (i < per) {
        const int j = tid + i * kThreads;
        const unsigned int ki = key_of(i);
        const bool eq = j < K && ki == prefix;
        const unsigned int ball = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) warp_cnt[warp] = __popc(ball);
        __syncthreads();
        unsigned int before = taken;
        for (int w = 0; w < warp; ++w) before += warp_cnt[w];
        before += __popc(ball & ((1u << lane) - 1u));
        const bool take = j < K && (ki > prefix || (eq && before < remaining));
        if (take) atomicOr(&words[j >> 5], 1u << (j & 31));
        unsigned int tot = 0u;
        for (int w = 0; w < kWarps; ++w) tot += warp_cnt[w];
        taken += tot;
        __syncthreads();
      }
    }
  }
  __syncthreads();
  for (int w = tid; w < nw; w += kThreads) bitmap[w] = words[w];
}

// Up to kRankMax columns, by ranks: column i is selected when fewer than k
// columns come before it in the order (key descending, column ascending), i.e.
// when #{j : key_j > key_i} + #{j < i : key_j == key_i} < k, key the bit pattern
// of the column maximum (non-negative fp32 orders like its bits). Every CTA
// stages all K keys in shared memory and ranks 32 columns, the ones of one
// bitmap word: lane l of each warp holds column 32*blockIdx + l and counts over
// a sixteenth of the j range (broadcast reads, four keys per load); the sixteen
// partial counts are summed and the word is written whole. K*K comparisons over
// the grid replace the one-CTA passes of the radix select.
constexpr int kRankMax = 8192;
constexpr int kRankThreads = 512;
constexpr int kRankWarps = kRankThreads / 32;

__global__ void __launch_bounds__(kRankThreads) topk_rank_kernel(const float* __restrict__ colmax,
                                                                 int K, int k,
                                                                 uint32_t* __restrict__ bitmap) {
  __shared__ __align__(16) unsigned int keys[kRankMax];
  __shared__ unsigned int part[kRankWarps][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K4 = (K + 3) & ~3;   // keys padded with 0, which never count (see below)
  for (int j = tid; j < K4; j += kRankThreads)
    keys[j] = j < K ? __float_as_uint(__ldg(colmax + j)) : 0u;
  __syncthreads();
  const int base = 32 * blockIdx.x;
  const int i = base + lane;
  const unsigned int ki = i < K ? keys[i] : 0u;
  // this warp's share of j, a multiple of 4 long
  const int span = ((K4 / 4 + kRankWarps - 1) / kRankWarps) * 4;
  const int j0 = warp * span;
  const int j1 = min(j0 + span, K4);
  unsigned int c = 0u;
  // A padded key (0, at j >= K > i) never counts: 0 > ki is false and j < i is false.
  if (j1 <= base) {
    // every j < i: ties count
    for (int j = j0; j < j1; j += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(keys + j);
      c += (v.x >= ki) + (v.y >= ki) + (v.z >= ki) + (v.w >= ki);
    }
  } else if (j0 >= base + 32) {
    // every j > i: only larger keys count
    for (int j = j0; j < j1; j += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(keys + j);
      c += (v.x > ki) + (v.y > ki) + (v.z > ki) + (v.w > ki);
    }
  } else {
    for (int j = j0; j < j1; ++j) {
      const unsigned int kj = keys[j];
      c += (kj > ki) || (kj == ki && j < i);
    }
  }
  part[warp][lane] = c;
  __syncthreads();
  if (warp == 0) {
    unsigned int r = 0u;
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) r += part[w][lane];
    const unsigned int word = __ballot_sync(0xffffffffu, i < K && r < static_cast<unsigned int>(k));
    if (lane == 0) bitmap[blockIdx.x] = word;
  }
}

}  // namespace

cudaError_t launch_topk_select(const float* colmax, int K, int k, uint32_t* bitmap,
                               cudaStream_t s) {
  if (K <= 0 || K > 65536) return cudaErrorInvalidValue;
  if (K <= kRankMax) {
    topk_rank_kernel<<<(K + 31) / 32, kRankThreads, 0, s>>>(colmax, K, k < 0 ? 0 : k, bitmap);
    return cudaGetLastError();
  }
  if (K <= 4 * kThreads)
    topk_select_kernel<4><<<1, kThreads, 0, s>>>(colmax, K, k, bitmap);
  else if (K <= 16 * kThreads)
    topk_select_kernel<16><<<1, kThreads, 0, s>>>(colmax, K, k, bitmap);
  else
    topk_select_kernel<64><<<1, kThreads, 0, s>>>(colmax, K, k, bitmap);
  return cudaGetLastError();
}

}  // namespace i8mm

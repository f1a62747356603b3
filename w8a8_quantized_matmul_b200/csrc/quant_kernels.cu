// Memory-bound kernels of the LLM.int8() path on sm_100a:
//   * quantize_weight_rows_kernel  - offline per-output-row absmax INT8 codes of W
//   * detect_outliers_kernel        - outlier-column bitmap of X (|x| > threshold),
//                                     finished by the last CTA into a count and the
//                                     ascending column list (stand-alone entry point)
//   * quantize_rows_kernel          - per-token absmax over the non-outlier columns and
//                                     INT8 codes, 0 at outliers (stand-alone entry point)
//   * weight_rowsum_kernel          - sum_k Wq[n][k] per output row, the weight factor of
//                                     the zero-point correction (offline)
// (The full path uses the fused, cooperative form of both in fused_quant.cu.)
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (magnitude-threshold detection, vector-wise absmax quantisation, FP16 outlier
// columns); tanjunchen "quantization explained part 2", section 1.2 (threshold
// 6.0; absmax of the remaining dims after the split).
//
// All loads of X and W are 128-bit (8 fp16 per lane) and coalesced along K.
// K is a multiple of 16, so a 16-byte vector never straddles a row end.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "quant_common.cuh"

namespace i8mm {


// ---------------------------------------------------------------------------
// Offline weight quantisation: one warp per output row n.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_weight_rows_kernel(const __half* __restrict__ W,
                                                                   int N, int K,
                                                                   int8_t* __restrict__ Wq,
                                                                   float* __restrict__ w_scale) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const uint4* src = reinterpret_cast<const uint4*>(W + static_cast<size_t>(row) * K);
  const int nv = K >> 3;
  float amax = 0.0f;
  for (int v = lane; v < nv; v += 32) {
    float f[8];
    unpack8(__ldg(src + v), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = warp_max(amax);
  uint2* dst = reinterpret_cast<uint2*>(Wq + static_cast<size_t>(row) * K);
  for (int v = lane; v < nv; v += 32) {
    float f[8];
    unpack8(__ldg(src + v), f);
    uint2 o;
    o.x = pack4(quant_code(f[0], amax), quant_code(f[1], amax), quant_code(f[2], amax),
                quant_code(f[3], amax));
    o.y = pack4(quant_code(f[4], amax), quant_code(f[5], amax), quant_code(f[6], amax),
                quant_code(f[7], amax));
    dst[v] = o;
  }
  if (lane == 0) w_scale[row] = amax;
}

// ---------------------------------------------------------------------------
// Outlier detection. Grid: x = column slabs of 256 columns (32 lanes x 8),
// y = row blocks of kDetectRows rows (each of the 8 warps takes every 8th row).
// `bitmap` and `counter` must be zero on entry. The last CTA to finish turns the
// bitmap into the count and the ascending list, and leaves the count in
// *counter (which doubles as the arrival counter until then).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) detect_outliers_kernel(
    const __half* __restrict__ X, int M, int K, float threshold, uint32_t* bitmap,
    int32_t* counter, int32_t* __restrict__ col_idx) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int v = blockIdx.x * 32 + lane;  // uint4 index along the row (8 columns)
  const int nv = K >> 3;
  const int r0 = blockIdx.y * kDetectRows;
  const int r1 = min(M, r0 + kDetectRows);

  uint32_t flags = 0;  // bit b: column 8v+b has |x| > threshold in some row seen here
  if (v < nv) {
    int r = r0 + warp;
#pragma unroll 4
    for (; r < r1; r += 8) {
      float f[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K) + v), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) flags |= (fabsf(f[i]) > threshold ? 1u : 0u) << i;
    }
  }
  // Lanes 4w..4w+3 cover the 32 columns of one bitmap word.
  uint32_t word = flags << (8 * (lane & 3));
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  if ((lane & 3) == 0 && word != 0 && v < nv) atomicOr(bitmap + (v >> 2), word);

  // Last-CTA finalisation (fence + arrival counter; no waiting).
  __shared__ bool is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int total = gridDim.x * gridDim.y;
    const int prev = atomicAdd(counter, 1);
    is_last = (prev == total - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  const int words = (K + 31) >> 5;
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < words; base += blockDim.x) {
    const int w = base + threadIdx.x;
    const uint32_t bits = (w < words) ? __ldcg(bitmap + w) : 0u;
    const int c = __popc(bits);
    // Block-wide exclusive scan of c.
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int s = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += t;
      }
      warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - c;
    if (w < words) {
      if (col_idx) {
        uint32_t b = bits;
        int p = excl;
        while (b) {
          const int j = __ffs(b) - 1;
          b &= b - 1;
          col_idx[p++] = w * 32 + j;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *counter = carry;
}

// ---------------------------------------------------------------------------
// Per-token quantisation for the stand-alone entry point. One warp per row;
// the row is held in registers (VPL 16-byte vectors per lane, VPL*256 >= K),
// so X is read from memory once; VPL == 0 streams longer rows twice.
// ---------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __half* __restrict__ X, int M,
                                                            int K,
                                                            const uint32_t* __restrict__ bitmap,
                                                            int8_t* __restrict__ Xq,
                                                            float* __restrict__ x_scale) {
  extern __shared__ uint32_t qsmem[];
  const int words = (K + 31) >> 5;
  uint32_t* s_bits = qsmem;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int w = threadIdx.x; w < words; w += blockDim.x) s_bits[w] = bitmap[w];
  __syncthreads();
  const int nv = K >> 3;

  const int rows_per_block = 8 * kQuantRowsPerWarp;
  const int rbeg = blockIdx.x * rows_per_block;
  for (int rr = warp; rr < rows_per_block; rr += 8) {
    const int row = rbeg + rr;
    if (row >= M) break;
    const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
    uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(row) * K);
    float amax = 0.0f;
    if constexpr (VPL > 0) {
      uint4 buf[VPL];
#pragma unroll
      for (int t = 0; t < VPL; ++t) {
        const int v = lane + 32 * t;
        if (v < nv) buf[t] = __ldg(src + v);
      }
#pragma unroll
      for (int t = 0; t < VPL; ++t) {
        const int v = lane + 32 * t;
        if (v < nv) amax = fmaxf(amax, masked_absmax8(buf[t], s_bits, v));
      }
      amax = warp_max(amax);
      const float ra = quant_rcp(amax);
#pragma unroll
      for (int t = 0; t < VPL; ++t) {
        const int v = lane + 32 * t;
        if (v < nv) quantize8<false>(buf[t], s_bits, nullptr, v, amax, ra, dst, nullptr);
      }
    } else {
      // Rows longer than the register budget: two passes, the second from L1/L2.
      for (int v = lane; v < nv; v += 32) amax = fmaxf(amax, masked_absmax8(__ldg(src + v), s_bits, v));
      amax = warp_max(amax);
      const float ra = quant_rcp(amax);
      for (int v = lane; v < nv; v += 32)
        quantize8<false>(__ldg(src + v), s_bits, nullptr, v, amax, ra, dst, nullptr);
    }
    if (lane == 0) x_scale[row] = amax;
  }
}

// Host-side dispatch on the register budget VPL (0 = streaming rows).
cudaError_t launch_quantize_rows(int vpl, int grid, size_t smem, cudaStream_t s,
                                 const QuantArgs& a) {
#define I8MM_CASE(V)                                                                       \
  case V:                                                                                  \
    quantize_rows_kernel<V><<<grid, 256, smem, s>>>(a.X, a.M, a.K, a.bitmap, a.Xq, a.x_scale); \
    break;
  switch (vpl) {
    I8MM_CASE(0)
    I8MM_CASE(1)
    I8MM_CASE(2)
    I8MM_CASE(4)
    I8MM_CASE(8)
    I8MM_CASE(16)
    I8MM_CASE(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef I8MM_CASE
  return cudaGetLastError();
}

// sum_k Wq[n, k] per row (the zero-point correction's weight factor), one warp
// per row, exact in int32 (|sum| <= 127 * 65536).
__global__ void weight_rowsum_kernel(const int8_t* __restrict__ Wq, int N, int K,
                                     int32_t* __restrict__ rowsum) {
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  const int8_t* w = Wq + static_cast<size_t>(n) * K;
  int acc = 0;
  for (int k = lane * 16; k < K; k += 32 * 16) {
    const int4 v = *reinterpret_cast<const int4*>(w + k);
    const int vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) acc = __dp4a(vv[i], 0x01010101, acc);
  }
  acc = __reduce_add_sync(0xffffffffu, acc);
  if (lane == 0) rowsum[n] = acc;
}

cudaError_t launch_weight_rowsum(const int8_t* Wq, int N, int K, int32_t* rowsum,
                                 cudaStream_t s) {
  weight_rowsum_kernel<<<(N + 7) / 8, 256, 0, s>>>(Wq, N, K, rowsum);
  return cudaGetLastError();
}

// Offline layout change of the fp16 weight for the outlier product: Wt[k][n] =
// W[n][k]. The LLM.int8() outlier term reads whole input features of the weight
// (AIInfra "05Quantization01", LLM.int8() section: W in h x o orientation, the
// rows W^h of the outlier dimensions h), which are contiguous rows of Wt.
// 32 x 32 tiles through shared memory (one padding column against bank
// conflicts); a block of 32 x 8 threads, four rows each.
__global__ void __launch_bounds__(256) transpose_weight_kernel(const __half* __restrict__ W, int N,
                                                               int K, __half* __restrict__ Wt) {
  __shared__ __half tile[32][33];
  const int n0 = blockIdx.x * 32, k0 = blockIdx.y * 32;   // N blocks in x: N may exceed 65535 * 32
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int n = n0 + j, k = k0 + threadIdx.x;
    if (n < N && k < K) tile[j][threadIdx.x] = W[static_cast<size_t>(n) * K + k];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int k = k0 + j, n = n0 + threadIdx.x;
    if (n < N && k < K) Wt[static_cast<size_t>(k) * N + n] = tile[threadIdx.x][j];
  }
}

cudaError_t launch_transpose_weight(const __half* W, int N, int K, __half* Wt, cudaStream_t s) {
  dim3 grid((N + 31) / 32, (K + 31) / 32);
  transpose_weight_kernel<<<grid, dim3(32, 8), 0, s>>>(W, N, K, Wt);
  return cudaGetLastError();
}

}  // namespace i8mm

// SmoothQuant W8A8 ([Tanjunchen] "quantization explained part 2", section 4):
// per input channel i the activations are divided by s_i and the weights
// multiplied by s_i, s_i = max|X_i|^alpha / max|W_i|^(1-alpha) (section 4.2),
// which leaves X.W unchanged and moves the activation outliers into the
// weights; then both operands are INT8 and the product is a pure INT8 GEMM.
//
// Kernels here:
//   column_absmax_kernel    running per-column max |x| of an fp16 [rows][K]
//                           matrix (calibration activations, or the weight)
//   smooth_factors_kernel   s and r = fl32(1/s) from the two column maxima
//   smooth_weight_kernel    W_hat = fl32(w * s) per column, quantised per row
//   smooth_quantize_kernel  X_hat = fl32(x * r) per column, quantised per token
// and the runtime matmul: smooth_quantize_kernel, then the tcgen05 INT8 GEMM of
// gemm_sm100.cu with its outlier product switched off.
//
// Codes: clamp(rint(fl32(fl32(v*127) / absmax)), +-127) with v the smoothed
// fp32 value: one rounded product and one correctly rounded division (the
// smoothed values are not fp16, so the division-free rule of the LLM.int8()
// kernels, checked for fp16 inputs only, is not used here).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "int8mm.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int sq_code(float v, float a) {
  if (a == 0.0f) return 0;
  const int q = __float2int_rn(__fdiv_rn(__fmul_rn(v, 127.0f), a));
  return max(-127, min(127, q));
}

__device__ __forceinline__ float block_max(float v, float* red) {
  // v >= 0: non-negative floats order like their bit patterns.
  const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = __uint_as_float(w);
  __syncthreads();
  float m = 0.0f;
  for (int i = 0; i < (kThreads >> 5); ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// A CTA covers 256 columns (32 threads of 8-column vectors) of a slice of rows
// (blockIdx.y); its 8 row lanes take every 8th row of the slice, reduce in
// shared memory, and merge with atomicMax on the bit patterns (one atomic per
// column per CTA).
__global__ void __launch_bounds__(kThreads) column_absmax_kernel(const __half* __restrict__ X,
                                                                 int rows, int K, int row_slice,
                                                                 float* __restrict__ colmax) {
  __shared__ uint4 part[8][32];
  const int cv = threadIdx.x & 31;           // vector within the CTA's 32
  const int rl = threadIdx.x >> 5;           // row lane 0..7
  const int v = blockIdx.x * 32 + cv;        // 8-column vector index
  const bool live = v * 8 < K;
  const int r0 = blockIdx.y * row_slice;
  const int r1 = min(rows, r0 + row_slice);
  __half2 m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = __float2half2_rn(0.0f);
  if (live) {
    // Four rows' loads in flight per thread (independent), then their maxima.
    const uint4* col = reinterpret_cast<const uint4*>(X) + v;
    const size_t rstride = static_cast<size_t>(K) / 8;
    for (int r = r0 + rl; r < r1; r += 32) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        u[j] = (r + 8 * j < r1) ? __ldg(col + static_cast<size_t>(r + 8 * j) * rstride)
                                : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&u[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t ab = w[i] & 0x7FFF7FFFu;
          m[i] = __hmax2(m[i], *reinterpret_cast<const __half2*>(&ab));
        }
      }
    }
  }
  part[rl][cv] = *reinterpret_cast<const uint4*>(m);
  __syncthreads();
  if (rl == 0 && live) {
#pragma unroll
    for (int l = 1; l < 8; ++l) {
      const uint4 o = part[l][cv];
      const __half2* h = reinterpret_cast<const __half2*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) m[i] = __hmax2(m[i], h[i]);
    }
    unsigned int* out = reinterpret_cast<unsigned int*>(colmax) + v * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(m[i]);
      if (f.x > 0.0f) atomicMax(out + 2 * i, __float_as_uint(f.x));
      if (f.y > 0.0f) atomicMax(out + 2 * i + 1, __float_as_uint(f.y));
    }
  }
}

__global__ void __launch_bounds__(kThreads) smooth_factors_kernel(const float* __restrict__ act,
                                                                  const float* __restrict__ wmax,
                                                                  int K, float alpha,
                                                                  float* __restrict__ s,
                                                                  float* __restrict__ r) {
  const int i = blockIdx.x * kThreads + threadIdx.x;
  if (i >= K) return;
  const float a = act[i], w = wmax[i];
  float si = 1.0f;   // nothing to migrate on an empty channel
  if (a > 0.0f && w > 0.0f) si = powf(a, alpha) / powf(w, 1.0f - alpha);
  s[i] = si;
  if (r) r[i] = __frcp_rn(si);
}

// One CTA per output row: W_hat = fl32(w * s), row absmax, codes.
__global__ void __launch_bounds__(kThreads) smooth_weight_kernel(const __half* __restrict__ W,
                                                                 const float* __restrict__ s,
                                                                 int K, int8_t* __restrict__ Wq,
                                                                 float* __restrict__ w_scale) {
  __shared__ float red[kThreads / 32];
  const size_t row = blockIdx.x;
  const __half* w = W + row * K;
  float m = 0.0f;
  for (int k = threadIdx.x; k < K; k += kThreads)
    m = fmaxf(m, fabsf(__fmul_rn(__half2float(w[k]), s[k])));
  const float a = block_max(m, red);
  for (int k = threadIdx.x; k < K; k += kThreads)
    Wq[row * K + k] = static_cast<int8_t>(sq_code(__fmul_rn(__half2float(w[k]), s[k]), a));
  if (threadIdx.x == 0) w_scale[row] = a;
}

// One CTA per token row: X_hat = fl32(x * r), row absmax, codes (the smoothed
// values are recomputed in the code pass; the row is L1/L2-resident by then).
__global__ void __launch_bounds__(kThreads) smooth_quantize_kernel(const __half* __restrict__ X,
                                                                   const float* __restrict__ r,
                                                                   int K, int8_t* __restrict__ Xq,
                                                                   float* __restrict__ x_scale) {
  __shared__ float red[kThreads / 32];
  const size_t row = blockIdx.x;
  const __half* x = X + row * K;
  const int nv = K >> 3;                 // 8-column vectors (K % 16 == 0)
  float m = 0.0f;
  for (int v = threadIdx.x; v < nv; v += kThreads) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + 8 * v);
    const __half* h = reinterpret_cast<const __half*>(&u);
    const float4 r0 = __ldg(reinterpret_cast<const float4*>(r + 8 * v));
    const float4 r1 = __ldg(reinterpret_cast<const float4*>(r + 8 * v) + 1);
    const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(__fmul_rn(__half2float(h[i]), rr[i])));
  }
  const float a = block_max(m, red);
  for (int v = threadIdx.x; v < nv; v += kThreads) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + 8 * v);
    const __half* h = reinterpret_cast<const __half*>(&u);
    const float4 r0 = __ldg(reinterpret_cast<const float4*>(r + 8 * v));
    const float4 r1 = __ldg(reinterpret_cast<const float4*>(r + 8 * v) + 1);
    const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    uint32_t b[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      b[i >> 2] |= (static_cast<uint32_t>(sq_code(__fmul_rn(__half2float(h[i]), rr[i]), a)) & 0xFFu)
                   << (8 * (i & 3));
    *reinterpret_cast<uint2*>(Xq + row * K + 8 * v) = make_uint2(b[0], b[1]);
  }
  if (threadIdx.x == 0) x_scale[row] = a;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct SqLayout {
  size_t status, x_scale, Xq, total;
};
SqLayout sq_layout(int M, int K) {
  SqLayout L;
  size_t off = 0;
  L.status = off;  off = align_up(off + 16);
  L.x_scale = off; off = align_up(off + static_cast<size_t>(M) * 4);
  L.Xq = off;      off = align_up(off + static_cast<size_t>(M) * K);
  L.total = off;
  return L;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sq_status(cudaError_t e) { return e == cudaSuccess ? I8MM_OK : I8MM_ERR_CUDA; }

int sq_sizes(int M, int N, int K) {
  if (M < 0 || N < 0 || K <= 0 || (K % 16) != 0 || K > 65536 || M > (1 << 22) || N > (1 << 22))
    return I8MM_ERR_INVALID_ARG;
  return I8MM_OK;
}

}  // namespace

cudaError_t launch_column_absmax(const __half* X, int rows, int K, float* colmax,
                                 cudaStream_t s) {
  const int nv = K / 8;
  const int col_blocks = (nv + 31) / 32;
  // about two CTAs per SM over the whole matrix (fewer slices, fewer atomics),
  // at least 8 rows per slice
  int slices = (2 * 148 + col_blocks - 1) / col_blocks;
  int row_slice = (rows + slices - 1) / slices;
  row_slice = row_slice < 8 ? 8 : row_slice;
  dim3 grid(col_blocks, (rows + row_slice - 1) / row_slice);
  column_absmax_kernel<<<grid, kThreads, 0, s>>>(X, rows, K, row_slice, colmax);
  return cudaGetLastError();
}

}  // namespace i8mm

using namespace i8mm;

extern "C" {

int int8_column_absmax(const void* X, int rows, int K, float* colmax, i8mm_stream_t stream) {
  if (sq_sizes(rows, 1, K) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (rows == 0) return I8MM_OK;
  if (!X || !colmax) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || !a16(colmax)) return I8MM_ERR_ALIGNMENT;
  return sq_status(launch_column_absmax(static_cast<const __half*>(X), rows, K, colmax,
                                        static_cast<cudaStream_t>(stream)));
}

int int8_smoothquant_factors(const float* act_absmax, const float* w_absmax, int K, float alpha,
                             float* s, float* s_rcp, i8mm_stream_t stream) {
  if (K <= 0 || !(alpha >= 0.0f && alpha <= 1.0f)) return I8MM_ERR_INVALID_ARG;
  if (!act_absmax || !w_absmax || !s) return I8MM_ERR_INVALID_ARG;
  smooth_factors_kernel<<<(K + kThreads - 1) / kThreads, kThreads, 0,
                          static_cast<cudaStream_t>(stream)>>>(act_absmax, w_absmax, K, alpha, s,
                                                               s_rcp);
  return sq_status(cudaGetLastError());
}

int int8_smoothquant_weight_rows(const void* W, const float* s, int N, int K, int8_t* Wq,
                                 float* w_scale, i8mm_stream_t stream) {
  if (sq_sizes(1, N, K) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (N == 0) return I8MM_OK;
  if (!W || !s || !Wq || !w_scale) return I8MM_ERR_INVALID_ARG;
  smooth_weight_kernel<<<N, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half*>(W), s, K, Wq, w_scale);
  return sq_status(cudaGetLastError());
}

size_t int8_smoothquant_workspace_size(int M, int N, int K) {
  if (sq_sizes(M, N, K) != I8MM_OK) return 0;
  return sq_layout(M, K).total;
}

int int8_smoothquant_matmul(const void* X, const int8_t* Wq, const float* w_scale,
                            const float* s_rcp, int M, int N, int K, void* Y, void* workspace,
                            size_t workspace_bytes, i8mm_stream_t stream) {
  if (sq_sizes(M, N, K) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!X || !Wq || !w_scale || !s_rcp || !Y || !workspace) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || !a16(Wq) || !a16(w_scale) || !a16(s_rcp) || !a16(Y)) return I8MM_ERR_ALIGNMENT;
  const SqLayout L = sq_layout(M, K);
  if (workspace_bytes < L.total) return I8MM_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return I8MM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  float* xs = reinterpret_cast<float*>(ws + L.x_scale);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.Xq);
  cudaError_t e = cudaMemsetAsync(status, 0, 16, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  smooth_quantize_kernel<<<M, kThreads, 0, st>>>(static_cast<const __half*>(X), s_rcp, K, Xq, xs);
  e = cudaGetLastError();
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  GemmArgs g{};
  g.Xq = Xq;
  g.Wq = Wq;
  g.x_scale = xs;
  g.w_scale = w_scale;
  g.n_outliers = nullptr;   // pure INT8 product: no outlier pass
  g.out = Y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.status = status;
  g.ld = 64;
  return sq_status(launch_gemm_mixed(g, st));
}

}  // extern "C"

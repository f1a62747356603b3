// Memory-bound kernels of the LLM.int8() path on sm_100a:
//   * quantize_weight_rows_kernel  - offline per-output-row absmax INT8 codes of W
//   * detect_outliers_kernel        - outlier-column bitmap of X (|x| > threshold),
//                                     finished by the last CTA into a count and the
//                                     ascending column list (stand-alone entry point)
//   * quantize_rows_kernel          - per-token absmax over the non-outlier columns and
//                                     INT8 codes, 0 at outliers (stand-alone entry point)
//   * detect_quantize_compact_kernel - the fused, cooperative form of both used by
//                                     the full path, which also compacts the fp16
//                                     outlier columns of X and W into dense panels
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

namespace i8mm {

namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// clamp(rint((x*127)/a), -127, 127): one exact fp32 product, one IEEE divide,
// round half to even. a == 0 gives 0.
__device__ __forceinline__ int quant_code(float x, float a) {
  if (a == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(__fmul_rn(x, 127.0f), a));
  return max(-127, min(127, q));
}

// The same code without a division on the common path: with inv = fl(127/a),
// y = fl(x*inv) is within 127*(2^-23 + 2^-48) < 1.6e-5 of the exact quotient
// t = x*127/a, and fl(t) within 127*2^-24 < 7.6e-6 of t, so y and fl(t) are less
// than 2.3e-5 apart. Unless y lies within 6.2e-5 of a half-integer, both round
// to the same integer; near a half-integer the correctly rounded quotient is
// formed exactly as quant_code does. Needs |x| <= a (true for every non-outlier
// entry of a row, since a is their absmax).
__device__ __forceinline__ int quant_code_fast(float x, float a, float inv) {
  if (a == 0.0f) return 0;
  const float y = __fmul_rn(x, inv);
  const float r = rintf(y);
  int q;
  if (fabsf(y - r) <= 0.5f - 6.2e-5f)
    q = static_cast<int>(r);
  else
    q = __float2int_rn(__fdiv_rn(__fmul_rn(x, 127.0f), a));
  return max(-127, min(127, q));
}

__device__ __forceinline__ float quant_inv(float a) {
  return a == 0.0f ? 0.0f : __fdiv_rn(127.0f, a);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Absmax of the non-outlier entries among the 8 columns 8v..8v+7.
__device__ __forceinline__ float masked_absmax8(const uint4& u, const uint32_t* s_bits, int v) {
  const uint32_t m8 = (s_bits[v >> 2] >> (8 * (v & 3))) & 0xFFu;
  float f[8];
  unpack8(u, f);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (!((m8 >> i) & 1u)) a = fmaxf(a, fabsf(f[i]));
  return a;
}

// Codes of the 8 columns 8v..8v+7 (0 at outliers); with COMPACT the outlier
// entries are also copied to their compacted position in the X_O row.
template <bool COMPACT>
__device__ __forceinline__ void quantize8(const uint4& u, const uint32_t* s_bits,
                                          const int32_t* s_prefix, int v, float amax, float inv,
                                          uint2* dst, __half* xo_row) {
  const uint32_t wbits = s_bits[v >> 2];
  const uint32_t m8 = (wbits >> (8 * (v & 3))) & 0xFFu;
  float f[8];
  unpack8(u, f);
  int q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = ((m8 >> i) & 1u) ? 0 : quant_code_fast(f[i], amax, inv);
  uint2 o;
  o.x = pack4(q[0], q[1], q[2], q[3]);
  o.y = pack4(q[4], q[5], q[6], q[7]);
  dst[v] = o;
  if (COMPACT && m8) {
    const __half* hv = reinterpret_cast<const __half*>(&u);
    const int base = s_prefix[v >> 2];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((m8 >> i) & 1u) {
        const int bit = 8 * (v & 3) + i;
        xo_row[base + __popc(wbits & ((1u << bit) - 1u))] = hv[i];
      }
    }
  }
}

}  // namespace

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
      const float inv = quant_inv(amax);
#pragma unroll
      for (int t = 0; t < VPL; ++t) {
        const int v = lane + 32 * t;
        if (v < nv) quantize8<false>(buf[t], s_bits, nullptr, v, amax, inv, dst, nullptr);
      }
    } else {
      // Rows longer than the register budget: two passes, the second from L1/L2.
      for (int v = lane; v < nv; v += 32) amax = fmaxf(amax, masked_absmax8(__ldg(src + v), s_bits, v));
      amax = warp_max(amax);
      const float inv = quant_inv(amax);
      for (int v = lane; v < nv; v += 32)
        quantize8<false>(__ldg(src + v), s_bits, nullptr, v, amax, inv, dst, nullptr);
    }
    if (lane == 0) x_scale[row] = amax;
  }
}

// ---------------------------------------------------------------------------
// Fused detection + quantisation + compaction for the full path, one
// cooperative launch (all CTAs co-resident). Each CTA owns a contiguous block
// of rows of X and a contiguous block of rows of W.
//   phase A  stream the CTA's rows of X once from HBM; per column |x| > thr
//            flags, OR-ed into the global bitmap (atomics only for non-zero words)
//   barrier  grid-wide arrival counter with a bounded wait
//   phase B  bitmap -> per-word prefix and the ascending outlier list in shared
//            memory (CTA 0 also publishes count and list); re-read the rows (now
//            L2-resident), per-row absmax over non-outlier columns, INT8 codes,
//            compacted X_O row; then gather the outlier columns of the CTA's W rows
//            into W_O.
// Thread t of the 512 owns the 16-byte vectors v = t + 512*c (c < VPT) of a row.
// ---------------------------------------------------------------------------
namespace {

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kRowGroup = 4;            // rows processed together in phase B
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

}  // namespace

template <int VPT>
__global__ void __launch_bounds__(kFusedThreads) detect_quantize_compact_kernel(FusedArgs a) {
  extern __shared__ __align__(16) uint8_t fsm[];
  const int K = a.K;
  const int words = (K + 31) >> 5;
  const int nv = K >> 3;
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(fsm);
  int32_t* s_prefix = reinterpret_cast<int32_t*>(s_bits + words);
  float* s_red = reinterpret_cast<float*>(s_prefix + words);           // [kFusedWarps][kRowGroup]
  int32_t* s_misc = reinterpret_cast<int32_t*>(s_red + kFusedWarps * kRowGroup);  // [0] carry
  uint16_t* s_idx = reinterpret_cast<uint16_t*>(s_misc + 4);           // [K] outlier columns
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int rows_per = (a.M + gridDim.x - 1) / gridDim.x;
  const int r0 = min(a.M, static_cast<int>(blockIdx.x) * rows_per);
  const int r1 = min(a.M, r0 + rows_per);

  // ---------------- phase A: column flags over this CTA's rows
  // RGA rows are loaded together so each thread keeps RGA*VPT loads in flight.
  constexpr int RGA = VPT >= 8 ? 1 : 8 / VPT;
  uint32_t flags[VPT];
#pragma unroll
  for (int c = 0; c < VPT; ++c) flags[c] = 0;
  for (int r = r0; r < r1; r += RGA) {
    uint4 u[RGA][VPT];
#pragma unroll
    for (int g = 0; g < RGA; ++g)
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        const int v = tid + kFusedThreads * c;
        u[g][c] = make_uint4(0, 0, 0, 0);
        if (r + g < r1 && v < nv)
          u[g][c] = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(r + g) * K) + v);
      }
#pragma unroll
    for (int g = 0; g < RGA; ++g)
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        float f[8];
        unpack8(u[g][c], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) flags[c] |= (fabsf(f[i]) > a.threshold ? 1u : 0u) << i;
      }
  }
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    const int v = tid + kFusedThreads * c;
    uint32_t word = flags[c] << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if ((lane & 3) == 0 && v < nv && word != 0) atomicOr(a.bitmap + (v >> 2), word);
  }

  // ---------------- grid barrier (bounded)
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(a.sync_ctr, 1);
    const uint64_t t0 = gtimer();
    while (ld_acquire(a.sync_ctr) < static_cast<int>(gridDim.x)) {
      __nanosleep(64);
      if (gtimer() - t0 > kBarrierLimitNs) {
        atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();

  // ---------------- phase B.1: bitmap, prefix and outlier list in shared memory
  if (tid == 0) s_misc[0] = 0;
  __syncthreads();
  for (int base = 0; base < words; base += kFusedThreads) {
    const int w = base + tid;
    const uint32_t bits = (w < words) ? __ldcg(a.bitmap + w) : 0u;
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_red[warp] = __int_as_float(incl);
    __syncthreads();
    int wsum = 0;
    for (int i = 0; i < warp; ++i) wsum += __float_as_int(s_red[i]);
    const int excl = s_misc[0] + wsum + incl - cnt;
    if (w < words) {
      s_bits[w] = bits;
      s_prefix[w] = excl;
      uint32_t b = bits;
      int p = excl;
      while (b) {
        const int j = __ffs(b) - 1;
        b &= b - 1;
        s_idx[p++] = static_cast<uint16_t>(w * 32 + j);
      }
    }
    __syncthreads();
    if (tid == kFusedThreads - 1) s_misc[0] = excl + cnt;
    __syncthreads();
  }
  const int count = s_misc[0];
  const int pad = (count + 63) & ~63;
  if (blockIdx.x == 0) {
    for (int p = tid; p < count; p += kFusedThreads) a.col_idx[p] = s_idx[p];
    if (tid == 0) *a.n_outliers = count;
  }

  // ---------------- phase B.2: quantise this CTA's rows (L2-resident now)
  constexpr int RGB = VPT >= 4 ? 1 : 4 / VPT;
  for (int rb = r0; rb < r1; rb += RGB) {
    const int ng = min(RGB, r1 - rb);
    uint4 u[RGB][VPT];
    float am[RGB];
#pragma unroll
    for (int g = 0; g < RGB; ++g) {
      am[g] = 0.0f;
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        const int v = tid + kFusedThreads * c;
        if (g < ng && v < nv)
          u[g][c] = __ldcg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(rb + g) * K) + v);
      }
    }
#pragma unroll
    for (int g = 0; g < RGB; ++g)
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        const int v = tid + kFusedThreads * c;
        if (g < ng && v < nv) am[g] = fmaxf(am[g], masked_absmax8(u[g][c], s_bits, v));
      }
#pragma unroll
    for (int g = 0; g < RGB; ++g) {
      am[g] = warp_max(am[g]);
      if (lane == 0) s_red[warp * kRowGroup + g] = am[g];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < RGB; ++g) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < kFusedWarps; ++i) m = fmaxf(m, s_red[i * kRowGroup + g]);
      am[g] = m;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < RGB; ++g) {
      if (g >= ng) break;
      const int row = rb + g;
      uint2* dst = reinterpret_cast<uint2*>(a.Xq + static_cast<size_t>(row) * K);
      __half* xo_row = a.X_O + static_cast<size_t>(row) * a.ld;
      const float inv = quant_inv(am[g]);
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        const int v = tid + kFusedThreads * c;
        if (v < nv) quantize8<true>(u[g][c], s_bits, s_prefix, v, am[g], inv, dst, xo_row);
      }
      for (int p = count + tid; p < pad; p += kFusedThreads) xo_row[p] = __float2half_rn(0.0f);
      if (tid == 0) a.x_scale[row] = am[g];
    }
  }

  // ---------------- phase B.3: W_O rows of this CTA (outlier columns of W)
  if (pad > 0) {
    const int nper = (a.N + gridDim.x - 1) / gridDim.x;
    const int n0 = min(a.N, static_cast<int>(blockIdx.x) * nper);
    const int n1 = min(a.N, n0 + nper);
    const int total = (n1 - n0) * pad;
    for (int e = tid; e < total; e += kFusedThreads) {
      const int n = n0 + e / pad;
      const int p = e - (n - n0) * pad;
      __half val = __float2half_rn(0.0f);
      if (p < count) val = a.W[static_cast<size_t>(n) * K + s_idx[p]];
      a.W_O[static_cast<size_t>(n) * a.ld + p] = val;
    }
  }
}

size_t fused_smem_bytes(int K) {
  const size_t words = static_cast<size_t>((K + 31) / 32);
  return words * 8 + kFusedWarps * kRowGroup * 4 + 16 + static_cast<size_t>(K) * 2 + 16;
}

int fused_vpt(int K) {
  const int nv = K / 8;
  if (nv <= kFusedThreads) return 1;
  if (nv <= 2 * kFusedThreads) return 2;
  if (nv <= 4 * kFusedThreads) return 4;
  if (nv <= 8 * kFusedThreads) return 8;
  return 16;
}

cudaError_t launch_detect_quantize_compact(const FusedArgs& a, cudaStream_t s) {
  const int vpt = fused_vpt(a.K);
  const size_t smem = fused_smem_bytes(a.K);
  const void* fn = nullptr;
  switch (vpt) {
    case 1: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<1>); break;
    case 2: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<2>); break;
    case 4: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<4>); break;
    case 8: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<8>); break;
    default: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<16>); break;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0, sms = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // Enough CTAs to keep every SM streaming, but not more than can be co-resident.
  int grid = per_sm * sms;
  const int want = max((a.M + 1) / 2, (a.N + 15) / 16);
  grid = max(1, min(grid, want));
  FusedArgs args = a;
  void* params[] = {&args};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kFusedThreads), params, smem, s);
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

}  // namespace i8mm

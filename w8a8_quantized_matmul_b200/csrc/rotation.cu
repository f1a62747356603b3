// Grouped Hadamard rotation before quantisation ([Baidu] developer.baidu.com
// "分组旋转方法从W8A8到W4A4", sections 2, 5.1, 5.2, 5.4).
//
// Y = X W^T is unchanged when both operands are multiplied along K by the
// block-diagonal orthogonal R = blockdiag(H_G / sqrt(G)), H_G the Sylvester
// Hadamard matrix (H[i][j] = (-1)^popcount(i & j)). The rotation spreads an
// outlier channel over its group of G columns, so the absmax scales shrink.
//
// Rotated value of an fp16 row: r = fl32(fl32(S) * c) with S the exact +-1
// sum over the group and c = fl32(1/sqrt(G)). S is formed by the fast
// Walsh-Hadamard butterfly in float64: every partial sum of at most 256 fp16
// values is a multiple of 2^-24 below 2^24 in magnitude, so every float64 add
// is exact and the order of the butterfly does not matter.
//
// Thread layout: a thread holds 16 consecutive columns of a row (two uint4
// loads); stages on column bits 0..3 run in registers, stages on bits 4.. run
// across the G/16 lanes of the group with shuffles.
//
// Kernels:
//   rotate_rows_kernel    W8A8: rotate, one absmax per row over all K (rotated
//                         values staged in shared memory), INT8 codes; serves
//                         the activations at run time and the weight offline
//   rotate_groups_kernel  W4A4: rotate, one absmax per (row, group) (the group
//                         max is a shuffle over the group's lanes), 4-bit codes
//                         as int8 and/or packed eight per uint32; with
//                         BLOCK_MAX it only folds the group maxima into the
//                         G x G block maxima of a weight (pass 1 of the weight
//                         quantiser), with BLOCK_SCALE it codes against those
//                         block maxima (pass 2)
// Codes: clamp(rint(fl32(fl32(r * qmax) / a)), -qmax, qmax), a = 0 giving 0.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "int8mm.h"
#include "kernels.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace i8mm {

namespace {

constexpr int kRowThreads = 512;
constexpr int kMaxRotK = 32768;

__device__ __forceinline__ int rot_code(float r, float a, float qmax) {
  if (a == 0.0f) return 0;
  const int q = __float2int_rn(__fdiv_rn(__fmul_rn(r, qmax), a));
  const int m = static_cast<int>(qmax);
  return max(-m, min(m, q));
}

// fp16 -> fp64 in one conversion (exact).
__device__ __forceinline__ double h2d(__half h) {
  double d;
  asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(__half_as_ushort(h)));
  return d;
}

// The 16 rotated values of columns [16p, 16p + 16) of a row, p = piece index;
// lanes of one group of G columns hold consecutive pieces. `live` false gives
// zeros (a piece past the end of the row; whole groups only).
template <int G>
__device__ __forceinline__ void rotate16(const __half* __restrict__ src, bool live, float c,
                                         float (&r)[16]) {
  double v[16];
  if (live) {
    const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const __half* h0 = reinterpret_cast<const __half*>(&u0);
    const __half* h1 = reinterpret_cast<const __half*>(&u1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = h2d(h0[i]);
      v[8 + i] = h2d(h1[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.0;
  }
#pragma unroll
  for (int h = 1; h < 16 && h < G; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (!(i & h)) {
        const double a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 1; s < G / 16; s <<= 1) {
    // lower lane: v + p; upper lane: p - v; one exact FMA by +-1 either way
    const double sg = (lane & s) ? -1.0 : 1.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fma_rn(sg, v[i], __shfl_xor_sync(0xffffffffu, v[i], s));
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = __fmul_rn(__double2float_rn(v[i]), c);
}

// Codes of 16 rotated values against the absmax a of their group, ra =
// quant_rcp(a): q = rint(fl32(n / a)) with n = fl32(r * qmax). The quotient is
// formed without a division: q0 = fl(n * ra), e = fma(q0, -a, n) (exact),
// qc = fma(e, ra, q0), within about one ulp of n / a. Where qc lies within
// about 2^-15 (four ulps at |q| < 128) of a half-integer the correctly rounded
// quotient could round the other way, so those codes are recomputed with a
// correctly rounded division; everywhere else rint(qc) is the code. rint is
// the low bits of fl(qc + 1.5 * 2^23) (ties to even); the near-tie test is
// |t^2 - 1/4| < 2^-15 with t = qc - rint(qc) (exact), i.e. ||t| - 1/2| < ~2^-15.
// The codes come back packed, four bytes per word.
__device__ __forceinline__ void rot_codes16(const float (&r)[16], float a, float ra, float qmax,
                                            uint32_t (&b)[4]) {
  const uint64_t na2 = f2pack(-a, -a), ra2 = f2pack(ra, ra), qm2 = f2pack(qmax, qmax);
  const uint64_t mg2 = f2pack(kMagic, kMagic), nq2 = f2pack(-0.25f, -0.25f);
  bool tie = false;
  uint32_t lo16[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint64_t n = mul2(f2pack(r[2 * j], r[2 * j + 1]), qm2);
    const uint64_t q0 = mul2(n, ra2);
    const uint64_t qc = fma2(fma2(q0, na2, n), ra2, q0);
    const uint64_t sm = add2(qc, mg2);
    const uint64_t t = sub2(qc, sub2(sm, mg2));            // qc - rint(qc), exact
    const uint64_t d = fma2(t, t, nq2);                    // t^2 - 1/4
    tie |= fabsf(lo(d)) < 0x1p-15f;
    tie |= fabsf(hi(d)) < 0x1p-15f;
    lo16[j] = __byte_perm(static_cast<uint32_t>(sm), static_cast<uint32_t>(sm >> 32), 0x0040);
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) b[w] = __byte_perm(lo16[2 * w], lo16[2 * w + 1], 0x5410);
  if (tie) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      b[w] = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        b[w] |= (static_cast<uint32_t>(rot_code(r[4 * w + i], a, qmax)) & 0xFFu) << (8 * i);
    }
  }
}

__device__ __forceinline__ void store_codes16(const uint32_t (&b)[4], int8_t* dst) {
  *reinterpret_cast<uint4*>(dst) = make_uint4(b[0], b[1], b[2], b[3]);
}

__device__ __forceinline__ float max16(const float (&r)[16]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(r[i]));
  return m;
}

// One CTA per row; pieces p = it * blockDim.x + tid. A row of at most
// blockDim.x pieces keeps its rotated values in registers; a longer row stages
// them in shared memory. Then the row max (warp redux, then across warps) and
// the codes.
template <int G>
__global__ void __launch_bounds__(kRowThreads) rotate_rows_kernel(
    const __half* __restrict__ X, int K, float c, int8_t* __restrict__ Xq,
    float* __restrict__ scale, float* __restrict__ R) {
  extern __shared__ float4 rot_smem[];
  float* rs = reinterpret_cast<float*>(rot_smem);
  __shared__ float red[kRowThreads / 32];
  const size_t row = blockIdx.x;
  const int np = K >> 4;
  const int nt = blockDim.x;
  const bool single = np <= nt;
  float r[16];
  float m = 0.0f;
  for (int base = 0; base < np; base += nt) {
    const int p = base + threadIdx.x;
    rotate16<G>(X + row * K + 16 * p, p < np, c, r);
    if (p < np) {
      m = fmaxf(m, max16(r));
      if (!single) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(rs + 16 * p)[i] = make_float4(r[4 * i], r[4 * i + 1],
                                                                 r[4 * i + 2], r[4 * i + 3]);
      }
    }
  }
  const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = __uint_as_float(w);
  __syncthreads();
  float a = 0.0f;
  for (int i = 0; i < (nt >> 5); ++i) a = fmaxf(a, red[i]);
  const float ra = a == 0.0f ? 0.0f : __frcp_rn(a);
  for (int p = threadIdx.x; p < np; p += nt) {
    if (!single) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = reinterpret_cast<const float4*>(rs + 16 * p)[i];
        r[4 * i] = f.x; r[4 * i + 1] = f.y; r[4 * i + 2] = f.z; r[4 * i + 3] = f.w;
      }
    }
    uint32_t q[4];
    rot_codes16(r, a, ra, 127.0f, q);
    store_codes16(q, Xq + row * K + 16 * p);
    if (R) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(R + row * K + 16 * p)[i] =
            make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    }
  }
  if (threadIdx.x == 0) scale[row] = a;
}

enum GroupMode { kActGroups = 0, kBlockMax = 1, kBlockScale = 2 };

// Grid (rows, ceil(np / 256)); 256 threads, one piece each. Group maxima by a
// shuffle over the G/16 lanes of the group.
template <int G, int MODE>
__global__ void __launch_bounds__(256) rotate_groups_kernel(
    const __half* __restrict__ X, int K, float c, int8_t* __restrict__ Xq,
    uint32_t* __restrict__ Xp, float* __restrict__ scale) {
  const size_t row = blockIdx.x;
  const int np = K >> 4;
  const int p = blockIdx.y * 256 + threadIdx.x;
  const bool live = p < np;
  float r[16];
  rotate16<G>(X + row * K + 16 * (live ? p : 0), live, c, r);
  float m = max16(r);
#pragma unroll
  for (int s = 1; s < G / 16; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
  if (!live) return;
  const int ng = K / G;
  const int g = (16 * p) / G;
  const bool first = ((16 * p) % G) == 0;
  if (MODE == kBlockMax) {
    if (first && m > 0.0f)
      atomicMax(reinterpret_cast<unsigned int*>(scale) + (row / G) * ng + g, __float_as_uint(m));
    return;
  }
  float a = m;
  if (MODE == kActGroups) {
    if (first) scale[row * ng + g] = m;
  } else {
    a = __ldg(scale + (row / G) * ng + g);
  }
  uint32_t q[4];
  rot_codes16(r, a, a == 0.0f ? 0.0f : __frcp_rn(a), 7.0f, q);
  if (Xq) store_codes16(q, Xq + row * K + 16 * p);
  if (Xp) {
    // bytes (two's complement, |q| <= 7) to nibbles: code i of byte word w
    uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w0 |= ((q[i >> 2] >> (8 * (i & 3))) & 0xFu) << (4 * i);
      w1 |= ((q[2 + (i >> 2)] >> (8 * (i & 3))) & 0xFu) << (4 * i);
    }
    *reinterpret_cast<uint2*>(Xp + row * (K / 8) + 2 * p) = make_uint2(w0, w1);
  }
}

// Packed 4-bit codes (eight per uint32, code j in bits 4j..4j+3) to one signed
// byte each; one thread per 16-byte group of four words (32 codes).
__global__ void __launch_bounds__(256) unpack_int4_kernel(const uint4* __restrict__ P,
                                                          size_t n_quads, uint4* __restrict__ Q) {
  for (size_t i = blockIdx.x * 256ull + threadIdx.x; i < n_quads; i += gridDim.x * 256ull) {
    const uint4 w = __ldg(P + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // nibbles 0..3 and 4..7 of the word into bytes, then sign-extend each byte
      const uint32_t lo4 = ws[k] & 0xFFFFu, hi4 = ws[k] >> 16;
      uint32_t a = (lo4 & 0xFu) | ((lo4 & 0xF0u) << 4) | ((lo4 & 0xF00u) << 8) | ((lo4 & 0xF000u) << 12);
      uint32_t b = (hi4 & 0xFu) | ((hi4 & 0xF0u) << 4) | ((hi4 & 0xF00u) << 8) | ((hi4 & 0xF000u) << 12);
      // a byte x in 0..15 becomes x - 16 when bit 3 is set: (x ^ 8) - 8 per byte
      a = ((a ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;
      b = ((b ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;
      o[2 * k] = a;
      o[2 * k + 1] = b;
    }
    Q[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    Q[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

float rot_scale(int G) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(G))); }

bool rot_group_ok(int G) { return G >= 16 && G <= 256 && (G & (G - 1)) == 0; }

template <int G>
cudaError_t launch_rows_g(const __half* X, int rows, int K, int8_t* Xq, float* scale, float* R,
                          cudaStream_t s) {
  const int np = K / 16;
  int nt = ((np + 31) / 32) * 32;
  if (nt > kRowThreads) nt = kRowThreads;
  // A row of at most nt pieces keeps its rotated values in registers.
  const size_t smem = np <= nt ? 0 : static_cast<size_t>(K) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(rotate_rows_kernel<G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  rotate_rows_kernel<G><<<rows, nt, smem, s>>>(X, K, rot_scale(G), Xq, scale, R);
  return cudaGetLastError();
}

template <int G, int MODE>
cudaError_t launch_groups_g(const __half* X, int rows, int K, int8_t* Xq, uint32_t* Xp,
                            float* scale, cudaStream_t s) {
  const int np = K / 16;
  dim3 grid(rows, (np + 255) / 256);
  rotate_groups_kernel<G, MODE><<<grid, 256, 0, s>>>(X, K, rot_scale(G), Xq, Xp, scale);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_groups(const __half* X, int rows, int K, int G, int8_t* Xq, uint32_t* Xp,
                          float* scale, cudaStream_t s) {
  switch (G) {
    case 16: return launch_groups_g<16, MODE>(X, rows, K, Xq, Xp, scale, s);
    case 32: return launch_groups_g<32, MODE>(X, rows, K, Xq, Xp, scale, s);
    case 64: return launch_groups_g<64, MODE>(X, rows, K, Xq, Xp, scale, s);
    case 128: return launch_groups_g<128, MODE>(X, rows, K, Xq, Xp, scale, s);
    default: return launch_groups_g<256, MODE>(X, rows, K, Xq, Xp, scale, s);
  }
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct RotLayout {
  size_t status, x_scale, Xq, total;
};
RotLayout rot_layout(int M, int K) {
  RotLayout L;
  size_t off = 0;
  L.status = off;  off = align_up(off + 16);
  L.x_scale = off; off = align_up(off + static_cast<size_t>(M) * 4);
  L.Xq = off;      off = align_up(off + static_cast<size_t>(M) * K);
  L.total = off;
  return L;
}

struct R4Layout {
  size_t status, x_absmax, Xq, total;
};
R4Layout r4_layout(int M, int K, int G) {
  R4Layout L;
  size_t off = 0;
  L.status = off;   off = align_up(off + 16);
  L.x_absmax = off; off = align_up(off + static_cast<size_t>(M) * (K / G) * 4);
  L.Xq = off;       off = align_up(off + static_cast<size_t>(M) * K);
  L.total = off;
  return L;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int rot_status(cudaError_t e) { return e == cudaSuccess ? I8MM_OK : I8MM_ERR_CUDA; }

int rot_sizes(int M, int N, int K, int G) {
  if (M < 0 || N < 0 || K <= 0 || K > kMaxRotK || M > (1 << 22) || N > (1 << 22))
    return I8MM_ERR_INVALID_ARG;
  if (!rot_group_ok(G) || (K % G) != 0) return I8MM_ERR_INVALID_ARG;
  return I8MM_OK;
}

}  // namespace

cudaError_t launch_rotate_rows(const __half* X, int rows, int K, int G, int8_t* Xq, float* scale,
                               float* R, cudaStream_t s) {
  switch (G) {
    case 16: return launch_rows_g<16>(X, rows, K, Xq, scale, R, s);
    case 32: return launch_rows_g<32>(X, rows, K, Xq, scale, R, s);
    case 64: return launch_rows_g<64>(X, rows, K, Xq, scale, R, s);
    case 128: return launch_rows_g<128>(X, rows, K, Xq, scale, R, s);
    default: return launch_rows_g<256>(X, rows, K, Xq, scale, R, s);
  }
}

cudaError_t launch_rotate_groups(const __half* X, int rows, int K, int G, int8_t* Xq,
                                 uint32_t* Xp, float* scale, cudaStream_t s) {
  return launch_groups<kActGroups>(X, rows, K, G, Xq, Xp, scale, s);
}

}  // namespace i8mm

using namespace i8mm;

extern "C" {

int int8_rotate_quantize_rows(const void* X, int rows, int K, int G, int8_t* Xq, float* absmax,
                              float* R, i8mm_stream_t stream) {
  if (rot_sizes(rows, 1, K, G) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (rows == 0) return I8MM_OK;
  if (!X || !Xq || !absmax) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || !a16(Xq) || (R && !a16(R))) return I8MM_ERR_ALIGNMENT;
  return rot_status(launch_rotate_rows(static_cast<const __half*>(X), rows, K, G, Xq, absmax, R,
                                       static_cast<cudaStream_t>(stream)));
}

size_t int8_rotated_workspace_size(int M, int N, int K) {
  if (M < 0 || N < 0 || K <= 0 || K > kMaxRotK) return 0;
  return rot_layout(M, K).total;
}

int int8_rotated_matmul(const void* X, const int8_t* Wq, const float* w_scale, int M, int N, int K,
                        int G, void* Y, void* workspace, size_t workspace_bytes,
                        i8mm_stream_t stream) {
  if (rot_sizes(M, N, K, G) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!X || !Wq || !w_scale || !Y || !workspace) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || !a16(Wq) || !a16(w_scale) || !a16(Y)) return I8MM_ERR_ALIGNMENT;
  const RotLayout L = rot_layout(M, K);
  if (workspace_bytes < L.total) return I8MM_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return I8MM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  float* xs = reinterpret_cast<float*>(ws + L.x_scale);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.Xq);
  cudaError_t e = cudaMemsetAsync(status, 0, 16, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  e = launch_rotate_rows(static_cast<const __half*>(X), M, K, G, Xq, xs, nullptr, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  GemmArgs g{};
  g.Xq = Xq;
  g.Wq = Wq;
  g.x_scale = xs;
  g.w_scale = w_scale;
  g.n_outliers = nullptr;   // every column goes through the INT8 product
  g.out = Y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.status = status;
  g.ld = 64;
  return rot_status(launch_gemm_mixed(g, st));
}

int int4_rotate_quantize_groups(const void* X, int rows, int K, int G, int8_t* Xq, uint32_t* Xp,
                                float* absmax, i8mm_stream_t stream) {
  if (rot_sizes(rows, 1, K, G) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (rows == 0) return I8MM_OK;
  if (!X || !absmax || (!Xq && !Xp)) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || (Xq && !a16(Xq)) || (Xp && (reinterpret_cast<uintptr_t>(Xp) & 7u)))
    return I8MM_ERR_ALIGNMENT;
  return rot_status(launch_rotate_groups(static_cast<const __half*>(X), rows, K, G, Xq, Xp,
                                         absmax, static_cast<cudaStream_t>(stream)));
}

int int4_rotate_quantize_weight_blocks(const void* W, int N, int K, int G, uint32_t* Wp,
                                       float* absmax, i8mm_stream_t stream) {
  if (rot_sizes(1, N, K, G) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (N % G != 0) return I8MM_ERR_INVALID_ARG;
  if (N == 0) return I8MM_OK;
  if (!W || !Wp || !absmax) return I8MM_ERR_INVALID_ARG;
  if (!a16(W) || (reinterpret_cast<uintptr_t>(Wp) & 7u)) return I8MM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half* w = static_cast<const __half*>(W);
  cudaError_t e = cudaMemsetAsync(absmax, 0, static_cast<size_t>(N / G) * (K / G) * 4, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  e = launch_groups<kBlockMax>(w, N, K, G, nullptr, nullptr, absmax, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  return rot_status(launch_groups<kBlockScale>(w, N, K, G, nullptr, Wp, absmax, st));
}

int int4_unpack(const uint32_t* P, int rows, int K, int8_t* Q, i8mm_stream_t stream) {
  if (rows < 0 || K <= 0 || (K % 32) != 0) return I8MM_ERR_INVALID_ARG;
  if (rows == 0) return I8MM_OK;
  if (!P || !Q) return I8MM_ERR_INVALID_ARG;
  if (!a16(P) || !a16(Q)) return I8MM_ERR_ALIGNMENT;
  const size_t quads = static_cast<size_t>(rows) * (K / 32);
  size_t blocks = (quads + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  unpack_int4_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(P), quads, reinterpret_cast<uint4*>(Q));
  return rot_status(cudaGetLastError());
}

size_t int4_rotated_workspace_size(int M, int N, int K, int G) {
  if (rot_sizes(M, N, K, G) != I8MM_OK) return 0;
  return r4_layout(M, K, G).total;
}

int int4_rotated_matmul(const void* X, const int8_t* Wq4, const float* w_absmax, int M, int N,
                        int K, int G, void* Y, void* workspace, size_t workspace_bytes,
                        i8mm_stream_t stream) {
  if (rot_sizes(M, N, K, G) != I8MM_OK) return I8MM_ERR_INVALID_ARG;
  if (G < 64 || (K % 128) != 0 || (N % G) != 0) return I8MM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!X || !Wq4 || !w_absmax || !Y || !workspace) return I8MM_ERR_INVALID_ARG;
  if (!a16(X) || !a16(Wq4) || !a16(Y)) return I8MM_ERR_ALIGNMENT;
  const R4Layout L = r4_layout(M, K, G);
  if (workspace_bytes < L.total) return I8MM_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return I8MM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  float* xa = reinterpret_cast<float*>(ws + L.x_absmax);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.Xq);
  cudaError_t e = cudaMemsetAsync(status, 0, 16, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  e = launch_rotate_groups(static_cast<const __half*>(X), M, K, G, Xq, nullptr, xa, st);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  return rot_status(launch_gemm_groups(Xq, Wq4, xa, w_absmax, static_cast<__half*>(Y), M, N, K,
                                       G, status, st));
}

}  // extern "C"

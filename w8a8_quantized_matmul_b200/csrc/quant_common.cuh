// Device helpers shared by the quantisation kernels: fp16 unpacking, the
// INT8 code of one value, byte packing and warp reductions.
//
// Code of x in a group with absmax a (AIInfra "05Quantization01", LLM.int8()
// section, vector-wise quantisation with c = 127/absmax; the rounding is to
// nearest, ties to even): q = clamp(rint(fl32(fl32(x*127)/a)), -127, 127),
// x*127 exact in fp32 for fp16 x, one correctly rounded fp32 division.
//
// The kernels form the correctly rounded quotient without a division: with
// n = x*127 (exact), ra = fl(1/a) (one correctly rounded reciprocal per group),
// q = fl(n*ra), r = fma(q, -a, n) and q' = fma(r, ra, q), q' equals fl(n/a)
// for every pair of fp16 values x, a with |x| <= a. This is Markstein's
// correction step for division with a fused multiply-add (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990; also "IA-64 and Elementary Functions", 2000):
// the exact remainder r = n - q*a comes from one FMA, and one more FMA adds
// its scaled value to the first quotient. Markstein's theorem needs a
// correctly rounded reciprocal; here the result was also checked for all such
// fp16 pairs exhaustively, and the check ships with the tests. The integer code of q'
// (|q'| <= 127) is then the low byte of fl(q' + 1.5*2^23), which rounds half
// to even. Entries of outlier columns may exceed a; their codes are discarded.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

namespace i8mm {

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

// 1/a correctly rounded; 0 for an all-zero group (every code is then 0).
__device__ __forceinline__ float quant_rcp(float a) { return a == 0.0f ? 0.0f : __frcp_rn(a); }

// The code of quant_code from the FMA-corrected quotient (ra = quant_rcp(a);
// exact for |x| <= a, see the file comment).
__device__ __forceinline__ int quant_code_fma(float x, float a, float ra) {
  const float n = __fmul_rn(x, 127.0f);
  const float q = __fmul_rn(n, ra);
  const float r = __fmaf_rn(q, -a, n);
  const int c = __float2int_rn(__fmaf_rn(r, ra, q));
  return max(-127, min(127, c));
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
                                          const int32_t* s_prefix, int v, float amax, float ra,
                                          uint2* dst, __half* xo_row) {
  const uint32_t wbits = s_bits[v >> 2];
  const uint32_t m8 = (wbits >> (8 * (v & 3))) & 0xFFu;
  float f[8];
  unpack8(u, f);
  int q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = ((m8 >> i) & 1u) ? 0 : quant_code_fma(f[i], amax, ra);
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


// Rounding constant of the paired code path: adding 1.5 * 2^23 to |y| < 2^22
// rounds y to the nearest integer (ties to even) and leaves it in the low
// mantissa bits, so the low byte of the sum is the two's-complement code.
constexpr float kMagic = 12582912.0f;

// Paired IEEE fp32 arithmetic (round to nearest even in each lane).
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  return static_cast<uint64_t>(__float_as_uint(a)) |
         (static_cast<uint64_t>(__float_as_uint(b)) << 32);
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// |x| of both halves (sign bits cleared) as a half2.
__device__ __forceinline__ __half2 habs2_bits(uint32_t w) {
  const uint32_t a = w & 0x7FFF7FFFu;
  return *reinterpret_cast<const __half2*>(&a);
}

// 0xFFFF in each half that is NOT an outlier column, for half2 i of an 8-column mask.
__device__ __forceinline__ uint32_t keep_half2(uint32_t m8, int i) {
  return (((m8 >> (2 * i)) & 1u) ? 0u : 0x0000FFFFu) | (((m8 >> (2 * i + 1)) & 1u) ? 0u : 0xFFFF0000u);
}

// 0xFF in each byte of a 4-code word that is NOT an outlier column.
__device__ __forceinline__ uint32_t keep_bytes(uint32_t m4) {
  return ((m4 & 1u) ? 0u : 0x000000FFu) | ((m4 & 2u) ? 0u : 0x0000FF00u) |
         ((m4 & 4u) ? 0u : 0x00FF0000u) | ((m4 & 8u) ? 0u : 0xFF000000u);
}

// Codes of the fp16 pair w, each in the low byte of its fp32 lane (the 1.5*2^23
// rounding): n = w*127, q = n*ra, r = fma(q, -a, n), q' = fma(r, ra, q).
// a2 = (-a, -a), ra2 = (ra, ra) packed once per group.
__device__ __forceinline__ uint64_t code_lanes(uint32_t w, uint64_t na2, uint64_t ra2) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  const uint64_t n = mul2(f2pack(f.x, f.y), f2pack(127.0f, 127.0f));
  const uint64_t q = mul2(n, ra2);
  const uint64_t r = fma2(q, na2, n);
  return add2(fma2(r, ra2, q), f2pack(kMagic, kMagic));
}

// Eight INT8 codes of the vector u (exact; see the file comment).
__device__ __forceinline__ uint2 codes8(const uint4& u, float amax, float ra) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
  const uint64_t na2 = f2pack(-amax, -amax), ra2 = f2pack(ra, ra);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t s = code_lanes(w[i], na2, ra2);
    b[2 * i] = static_cast<uint32_t>(s);
    b[2 * i + 1] = static_cast<uint32_t>(s >> 32);
  }
  const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(w0, w1);
}

// Two INT8 codes (low two bytes) of the fp16 pair w, same rule as codes8.
__device__ __forceinline__ uint32_t codes2(uint32_t w, float amax, float ra) {
  const uint64_t s = code_lanes(w, f2pack(-amax, -amax), f2pack(ra, ra));
  return __byte_perm(static_cast<uint32_t>(s), static_cast<uint32_t>(s >> 32), 0x0040) & 0xFFFFu;
}
}  // namespace i8mm

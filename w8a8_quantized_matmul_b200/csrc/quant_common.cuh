// Device helpers shared by the quantisation kernels: fp16 unpacking, the
// INT8 code of one value, byte packing and warp reductions.
//
// Code of x in a group with absmax a (AIInfra "05Quantization01", LLM.int8()
// section, vector-wise quantisation with c = 127/absmax; the rounding is to
// nearest, ties to even): q = clamp(rint(fl32(fl32(x*127)/a)), -127, 127),
// x*127 exact in fp32 for fp16 x, one correctly rounded fp32 division.
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


// Rounding constant of the paired code path: adding 1.5 * 2^23 to |y| < 2^22
// rounds y to the nearest integer (ties to even) and leaves it in the low
// mantissa bits, so the low byte of the sum is the two's-complement code.
constexpr float kMagic = 12582912.0f;
// |y - rint(y)| above this means y is within 6.2e-5 of a half-integer.
constexpr float kTieMargin = 0.5f - 6.2e-5f;

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

// Eight INT8 codes of the vector u (exact; see the file comment).
__device__ __forceinline__ uint2 codes8(const uint4& u, float amax, float inv) {
  if (amax == 0.0f) return make_uint2(0u, 0u);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
  const uint64_t inv2 = f2pack(inv, inv);
  const uint64_t magic2 = f2pack(kMagic, kMagic);
  uint32_t b[8];
  float emax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    const uint64_t y = mul2(f2pack(f.x, f.y), inv2);
    const uint64_t s = add2(y, magic2);
    const uint64_t e = sub2(y, sub2(s, magic2));
    emax = fmaxf(emax, fmaxf(fabsf(lo(e)), fabsf(hi(e))));
    b[2 * i] = static_cast<uint32_t>(s);
    b[2 * i + 1] = static_cast<uint32_t>(s >> 32);
  }
  if (emax > kTieMargin) {
    // Within reach of a rounding tie: form the correctly rounded quotient.
    float f[8];
    unpack8(u, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = static_cast<uint32_t>(quant_code(f[i], amax));
  }
  const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(w0, w1);
}

// Exact codes of four fp16 values (the tie fallback of codes4), kept out of line
// so the common path stays short.
static __device__ __noinline__ uint32_t codes4_exact(uint32_t w0, uint32_t w1, float amax) {
  const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w0));
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w1));
  return pack4(quant_code(f0.x, amax), quant_code(f0.y, amax), quant_code(f1.x, amax),
               quant_code(f1.y, amax));
}

// Four INT8 codes of the fp16 values in h (two half2 words), same rule as codes8.
__device__ __forceinline__ uint32_t codes4(const uint2& h, float amax, float inv) {
  if (amax == 0.0f) return 0u;
  const uint64_t inv2 = f2pack(inv, inv);
  const uint64_t magic2 = f2pack(kMagic, kMagic);
  const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
  const uint64_t y0 = mul2(f2pack(f0.x, f0.y), inv2);
  const uint64_t y1 = mul2(f2pack(f1.x, f1.y), inv2);
  const uint64_t s0 = add2(y0, magic2);
  const uint64_t s1 = add2(y1, magic2);
  const uint64_t e0 = sub2(y0, sub2(s0, magic2));
  const uint64_t e1 = sub2(y1, sub2(s1, magic2));
  const float emax = fmaxf(fmaxf(fabsf(lo(e0)), fabsf(hi(e0))), fmaxf(fabsf(lo(e1)), fabsf(hi(e1))));
  if (emax > kTieMargin) return codes4_exact(h.x, h.y, amax);
  const uint32_t b0 = static_cast<uint32_t>(s0), b1 = static_cast<uint32_t>(s0 >> 32);
  const uint32_t b2 = static_cast<uint32_t>(s1), b3 = static_cast<uint32_t>(s1 >> 32);
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}
}  // namespace i8mm

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


}  // namespace i8mm

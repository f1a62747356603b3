/* Checks the division-free INT8 code rule of the CUDA kernels on the CPU.
 *
 * For fp16 values x and a with 0 < x <= a the kernels form
 *   n = x*127 (exact), ra = fl(1/a), q = fl(n*ra), r = fma(q, -a, n),
 *   q' = fma(r, ra, q)
 * and take the code from fl(q' + 1.5*2^23). This program checks q' == fl(n/a)
 * (one IEEE single-precision division) and that the codes agree, for every a
 * in the given index range (stride s) and every x <= a. Negative x follows by
 * symmetry of round-to-nearest. Must be built without FP contraction.
 * Usage: fma_quotient_check [stride] ; exit status 1 on any mismatch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float half_to_float(uint16_t h) {
  const uint32_t sign = (uint32_t)(h >> 15) << 31;
  uint32_t e = (h >> 10) & 31, m = h & 1023, f;
  if (e == 0) {
    if (m == 0) {
      f = sign;
    } else {              /* subnormal: normalise */
      int k = 0;
      while (!(m & 1024)) { m <<= 1; ++k; }
      f = sign | ((uint32_t)(113 - k) << 23) | ((m & 1023) << 13);
    }
  } else if (e == 31) {
    f = sign | 0x7F800000u | (m << 13);
  } else {
    f = sign | ((e + 112) << 23) | (m << 13);
  }
  float r;
  memcpy(&r, &f, 4);
  return r;
}

int main(int argc, char** argv) {
  const int stride = argc > 1 ? atoi(argv[1]) : 1;
  static float v[0x7C00];                       /* 0 .. 65504 ascending */
  for (int i = 0; i < 0x7C00; ++i) v[i] = half_to_float((uint16_t)i);
  volatile float magic = 12582912.0f;
  long long pairs = 0, bad = 0;
  for (int ia = 1; ia < 0x7C00; ia += stride) {
    const float a = v[ia];
    const float ra = 1.0f / a;
    for (int ix = 1; ix <= ia; ++ix) {
      const float n = v[ix] * 127.0f;
      const float q = n * ra;
      const float r = fmaf(q, -a, n);
      const float q2 = fmaf(r, ra, q);
      const float ref = n / a;
      const float code = (q2 + magic) - magic;
      ++pairs;
      if (q2 != ref || code != rintf(ref)) {
        if (bad < 5) printf("mismatch: x=%a a=%a q'=%a ref=%a\n", v[ix], a, q2, ref);
        ++bad;
      }
    }
  }
  printf("pairs %lld mismatches %lld\n", pairs, bad);
  return bad ? 1 : 0;
}

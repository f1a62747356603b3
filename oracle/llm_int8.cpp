// CPU oracle of the LLM.int8() mixed-precision decomposition matmul Y = X.W^T,
// in plain C++17.
//
// TEST INFRASTRUCTURE ONLY. This is the slow, obviously correct definition the
// CUDA path is checked against. Only the tests, the smoke check and the
// benchmark's CPU-baseline and reference legs load it (through the ctypes shim
// in llm_int8.py); the product library never does, and the two share no code,
// header, table or helper.
//
// Build: g++ -std=c++17 -O3 -ffp-contract=off -fPIC -shared -pthread (no
// -ffast-math), so that every float operation below is one IEEE binary32 or
// binary64 operation rounded to nearest even, in the order written.
//
// Sources (web pages, cited by title and section):
//   [AIInfra]    Infrasys-AI/AIInfra "05Infer/06CompDistill/05Quantization01",
//                LLM.int8() section: outlier feature dimensions found by a
//                magnitude threshold; vector-wise absmax INT8 quantisation of
//                the rest (one scale per activation row, one per weight column
//                of the h x o weight); INT8 matmul accumulated in INT32;
//                dequantisation by the outer product of the two scale vectors;
//                FP16 matmul over the outlier dimensions; the two parts summed.
//                Training notes: the top 1-2% largest-magnitude dimensions in
//                FP16.
//   [Scholia]    scholia-log "Inference Quantization" notes, section 4 (step
//                s = absmax/qmax, q = round(x/s), x_hat = s*q; all-zero tensors
//                need separate handling), section 6 (zero point:
//                q = clip(round(x/s) + z, qmin, qmax), x_hat = s*(q - z)).
//   [Tanjunchen] "quantization explained part 2", section 1.2 (threshold 6.0 on
//                the activation magnitude; after splitting out the outlier
//                dimension the remaining dimensions set the scale), section 4.5
//                (symmetric clamp to +-qmax, rounding half to even).
//
// Readings where the pages are silent or garbled (each is listed in the design
// notes): a column is an outlier iff some |x| > threshold (strict), compared in
// binary32 over all rows of the current X; the activation absmax of a row is
// taken over the non-outlier columns, the weight absmax of an output row over
// all K; codes are clamp(rint(fl32(fl32(x*qmax)/absmax)), -qmax, qmax) with rint
// rounding half to even; a zero absmax gives zero codes; the outlier columns
// leave the INT8 product by zeroing their activation codes; dequantisation is
// C * x_absmax * w_absmax / 127^2 in binary64; the outlier product is summed in
// binary64 over the ascending outlier list; Y is the binary64 sum rounded once
// to binary16.
//
// Parity status: every exported function is pinned by the CPU tests (the pages'
// worked examples, closed forms, brute force, exact rational arithmetic, error
// bounds, the threshold = inf / threshold = 0 endpoints, and the binary16
// conversions against numpy on every bit pattern).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <thread>
#include <vector>

namespace {

// ----------------------------------------------------------------- threads
int g_threads = 0;   // 0: one per hardware thread

int thread_count() {
  if (g_threads > 0) return g_threads;
  const char* env = std::getenv("ORACLE_THREADS");
  if (env && std::atoi(env) > 0) return std::atoi(env);
  const unsigned h = std::thread::hardware_concurrency();
  return h > 0 ? static_cast<int>(h) : 1;
}

// Runs body(r) for r in [0, rows) on up to thread_count() threads, each thread
// taking a contiguous block of rows. The rows are independent; the order in
// which they are done changes no result.
template <class F>
void for_each_row(int64_t rows, F body) {
  const int64_t nt = std::max<int64_t>(1, std::min<int64_t>(thread_count(), rows));
  if (nt == 1) {
    for (int64_t r = 0; r < rows; ++r) body(r);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (rows + nt - 1) / nt;
  for (int64_t t = 0; t < nt; ++t) {
    const int64_t r0 = t * per, r1 = std::min(rows, r0 + per);
    if (r0 >= r1) break;
    pool.emplace_back([=] {
      for (int64_t r = r0; r < r1; ++r) body(r);
    });
  }
  for (auto& th : pool) th.join();
}

// ----------------------------------------------------------------- binary16
// IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
float half_to_float(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  float v;
  if (e == 0) {
    v = std::ldexp(static_cast<float>(f), -24);            // zero or subnormal: f * 2^-24
  } else if (e == 31) {
    v = f == 0 ? INFINITY : NAN;
  } else {
    v = std::ldexp(static_cast<float>(1024 + f), e - 25);  // (1 + f/1024) * 2^(e-15)
  }
  return sign ? -v : v;
}

double half_to_double(uint16_t h) { return static_cast<double>(half_to_float(h)); }

// Nearest binary16 to d, ties to even (one rounding, straight from binary64).
uint16_t double_to_half(double d) {
  if (std::isnan(d)) return 0x7E00;
  const uint16_t sign = std::signbit(d) ? 0x8000 : 0;
  const double a = std::fabs(d);
  // 65504 is the largest finite binary16; halfway to the next power of two
  // (65520) and above rounds to infinity.
  if (a >= 65520.0) return sign | 0x7C00;
  if (a < std::ldexp(1.0, -14)) {
    // Subnormal range: multiples of 2^-24. The scaled value is exact in
    // binary64 and nearbyint rounds it half to even; 1024 becomes the smallest
    // normal, whose bit pattern is the same integer.
    const double q = std::nearbyint(std::ldexp(a, 24));
    return sign | static_cast<uint16_t>(q);
  }
  int ex = 0;
  std::frexp(a, &ex);                     // a = m * 2^ex, m in [0.5, 1)
  int E = ex - 1;                         // a in [2^E, 2^(E+1))
  double q = std::nearbyint(std::ldexp(a, 10 - E));   // significand * 1024, in [1024, 2048]
  if (q == 2048.0) {
    q = 1024.0;
    ++E;
  }
  if (E + 15 >= 31) return sign | 0x7C00;
  return sign | static_cast<uint16_t>(((E + 15) << 10) | (static_cast<int>(q) - 1024));
}

// ----------------------------------------------------------------- quantiser
// [Scholia] section 4, [Tanjunchen] section 4.5: q = clamp(rint((x*qmax)/a),
// -qmax, qmax); one binary32 product, one binary32 division, rint half to even
// (the default rounding mode). a == 0: the group is all zero, code 0.
int32_t absmax_code(float x, float a, int qmax) {
  if (!(a > 0.0f)) return 0;
  const float prod = x * static_cast<float>(qmax);
  const float quot = prod / a;
  if (std::isnan(quot)) return 0;   // outside the contract (inputs are finite)
  const float q = std::rint(quot);
  if (q > static_cast<float>(qmax)) return qmax;
  if (q < static_cast<float>(-qmax)) return -qmax;
  return static_cast<int32_t>(q);
}

}  // namespace

extern "C" {

// ------------------------------------------------------------------- plumbing
int orc_threads(void) { return thread_count(); }
void orc_set_threads(int n) { g_threads = n; }

void orc_half_to_float(const uint16_t* h, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = half_to_float(h[i]);
}

void orc_double_to_half(const double* d, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_half(d[i]);
}

// Codes of n binary32 values against their absmax (elementwise), as int32.
void orc_absmax_codes(const float* x, const float* a, int64_t n, int qmax, int32_t* q) {
  for (int64_t i = 0; i < n; ++i) q[i] = absmax_code(x[i], a[i], qmax);
}

// Largest |x| of n binary32 values (0 for none): the absmax of one tensor.
float orc_absmax(const float* x, int64_t n) {
  float a = 0.0f;
  for (int64_t i = 0; i < n; ++i) a = std::max(a, std::fabs(x[i]));
  return a;
}

// [Scholia] section 4: step s = absmax/qmax and x_hat = s*q, in binary64
// (elementwise over n codes; s alone when q is null).
void orc_dequantize_codes(const int32_t* q, const double* a, int64_t n, int qmax, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    const double s = a[i] / static_cast<double>(qmax);
    out[i] = q ? static_cast<double>(q[i]) * s : s;
  }
}

// ----------------------------------------------------------------- weights
// [AIInfra]: one scale per weight column of the h x o matrix, i.e. per output
// row n of our [N][K] layout, over all K: aw[n] = max_k |W[n][k]|.
void orc_quantize_weight_rows(const uint16_t* W, int N, int K, int8_t* Wq, float* aw) {
  for_each_row(N, [&](int64_t n) {
    const uint16_t* w = W + n * K;
    float a = 0.0f;
    for (int k = 0; k < K; ++k) a = std::max(a, std::fabs(half_to_float(w[k])));
    aw[n] = a;
    for (int k = 0; k < K; ++k)
      Wq[n * K + k] = static_cast<int8_t>(absmax_code(half_to_float(w[k]), a, 127));
  });
}

// ----------------------------------------------------------------- detection
// [AIInfra] detection by a magnitude threshold; [Tanjunchen] section 1.2 (a
// dimension whose activation magnitude exceeds the threshold): column j is an
// outlier iff |X[i][j]| > threshold for some row i. Returns the count.
int orc_find_outlier_cols(const uint16_t* X, int M, int K, float threshold, uint8_t* mask) {
  int count = 0;
  for (int j = 0; j < K; ++j) {
    bool out = false;
    for (int i = 0; i < M && !out; ++i)
      if (std::fabs(half_to_float(X[static_cast<int64_t>(i) * K + j])) > threshold) out = true;
    mask[j] = out ? 1 : 0;
    count += out ? 1 : 0;
  }
  return count;
}

// The bitmap (bit j % 32 of word j / 32 set for an outlier column) and the
// ascending list of a column mask. Returns the count.
int orc_mask_to_bitmap(const uint8_t* mask, int K, uint32_t* bitmap, int32_t* idx) {
  const int words = (K + 31) / 32;
  for (int w = 0; w < words; ++w) bitmap[w] = 0;
  int count = 0;
  for (int j = 0; j < K; ++j) {
    if (!mask[j]) continue;
    bitmap[j / 32] |= 1u << (j % 32);
    idx[count++] = j;
  }
  return count;
}

// [AIInfra] training notes: keep the k dimensions of largest magnitude in FP16.
// A column's magnitude is its max |x| over the rows; ties go to the lower
// column index; k is clipped to [0, K].
void orc_find_topk_cols(const uint16_t* X, int M, int K, int k, uint8_t* mask) {
  std::vector<float> colmax(K, 0.0f);
  for (int j = 0; j < K; ++j)
    for (int i = 0; i < M; ++i)
      colmax[j] = std::max(colmax[j], std::fabs(half_to_float(X[static_cast<int64_t>(i) * K + j])));
  std::vector<int> order(K);
  for (int j = 0; j < K; ++j) order[j] = j;
  std::stable_sort(order.begin(), order.end(),
                   [&](int p, int q) { return colmax[p] > colmax[q]; });   // equal: index order kept
  k = std::max(0, std::min(k, K));
  for (int j = 0; j < K; ++j) mask[j] = 0;
  for (int t = 0; t < k; ++t) mask[order[t]] = 1;
}

// ----------------------------------------------------------------- activations
// [AIInfra] vector-wise quantisation of each row of X after the split;
// [Tanjunchen] section 1.2 (the remaining dimensions set the scale):
// ax[i] = max over non-outlier j of |X[i][j]|, Xq = code against ax[i], 0 at
// the outlier columns.
void orc_quantize_act_rows(const uint16_t* X, int M, int K, const uint8_t* mask, int8_t* Xq,
                           float* ax) {
  for_each_row(M, [&](int64_t i) {
    const uint16_t* x = X + i * K;
    float a = 0.0f;
    for (int j = 0; j < K; ++j)
      if (!mask[j]) a = std::max(a, std::fabs(half_to_float(x[j])));
    ax[i] = a;
    for (int j = 0; j < K; ++j)
      Xq[i * K + j] = mask[j] ? 0 : static_cast<int8_t>(absmax_code(half_to_float(x[j]), a, 127));
  });
}

// [Scholia] section 6, zero point: per row over the non-outlier columns,
// lo = min(0, min x), hi = max(0, max x) (real 0 stays representable),
// step = fl32(fl32(hi - lo) / 255), zero = clamp(-128 - rint(fl32(lo / step)),
// -128, 127), q = clamp(rint(fl32(x / step)) + zero, -128, 127); q = zero at the
// outlier columns; a row with step 0 gets zero 0 and all codes 0.
void orc_quantize_act_rows_zp(const uint16_t* X, int M, int K, const uint8_t* mask, int8_t* Xq,
                              float* step_out, int32_t* zero_out) {
  for_each_row(M, [&](int64_t i) {
    const uint16_t* x = X + i * K;
    float lo = 0.0f, hi = 0.0f;
    for (int j = 0; j < K; ++j) {
      if (mask[j]) continue;
      const float v = half_to_float(x[j]);
      lo = std::min(lo, v);
      hi = std::max(hi, v);
    }
    const float range = hi - lo;
    const float step = range / 255.0f;
    step_out[i] = step;
    if (!(step > 0.0f)) {
      zero_out[i] = 0;
      for (int j = 0; j < K; ++j) Xq[i * K + j] = 0;
      return;
    }
    const float lq = lo / step;
    const int32_t zero = static_cast<int32_t>(
        std::max(-128.0f, std::min(127.0f, -128.0f - std::rint(lq))));
    zero_out[i] = zero;
    for (int j = 0; j < K; ++j) {
      if (mask[j]) {
        Xq[i * K + j] = static_cast<int8_t>(zero);
        continue;
      }
      const float t = half_to_float(x[j]) / step;
      const float q = std::rint(t) + static_cast<float>(zero);
      Xq[i * K + j] = static_cast<int8_t>(std::max(-128.0f, std::min(127.0f, q)));
    }
  });
}

// ----------------------------------------------------------------- products
// [AIInfra]: C_i32 = X_i8 . W_i8, accumulated in INT32 to avoid overflow.
// C[i][n] = sum_k A[i][k] * B[n][k], a plain triple loop in 64-bit integers;
// returns -1 (and leaves C partly written) if a result does not fit int32.
int orc_int32_gemm(const int8_t* A, const int8_t* B, int M, int N, int K, int32_t* C) {
  std::vector<int> bad(M > 0 ? M : 1, 0);
  for_each_row(M, [&](int64_t i) {
    const int8_t* a = A + i * K;
    for (int n = 0; n < N; ++n) {
      const int8_t* b = B + static_cast<int64_t>(n) * K;
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);
      if (s > INT32_MAX || s < INT32_MIN) bad[i] = 1;
      C[i * N + n] = static_cast<int32_t>(s);
    }
  });
  for (int i = 0; i < M; ++i)
    if (bad[i]) return -1;
  return 0;
}

// sum_k Wq[n][k] (the zero-point correction's weight factor).
void orc_weight_rowsum(const int8_t* Wq, int N, int K, int32_t* s) {
  for (int n = 0; n < N; ++n) {
    int64_t t = 0;
    for (int k = 0; k < K; ++k) t += Wq[static_cast<int64_t>(n) * K + k];
    s[n] = static_cast<int32_t>(t);
  }
}

// [AIInfra] dequantisation: C_normal ~ C_i32 / (c_x (x) c_w), c = 127/absmax,
// i.e. C * x_absmax[i] * w_absmax[n] / 127^2, in binary64 left to right.
void orc_dequantize(const int32_t* C, const float* xs, const float* ws, int M, int N, double* Cn) {
  for_each_row(M, [&](int64_t i) {
    for (int n = 0; n < N; ++n)
      Cn[i * N + n] = static_cast<double>(C[i * N + n]) * static_cast<double>(xs[i]) *
                      static_cast<double>(ws[n]) / 16129.0;
  });
}

// Zero-point rows: sum_k step*(q - z)*w_absmax/127*wq = (C - z*sum_k wq) *
// step * w_absmax / 127; the correction is exact in 64-bit integers.
void orc_dequantize_zp(const int32_t* C, const int32_t* zero, const float* step,
                       const int32_t* wsum, const float* ws, int M, int N, double* Cn) {
  for_each_row(M, [&](int64_t i) {
    for (int n = 0; n < N; ++n) {
      const int64_t c = static_cast<int64_t>(C[i * N + n]) -
                        static_cast<int64_t>(zero[i]) * static_cast<int64_t>(wsum[n]);
      Cn[i * N + n] = static_cast<double>(c) * static_cast<double>(step[i]) *
                      static_cast<double>(ws[n]) / 127.0;
    }
  });
}

// [AIInfra]: C_outlier = sum over h in O of X_f16^h W_f16^h, in binary64 over
// the ascending list idx[0..count).
void orc_outlier_gemm(const uint16_t* X, const uint16_t* W, int M, int N, int K,
                      const int32_t* idx, int count, double* Co) {
  for_each_row(M, [&](int64_t i) {
    for (int n = 0; n < N; ++n) {
      double s = 0.0;
      for (int p = 0; p < count; ++p)
        s += half_to_double(X[i * K + idx[p]]) * half_to_double(W[static_cast<int64_t>(n) * K + idx[p]]);
      Co[i * N + n] = s;
    }
  });
}

// [AIInfra]: C_f16 = C_outlier + C_normal, one rounding to binary16.
void orc_sum_to_half(const double* Cn, const double* Co, int64_t n, uint16_t* Y) {
  for (int64_t e = 0; e < n; ++e) Y[e] = double_to_half(Cn[e] + Co[e]);
}

// ----------------------------------------------------------------- whole path
// Every step above in the pages' order, on X fp16 [M][K], W fp16 [N][K] and the
// pre-quantised weight (Wq, w_scale). mask_in (nullable) replaces detection by
// a given outlier set (the set of a batch whose tokens are split over several
// processes). zp selects zero-point activation codes. The intermediates C, Cn,
// Co are written when their pointers are not null. Returns the outlier count,
// or -1 if an INT32 result overflowed.
int orc_llm_int8_matmul(const uint16_t* X, const uint16_t* W, int M, int N, int K,
                        float threshold, const int8_t* Wq, const float* w_scale,
                        const uint8_t* mask_in, int zp, uint8_t* mask, uint32_t* bitmap,
                        int32_t* idx, int8_t* Xq, float* x_scale, int32_t* zero, int32_t* wsum,
                        int32_t* C_out, double* Cn_out, double* Co_out, uint16_t* Y) {
  if (mask_in) {
    for (int j = 0; j < K; ++j) mask[j] = mask_in[j] ? 1 : 0;
  } else {
    orc_find_outlier_cols(X, M, K, threshold, mask);
  }
  const int count = orc_mask_to_bitmap(mask, K, bitmap, idx);
  if (zp)
    orc_quantize_act_rows_zp(X, M, K, mask, Xq, x_scale, zero);
  else
    orc_quantize_act_rows(X, M, K, mask, Xq, x_scale);
  const size_t MN = static_cast<size_t>(M) * static_cast<size_t>(N);
  std::vector<int32_t> Cv;
  std::vector<double> Cnv, Cov;
  int32_t* C = C_out;
  double* Cn = Cn_out;
  double* Co = Co_out;
  if (!C) { Cv.resize(MN); C = Cv.data(); }
  if (!Cn) { Cnv.resize(MN); Cn = Cnv.data(); }
  if (!Co) { Cov.resize(MN); Co = Cov.data(); }
  if (orc_int32_gemm(Xq, Wq, M, N, K, C) != 0) return -1;
  if (zp) {
    orc_weight_rowsum(Wq, N, K, wsum);
    orc_dequantize_zp(C, zero, x_scale, wsum, w_scale, M, N, Cn);
  } else {
    orc_dequantize(C, x_scale, w_scale, M, N, Cn);
  }
  orc_outlier_gemm(X, W, M, N, K, idx, count, Co);
  orc_sum_to_half(Cn, Co, static_cast<int64_t>(MN), Y);
  return count;
}

// Y[rows[t]][cols[t]] for T sampled outputs, one by one: detection over the
// whole X (the outlier set depends on every row), then for each sample its
// row's codes and scale, the INT32 dot product, its dequantisation, the
// outlier term and the rounding. Writes the mask of the set, and per sample Y,
// C and the row's x_scale. Returns the outlier count.
int orc_llm_int8_matmul_at(const uint16_t* X, const uint16_t* W, const int8_t* Wq,
                           const float* w_scale, int M, int N, int K, float threshold,
                           const int64_t* rows, const int64_t* cols, int64_t T, uint8_t* mask,
                           uint16_t* Y, int32_t* C, float* xs) {
  orc_find_outlier_cols(X, M, K, threshold, mask);
  std::vector<uint32_t> bitmap((K + 31) / 32 + 1);
  std::vector<int32_t> idx(K + 1);
  const int count = orc_mask_to_bitmap(mask, K, bitmap.data(), idx.data());
  for_each_row(T, [&](int64_t t) {
    const int64_t i = rows[t], n = cols[t];
    std::vector<int8_t> xq(K);
    float a = 0.0f;
    orc_quantize_act_rows(X + i * K, 1, K, mask, xq.data(), &a);
    int64_t s = 0;
    for (int k = 0; k < K; ++k)
      s += static_cast<int32_t>(xq[k]) * static_cast<int32_t>(Wq[n * K + k]);
    const double cn = static_cast<double>(s) * static_cast<double>(a) *
                      static_cast<double>(w_scale[n]) / 16129.0;
    double co = 0.0;
    for (int p = 0; p < count; ++p)
      co += half_to_double(X[i * K + idx[p]]) * half_to_double(W[n * K + idx[p]]);
    C[t] = static_cast<int32_t>(s);
    xs[t] = a;
    Y[t] = double_to_half(cn + co);
  });
  return count;
}

}  // extern "C"

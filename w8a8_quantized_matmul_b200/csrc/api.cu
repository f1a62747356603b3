// C ABI of libint8mm (declared in include/int8mm.h): argument validation,
// workspace carving, and the launch sequence of the LLM.int8() path.
//
// int8_mixed_matmul on one stream, no host synchronisation:
//   1. cudaMemsetAsync   zero the count/status/barrier words and the outlier bitmap
//   2. fused K1          cooperative kernel: |x| > threshold column bitmap, grid
//                        barrier, per-token absmax INT8 codes over the non-outlier
//                        columns, compacted fp16 outlier panels X_O and W_O
//   3. GEMM              tcgen05 INT8 GEMM + fp16 outlier GEMM + dequantising epilogue
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>

#include "int8mm.h"
#include "kernels.cuh"

namespace {

using namespace i8mm;

constexpr size_t kAlign = 256;
constexpr int kMaxK = 65536;      // bitmap + prefix of a row fit the quantiser's shared memory
constexpr int kMaxMN = 1 << 22;   // keeps the GEMM grid below 2^31 CTAs

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int panel_ld(int K) { return (K + kPanelAlign - 1) / kPanelAlign * kPanelAlign; }

// Sizes the ABI accepts: K a positive multiple of 16, and every product that
// indexes memory must fit the kernels' 32-bit tile coordinates.
int check_sizes(int M, int N, int K) {
  if (M < 0 || N < 0 || K <= 0) return I8MM_ERR_INVALID_ARG;
  if (K % 16 != 0) return I8MM_ERR_ALIGNMENT;
  if (K > kMaxK || M > kMaxMN || N > kMaxMN) return I8MM_ERR_INVALID_ARG;
  return I8MM_OK;
}

int check_threshold(float t) {
  if (std::isnan(t) || t < 0.0f) return I8MM_ERR_INVALID_ARG;
  return I8MM_OK;
}

// Only sm_100 (B200) runs these kernels; checked once per device.
int check_device() {
  static int cached[64] = {};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return I8MM_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] == 1 ? I8MM_OK : I8MM_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return I8MM_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
  return ok ? I8MM_OK : I8MM_ERR_UNSUPPORTED_DEVICE;
}

thread_local char g_last_error[256] = "";

// Records which step failed and why, and returns I8MM_ERR_CUDA (I8MM_OK on success).
int cuda_fail(const char* what, cudaError_t e) {
  if (e == cudaSuccess) return I8MM_OK;
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what, cudaGetErrorName(e),
                cudaGetErrorString(e));
  return I8MM_ERR_CUDA;
}

int cuda_status(cudaError_t e) { return cuda_fail("launch", e); }

// Register-resident vectors per lane for a row of K fp16 values (0 = streaming).
int vpl_for(int K) {
  const int nv = K / 8;
  if (nv <= 32) return 1;
  if (nv <= 64) return 2;
  if (nv <= 128) return 4;
  if (nv <= 256) return 8;
  if (nv <= 512) return 16;
  if (nv <= 1024) return 32;
  return 0;
}

struct Layout {
  i8mm_workspace_layout l;
};

bool make_layout(int M, int N, int K, Layout* out) {
  if (check_sizes(M, N, K) != I8MM_OK) return false;
  const size_t words = static_cast<size_t>((K + 31) / 32);
  const int ld = panel_ld(K);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  Layout L{};
  // The count and the bitmap sit together so one memset clears both.
  L.l.n_outliers = take(16);              // [0] count, [1] status, [2] grid-barrier counter
  L.l.status = L.l.n_outliers + 4;
  L.l.col_bitmap = L.l.n_outliers + 16;   // directly after, inside the same memset span
  off = align_up(L.l.col_bitmap + words * 4, kAlign);
  L.l.col_idx = take(static_cast<size_t>(K) * 4);
  L.l.x_scale = take(static_cast<size_t>(M) * 4);
  L.l.Xq = take(static_cast<size_t>(M) * K);
  L.l.X_O = take(static_cast<size_t>(M) * ld * 2);
  L.l.W_O = take(static_cast<size_t>(N) * ld * 2);
  L.l.total = off;
  L.l.panel_ld = ld;
  *out = L;
  return true;
}

}  // namespace

namespace i8mm {
int abi_check_device() { return check_device(); }
int abi_cuda_fail(const char* what, cudaError_t e) { return cuda_fail(what, e); }
}  // namespace i8mm

extern "C" {

const char* int8_last_error_string(void) { return g_last_error; }

const char* int8_status_string(int status) {
  switch (status) {
    case I8MM_OK: return "ok";
    case I8MM_ERR_INVALID_ARG: return "invalid argument";
    case I8MM_ERR_ALIGNMENT: return "misaligned pointer or K not a multiple of 16";
    case I8MM_ERR_WORKSPACE: return "workspace missing or too small";
    case I8MM_ERR_CUDA: return "CUDA error";
    case I8MM_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case I8MM_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    default: return "unknown status";
  }
}

size_t int8_mixed_matmul_workspace_size(int M, int N, int K) {
  Layout L;
  if (!make_layout(M, N, K, &L)) return 0;
  return L.l.total;
}

int int8_mixed_matmul_workspace_layout(int M, int N, int K, i8mm_workspace_layout* out) {
  if (!out) return I8MM_ERR_INVALID_ARG;
  const int st = check_sizes(M, N, K);
  if (st != I8MM_OK) return st;
  Layout L;
  make_layout(M, N, K, &L);
  *out = L.l;
  return I8MM_OK;
}

int int8_weight_rowsum(const int8_t* Wq, int N, int K, int32_t* rowsum, i8mm_stream_t stream) {
  const int st = check_sizes(1, N, K);
  if (st != I8MM_OK) return st;
  if (N == 0) return I8MM_OK;
  if (!Wq || !rowsum) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(Wq) || !aligned16(rowsum)) return I8MM_ERR_ALIGNMENT;
  return cuda_status(launch_weight_rowsum(Wq, N, K, rowsum, static_cast<cudaStream_t>(stream)));
}

int int8_quantize_weight_rows(const void* W, int N, int K, int8_t* Wq, float* w_scale,
                              i8mm_stream_t stream) {
  int st = check_sizes(1, N, K);
  if (st != I8MM_OK) return st;
  if (N == 0) return I8MM_OK;
  if (!W || !Wq || !w_scale) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(w_scale)) return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  const int blocks = (N + 7) / 8;
  quantize_weight_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __half*>(W), N, K, Wq,
                                                         w_scale);
  return cuda_status(cudaGetLastError());
}

int int8_transpose_weight(const void* W, int N, int K, void* Wt, i8mm_stream_t stream) {
  int st = check_sizes(1, N, K);
  if (st != I8MM_OK) return st;
  if (N == 0) return I8MM_OK;
  if (!W || !Wt) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wt)) return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  return cuda_status(launch_transpose_weight(static_cast<const __half*>(W), N, K,
                                             static_cast<__half*>(Wt),
                                             static_cast<cudaStream_t>(stream)));
}

int int8_find_outlier_cols(const void* X, int M, int K, float threshold, uint32_t* col_bitmap,
                           int32_t* n_outliers, int32_t* col_idx, i8mm_stream_t stream) {
  int st = check_sizes(M, 1, K);
  if (st != I8MM_OK) return st;
  if ((st = check_threshold(threshold)) != I8MM_OK) return st;
  if ((M > 0 && !X) || !col_bitmap || !n_outliers) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(col_bitmap) || !aligned16(n_outliers) ||
      (col_idx && !aligned16(col_idx)))
    return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  const size_t words = static_cast<size_t>((K + 31) / 32);
  cudaError_t e = cudaMemsetAsync(col_bitmap, 0, words * 4, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(n_outliers, 0, 4, stream);
  if (e != cudaSuccess) return I8MM_ERR_CUDA;
  const int nv = K / 8;
  dim3 grid((nv + 31) / 32, M > 0 ? (M + kDetectRows - 1) / kDetectRows : 1);
  detect_outliers_kernel<<<grid, 256, 0, stream>>>(static_cast<const __half*>(X), M, K, threshold,
                                                  col_bitmap, n_outliers, col_idx);
  return cuda_status(cudaGetLastError());
}

int int8_quantize_act_rows(const void* X, int M, int K, const uint32_t* col_bitmap, int8_t* Xq,
                           float* x_scale, i8mm_stream_t stream) {
  int st = check_sizes(M, 1, K);
  if (st != I8MM_OK) return st;
  if (M == 0) return I8MM_OK;
  if (!X || !col_bitmap || !Xq || !x_scale) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(col_bitmap) || !aligned16(Xq) || !aligned16(x_scale))
    return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  const int words = (K + 31) / 32;
  const int rows_per_block = 8 * kQuantRowsPerWarp;
  const int qb = (M + rows_per_block - 1) / rows_per_block;
  const size_t smem = static_cast<size_t>(words) * 4;
  QuantArgs qa{};
  qa.X = static_cast<const __half*>(X);
  qa.M = M;
  qa.K = K;
  qa.bitmap = col_bitmap;
  qa.Xq = Xq;
  qa.x_scale = x_scale;
  return cuda_status(launch_quantize_rows(vpl_for(K), qb, smem, stream, qa));
}

}  // extern "C"

namespace {

// stages: bit 0 = control-word clear + fused quantisation kernel, bit 1 = GEMM.
// given / given_n: token-sharded mode (outlier set = OR of the given bitmaps).
int mixed_matmul_impl(const void* X, const int8_t* Wq, const float* w_scale, const void* Wt_fp16,
                      int M, int N, int K, float threshold, void* Y, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream, cudaEvent_t const* ev,
                      int stages = 3, const uint32_t* given = nullptr, int given_n = 0,
                      int32_t* x_zero = nullptr, const int32_t* w_rowsum = nullptr) {
  int st = check_sizes(M, N, K);
  if (st != I8MM_OK) return st;
  if ((st = check_threshold(threshold)) != I8MM_OK) return st;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!X || !Wq || !w_scale || !Wt_fp16 || !Y) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scale) || !aligned16(Wt_fp16) ||
      !aligned16(Y))
    return I8MM_ERR_ALIGNMENT;
  Layout L;
  make_layout(M, N, K, &L);
  if (!workspace || workspace_bytes < L.l.total) return I8MM_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return I8MM_ERR_ALIGNMENT;
  const int words = (K + 31) / 32;
  if ((st = check_device()) != I8MM_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* count = reinterpret_cast<int32_t*>(ws + L.l.n_outliers);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.l.status);
  int32_t* sync_ctr = reinterpret_cast<int32_t*>(ws + L.l.status + 4);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws + L.l.col_bitmap);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.l.col_idx);
  float* xs = reinterpret_cast<float*>(ws + L.l.x_scale);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + L.l.Xq);
  __half* XO = reinterpret_cast<__half*>(ws + L.l.X_O);
  __half* WO = reinterpret_cast<__half*>(ws + L.l.W_O);
  const __half* Xh = static_cast<const __half*>(X);
  const __half* Wh = static_cast<const __half*>(Wt_fp16);

  // Decode shapes: one clustered kernel for the whole call.
  if (stages == 3 && !ev && !given && !x_zero && decode_supported(M, K)) {
    DecodeArgs da{};
    da.X = Xh;
    da.W = Wh;
    da.Wq = Wq;
    da.w_scale = w_scale;
    da.Y = static_cast<__half*>(Y);
    da.M = M;
    da.N = N;
    da.K = K;
    da.threshold = threshold;
    da.bitmap = bitmap;
    da.n_outliers = count;
    da.col_idx = idx;
    da.x_scale = xs;
    da.Xq = Xq;
    da.status = status;
    return cuda_fail("decode_kernel launch", launch_decode(da, stream));
  }
  if (ev && cudaEventRecord(ev[0], stream) != cudaSuccess) return I8MM_ERR_CUDA;
  if (stages & 1) {
    // 1. count, status, barrier counter and bitmap are contiguous: one memset.
    const size_t ctrl = (L.l.col_bitmap - L.l.n_outliers) + static_cast<size_t>(words) * 4;
    cudaError_t e = cudaMemsetAsync(ws + L.l.n_outliers, 0, ctrl, stream);
    if (e != cudaSuccess) return cuda_fail("control-word memset", e);
    // 2. detection, quantisation and compaction: one cooperative kernel
    FusedArgs fa{};
    fa.X = Xh;
    fa.M = M;
    fa.K = K;
    fa.N = N;
    fa.threshold = threshold;
    fa.bitmap = bitmap;
    fa.sync_ctr = sync_ctr;
    fa.n_outliers = count;
    fa.col_idx = idx;
    fa.Xq = Xq;
    fa.x_scale = xs;
    fa.X_O = XO;
    fa.W = Wh;
    fa.W_O = WO;
    fa.ld = L.l.panel_ld;
    fa.status = status;
    fa.given = given;
    fa.given_n = given_n;
    fa.x_zero = x_zero;
    e = launch_detect_quantize_compact(fa, stream);
    if (e != cudaSuccess) return cuda_fail("detect_quantize_compact_kernel launch", e);
  }
  if (ev && cudaEventRecord(ev[1], stream) != cudaSuccess) return I8MM_ERR_CUDA;
  if (!(stages & 2)) return I8MM_OK;
  // 3. GEMM
  GemmArgs g{};
  g.Xq = Xq;
  g.Wq = Wq;
  g.X_O = XO;
  g.W_O = WO;
  g.ld = L.l.panel_ld;
  g.x_scale = xs;
  g.w_scale = w_scale;
  g.n_outliers = count;
  g.x_zero = x_zero;
  g.w_rowsum = w_rowsum;
  g.out = Y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.status = status;
  const cudaError_t ge = launch_gemm_mixed(g, stream);
  if (ge != cudaSuccess) return cuda_fail("GEMM kernel launch", ge);
  if (ev && cudaEventRecord(ev[2], stream) != cudaSuccess) return I8MM_ERR_CUDA;
  return I8MM_OK;
}

}  // namespace

extern "C" {

int int8_mixed_matmul(const void* X, const int8_t* Wq, const float* w_scale, const void* Wt_fp16,
                      int M, int N, int K, float threshold, void* Y, void* workspace,
                      size_t workspace_bytes, i8mm_stream_t stream) {
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, workspace,
                           workspace_bytes, stream, nullptr);
}

int int8_mixed_matmul_stage(int stage, const void* X, const int8_t* Wq, const float* w_scale,
                            const void* Wt_fp16, int M, int N, int K, float threshold, void* Y,
                            void* workspace, size_t workspace_bytes, i8mm_stream_t stream) {
  if (stage != 1 && stage != 2) return I8MM_ERR_INVALID_ARG;
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, workspace,
                           workspace_bytes, stream, nullptr, stage);
}

// Extra workspace of the zero-point path, after the regular layout: the
// per-token zero points (int32 [M]), 256-byte aligned.
size_t int8_mixed_matmul_zp_workspace_size(int M, int N, int K) {
  Layout L;
  if (!make_layout(M, N, K, &L)) return 0;
  const size_t zoff = (L.l.total + 255) & ~static_cast<size_t>(255);
  return (zoff + static_cast<size_t>(M) * 4 + 255) & ~static_cast<size_t>(255);
}

int int8_mixed_matmul_zp(const void* X, const int8_t* Wq, const float* w_scale,
                         const int32_t* w_rowsum, const void* Wt_fp16, int M, int N, int K,
                         float threshold, void* Y, void* workspace, size_t workspace_bytes,
                         i8mm_stream_t stream) {
  const int st = check_sizes(M, N, K);
  if (st != I8MM_OK) return st;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!w_rowsum || !workspace) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(w_rowsum)) return I8MM_ERR_ALIGNMENT;
  Layout L;
  make_layout(M, N, K, &L);
  if (workspace_bytes < int8_mixed_matmul_zp_workspace_size(M, N, K)) return I8MM_ERR_WORKSPACE;
  int32_t* x_zero = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                               ((L.l.total + 255) & ~static_cast<size_t>(255)));
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream), nullptr, 3, nullptr,
                           0, x_zero, w_rowsum);
}

// Extra workspace of the top-k path, after the regular layout: column maxima
// (fp32 [K]) and the selection bitmap (ceil(K/32) words), each 256-byte aligned.
size_t int8_mixed_matmul_topk_workspace_size(int M, int N, int K) {
  Layout L;
  if (!make_layout(M, N, K, &L)) return 0;
  const size_t colmax = (L.l.total + 255) & ~static_cast<size_t>(255);
  const size_t sel = (colmax + static_cast<size_t>(K) * 4 + 255) & ~static_cast<size_t>(255);
  return (sel + static_cast<size_t>((K + 31) / 32) * 4 + 255) & ~static_cast<size_t>(255);
}

int int8_mixed_matmul_topk(const void* X, const int8_t* Wq, const float* w_scale,
                           const void* Wt_fp16, int M, int N, int K, int k, void* Y,
                           void* workspace, size_t workspace_bytes, i8mm_stream_t stream) {
  int st = check_sizes(M, N, K);
  if (st != I8MM_OK) return st;
  if (k < 0) return I8MM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!X || !workspace) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(X)) return I8MM_ERR_ALIGNMENT;
  Layout L;
  make_layout(M, N, K, &L);
  const size_t need = int8_mixed_matmul_topk_workspace_size(M, N, K);
  if (workspace_bytes < need) return I8MM_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t colmax_off = (L.l.total + 255) & ~static_cast<size_t>(255);
  const size_t sel_off = (colmax_off + static_cast<size_t>(K) * 4 + 255) & ~static_cast<size_t>(255);
  float* colmax = reinterpret_cast<float*>(ws + colmax_off);
  uint32_t* sel = reinterpret_cast<uint32_t*>(ws + sel_off);
  cudaError_t e = cudaMemsetAsync(colmax, 0, static_cast<size_t>(K) * 4, s);
  if (e != cudaSuccess) return cuda_fail("column-max memset", e);
  e = launch_column_absmax(static_cast<const __half*>(X), M, K, colmax, s);
  if (e != cudaSuccess) return cuda_fail("column_absmax_kernel launch", e);
  e = launch_topk_select(colmax, K, k, sel, s);
  if (e != cudaSuccess) return cuda_fail("topk_select_kernel launch", e);
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, 0.0f, Y, workspace, workspace_bytes,
                           s, nullptr, 3, sel, 1);
}

int int8_mixed_matmul_sharded(const void* X, const int8_t* Wq, const float* w_scale,
                              const void* Wt_fp16, int M, int N, int K, const uint32_t* bitmaps,
                              int n_bitmaps, void* Y, void* workspace, size_t workspace_bytes,
                              i8mm_stream_t stream) {
  if (!bitmaps || n_bitmaps < 1 || n_bitmaps > 65536) return I8MM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(bitmaps) & 3u) != 0) return I8MM_ERR_ALIGNMENT;
  // The threshold only enters detection, which the caller has done per rank.
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, 0.0f, Y, workspace, workspace_bytes,
                           stream, nullptr, 3, bitmaps, n_bitmaps);
}

int int8_mixed_matmul_profiled(const void* X, const int8_t* Wq, const float* w_scale,
                               const void* Wt_fp16, int M, int N, int K, float threshold, void* Y,
                               void* workspace, size_t workspace_bytes, i8mm_stream_t stream,
                               void* const* events) {
  if (!events || !events[0] || !events[1] || !events[2]) return I8MM_ERR_INVALID_ARG;
  cudaEvent_t ev[3] = {static_cast<cudaEvent_t>(events[0]), static_cast<cudaEvent_t>(events[1]),
                       static_cast<cudaEvent_t>(events[2])};
  return mixed_matmul_impl(X, Wq, w_scale, Wt_fp16, M, N, K, threshold, Y, workspace,
                           workspace_bytes, stream, ev);
}

int int8_debug_gemm_i32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K, int32_t* C,
                        i8mm_stream_t stream) {
  int st = check_sizes(M, N, K);
  if (st != I8MM_OK) return st;
  if (M == 0 || N == 0) return I8MM_OK;
  if (!Xq || !Wq || !C) return I8MM_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(C)) return I8MM_ERR_ALIGNMENT;
  if ((st = check_device()) != I8MM_OK) return st;
  GemmArgs g{};
  g.Xq = Xq;
  g.Wq = Wq;
  g.out = C;
  g.M = M;
  g.N = N;
  g.K = K;
  return cuda_status(launch_gemm_i32(g, stream));
}

int int8_device_status(const void* workspace, i8mm_stream_t stream) {
  if (!workspace) return I8MM_ERR_INVALID_ARG;
  int32_t h = 0;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  // The status word is the second int32 of the workspace (see make_layout).
  if (cudaMemcpyAsync(&h, ws + 4, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return I8MM_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return I8MM_ERR_CUDA;
  return h == 0 ? I8MM_OK : (h == I8MM_ERR_TIMEOUT ? I8MM_ERR_TIMEOUT : I8MM_ERR_CUDA);
}

}  // extern "C"

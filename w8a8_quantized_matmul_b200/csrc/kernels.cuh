// Kernel declarations and launch-shape constants shared by the kernel files
// and the C-ABI layer of libint8mm.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace i8mm {

constexpr int kDetectRows = 32;        // rows of X per detection CTA
constexpr int kQuantRowsPerWarp = 1;   // rows of X per warp in the quantisation kernel
constexpr int kPanelAlign = 64;        // outlier panels are padded to this many columns

__global__ void quantize_weight_rows_kernel(const __half* W, int N, int K, int8_t* Wq,
                                            float* w_scale);

__global__ void detect_outliers_kernel(const __half* X, int M, int K, float threshold,
                                       uint32_t* bitmap, int32_t* counter, int32_t* col_idx);

struct QuantArgs {
  const __half* X;
  int M, K;
  const uint32_t* bitmap;
  int8_t* Xq;
  float* x_scale;
};

// Stand-alone quantisation launch; vpl = 16-byte vectors per lane kept in
// registers (1..32, K <= 256*vpl) or 0 for rows streamed twice.
cudaError_t launch_quantize_rows(int vpl, int grid, size_t smem, cudaStream_t s,
                                 const QuantArgs& a);

// Fused detection + quantisation + compaction (cooperative launch).
struct FusedArgs {
  const __half* X;
  int M, K, N;
  float threshold;
  uint32_t* bitmap;       // [ceil(K/32)], zero on entry
  int32_t* sync_ctr;      // zero on entry; grid-barrier arrival counter
  int32_t* n_outliers;    // out: count
  int32_t* col_idx;       // out: ascending outlier columns
  int8_t* Xq;             // out: [M][K]
  float* x_scale;         // out: [M]
  __half* X_O;            // out: [M][ld]
  const __half* W;        // in : [K][N], the fp16 weight transposed (row k = feature k)
  __half* W_O;            // out: [N][ld]
  int ld;
  int32_t* status;        // device status word
  // Token-sharded mode: the outlier set is the OR of given_n bitmaps of
  // ceil(K/32) words each (one per rank, gathered by the caller); detection and
  // the grid barrier are skipped and the OR is written to bitmap.
  const uint32_t* given;
  int given_n;
  // Zero-point codes (scholia section 6) instead of absmax codes when not null:
  // x_scale gets the step (hi - lo)/255 and x_zero [M] the zero point.
  int32_t* x_zero;
};

cudaError_t launch_detect_quantize_compact(const FusedArgs& a, cudaStream_t s);
// Single-pass form of the same step for the absmax codes with detection
// (stream_quant.cu); the launcher above hands those calls to it.
cudaError_t launch_detect_quantize_stream(const FusedArgs& a, cudaStream_t s);

// Host-side launchers of the tensor-core GEMM (gemm_sm100.cu). They encode the
// TMA tensor maps and launch; the return value is the cudaError_t of the launch.
struct GemmArgs {
  const int8_t* Xq;           // [M][K]
  const int8_t* Wq;           // [N][K]
  const __half* X_O;          // [M][ld] compacted outlier columns of X (or nullptr)
  const __half* W_O;          // [N][ld] compacted outlier columns of W (or nullptr)
  int ld;                     // row stride of the panels, multiple of 64
  const float* x_scale;       // [M]
  const float* w_scale;       // [N]
  const int32_t* n_outliers;  // device count, or nullptr for no outlier pass
  const int32_t* x_zero;      // [M] zero points (zero-point codes), or nullptr (absmax codes)
  const int32_t* w_rowsum;    // [N] sum_k Wq[n, k] (with x_zero)
  void* out;                  // fp16 Y [M][N] or int32 C [M][N]
  int M, N, K;
  int32_t* status;            // device status word (may be nullptr)
};

cudaError_t launch_gemm_mixed(const GemmArgs& a, cudaStream_t s);
cudaError_t launch_gemm_i32(const GemmArgs& a, cudaStream_t s);

// Group-scaled GEMM of the W4A4 path (gemm_groups.cu): Y = fp16(sum_g C_g *
// x_absmax[m][g] * w_absmax[n/G][g] / 49) over groups of G columns of K.
// G in {64, 128, 256}; K % 128 == 0, K % G == 0, N % G == 0.
cudaError_t launch_gemm_groups(const int8_t* Xq, const int8_t* Wq, const float* x_absmax,
                               const float* w_absmax, __half* Y, int M, int N, int K, int G,
                               int32_t* status, cudaStream_t s);

// Row-major [rows][cols] tensor map with a box of box_rows x box_bytes (one
// swizzle span wide); defined in gemm_sm100.cu.
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint32_t box_rows, uint32_t box_bytes,
                  CUtensorMapSwizzle swz);
inline bool make_tmap_sw128(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                            int elem_bytes, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_tmap_2d(m, base, dt, elem_bytes, cols, rows, box_rows, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// Decode-shape path (M <= 16): one clustered kernel (decode.cu).
struct DecodeArgs {
  const __half* X;        // [M][K]
  const __half* W;        // [K][N] fp16 weight, transposed (outlier rows are read)
  const int8_t* Wq;       // [N][K]
  const float* w_scale;   // [N]
  __half* Y;              // [M][N]
  int M, N, K;
  float threshold;
  uint32_t* bitmap;       // workspace outputs (written by the first cluster)
  int32_t* n_outliers;
  int32_t* col_idx;
  float* x_scale;
  int8_t* Xq;
  int32_t* status;
  int nbox;               // Wq boxes per CTA (set by launch_decode)
};

bool decode_supported(int M, int K);

// Running column max |x| of an fp16 [rows][K] matrix into fp32 colmax [K]
// (smoothquant.cu) and the top-k column selection into a bitmap (topk.cu).
cudaError_t launch_weight_rowsum(const int8_t* Wq, int N, int K, int32_t* rowsum,
                                 cudaStream_t s);
cudaError_t launch_column_absmax(const __half* X, int rows, int K, float* colmax, cudaStream_t s);
cudaError_t launch_topk_select(const float* colmax, int K, int k, uint32_t* bitmap,
                               cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

// Offline: Wt[k][n] = W[n][k] for an fp16 [N][K] weight (quant_kernels.cu).
cudaError_t launch_transpose_weight(const __half* W, int N, int K, __half* Wt, cudaStream_t s);

// The C-ABI layer's device check (I8MM_OK or I8MM_ERR_UNSUPPORTED_DEVICE /
// I8MM_ERR_CUDA) and its error recorder (the text int8_last_error_string
// returns; I8MM_ERR_CUDA unless e is cudaSuccess), for the other ABI files.
int abi_check_device();
int abi_cuda_fail(const char* what, cudaError_t e);

}  // namespace i8mm

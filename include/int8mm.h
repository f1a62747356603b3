/*
 * int8mm.h - C ABI of libint8mm, the B200 (sm_100a) LLM.int8() mixed-precision
 * decomposition matmul  Y = X . W^T.
 *
 * Method (AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section;
 * tanjunchen "quantization explained part 2", section 1.2):
 *   1. outlier feature columns O of the FP16 activations: any |x| > threshold;
 *   2. per-token (row) absmax INT8 quantisation of the non-outlier columns,
 *      per-output-row absmax INT8 quantisation of W (done once, offline);
 *   3. INT8 x INT8 -> INT32 matrix product;
 *   4. dequantisation by the outer product of the row and column absmax / 127^2;
 *   5. FP16 product over the outlier columns, added into the result.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers, allocated and owned by the
 *     caller. The library never allocates or frees device memory.
 *   - Matrices are row-major and dense (row stride = number of columns):
 *     X [M][K] fp16, W [N][K] fp16 (out-features x in-features), Wq [N][K]
 *     int8, Y [M][N] fp16; the mixed-matmul entry points take the fp16
 *     weight transposed, Wt [K][N] (see int8_transpose_weight). fp16 is IEEE
 *     binary16, passed as `const void*`.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and does no host synchronisation. Device-side
 *     results such as the outlier count stay on the device.
 *   - Argument errors are detected on the host BEFORE anything is launched
 *     and returned as a negative i8mm_status; nothing is written then.
 *     No exception or abort crosses the ABI.
 *   - Requirements: K a positive multiple of 16 and <= 65536; M, N <= 2^22;
 *     every pointer 16-byte aligned; threshold not NaN and >= 0 (+inf
 *     allowed). M == 0 or N == 0 is a valid empty problem and returns
 *     I8MM_OK without launching (int8_find_outlier_cols with M == 0 still
 *     writes a count of 0).
 *   - X is assumed finite; NaN/Inf activations are outside the contract.
 *   - Codes are clamp(rint((x*127)/absmax), -127, 127) with one fp32
 *     product and one correctly rounded fp32 division, rint = round half to
 *     even; a group whose absmax is 0 gets scale 0 and all-zero codes.
 *   - Scales are stored as the absmax itself (fp32); dequantisation
 *     multiplies by x_scale[i] * w_scale[n] / 127^2.
 */
#ifndef INT8MM_H_
#define INT8MM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st* i8mm_stream_t;

typedef enum {
  I8MM_OK = 0,
  I8MM_ERR_INVALID_ARG = -1,        /* null pointer, bad size, NaN/negative threshold */
  I8MM_ERR_ALIGNMENT = -2,          /* a pointer is not 16-byte aligned, or K % 16 != 0 */
  I8MM_ERR_WORKSPACE = -3,          /* workspace null or smaller than the required size */
  I8MM_ERR_CUDA = -4,               /* a CUDA runtime/driver call or launch failed */
  I8MM_ERR_TIMEOUT = -5,            /* a bounded device-side wait gave up (see int8_device_status) */
  I8MM_ERR_UNSUPPORTED_DEVICE = -6  /* the current device is not sm_100 (B200) */
} i8mm_status;

/*
 * Offline weight quantisation (AIInfra LLM.int8() section, "vector-wise
 * quantisation": one scale per weight column of the h x o matrix, i.e. per
 * output row of the [N][K] layout used here).
 *   W        in : fp16 [N][K]
 *   Wq       out: int8 [N][K], codes over the whole row
 *   w_scale  out: fp32 [N], absmax of each row over all K columns
 * Off the per-call hot path: a deployed layer quantises its weight once.
 */
int int8_quantize_weight_rows(const void* W, int N, int K, int8_t* Wq, float* w_scale,
                              i8mm_stream_t stream);

/*
 * Offline layout of the fp16 weight for the outlier product: Wt[k][n] = W[n][k].
 * AIInfra LLM.int8() section: W is h x o (input features x outputs) and the
 * outlier term multiplies the rows W^h of the outlier dimensions h, which are
 * contiguous rows of Wt. The mixed-matmul entry points take this Wt.
 *   W   in : fp16 [N][K] (out features x in features, the PyTorch Linear layout)
 *   Wt  out: fp16 [K][N]; must not overlap W
 * Errors: I8MM_ERR_INVALID_ARG (null pointer, bad sizes), I8MM_ERR_ALIGNMENT
 * (pointers not 16-byte aligned or K not a multiple of 16), I8MM_ERR_CUDA.
 * Off the per-call hot path, like int8_quantize_weight_rows.
 */
int int8_transpose_weight(const void* W, int N, int K, void* Wt, i8mm_stream_t stream);

/*
 * Outlier feature-column detection (AIInfra LLM.int8() section, "detection:
 * set a magnitude threshold"; tanjunchen section 1.2: a channel whose
 * activation magnitude exceeds the threshold, 6.0 by default).
 * Column j is an outlier iff |float(X[i][j])| > threshold for some row i
 * of this X (strict comparison in fp32).
 *   X           in : fp16 [M][K]
 *   col_bitmap  out: uint32 [ceil(K/32)], bit (j%32) of word (j/32) set for outliers
 *   n_outliers  out: int32 [1] on the device, the number of outlier columns
 *   col_idx     out: int32 [K], outlier column indices in ascending order in the
 *                    first n_outliers entries (the rest is unspecified); may be NULL
 */
int int8_find_outlier_cols(const void* X, int M, int K, float threshold,
                           uint32_t* col_bitmap, int32_t* n_outliers, int32_t* col_idx,
                           i8mm_stream_t stream);

/*
 * Per-token absmax INT8 quantisation of the non-outlier part (AIInfra
 * LLM.int8() section, vector-wise quantisation of each row of X after the
 * outliers are separated; tanjunchen section 1.2, the 4096-dim example).
 *   X          in : fp16 [M][K]
 *   col_bitmap in : uint32 [ceil(K/32)] as produced by int8_find_outlier_cols
 *   Xq         out: int8 [M][K], 0 at outlier columns
 *   x_scale    out: fp32 [M], absmax of each row over the non-outlier columns
 */
int int8_quantize_act_rows(const void* X, int M, int K, const uint32_t* col_bitmap,
                           int8_t* Xq, float* x_scale, i8mm_stream_t stream);

/* Bytes of device workspace int8_mixed_matmul needs for these sizes (0 on bad sizes). */
size_t int8_mixed_matmul_workspace_size(int M, int N, int K);

/*
 * Where int8_mixed_matmul leaves its intermediates inside the workspace
 * (byte offsets from the workspace base; each at least 16-byte aligned). Lets a
 * caller or a test read the outlier set, codes and scales of the last call.
 * The outlier panels have row stride panel_ld elements (fp16) and hold the
 * compacted outlier columns in ascending column order, zero-padded to a
 * multiple of 16 columns (one K step of the tensor-core outlier product; the
 * zero-point path pads to 64). Columns past the padding are never read.
 * Nothing is written to them when there are no outliers.
 */
typedef struct {
  size_t n_outliers;   /* int32 [1] */
  size_t status;       /* int32 [1], device status word (0 = ok) */
  size_t col_bitmap;   /* uint32 [ceil(K/32)] */
  size_t col_idx;      /* int32 [K] */
  size_t x_scale;      /* fp32 [M] */
  size_t Xq;           /* int8 [M][K] */
  size_t X_O;          /* fp16 [M][panel_ld] */
  size_t W_O;          /* fp16 [N][panel_ld] */
  size_t total;        /* == int8_mixed_matmul_workspace_size(M, N, K) */
  int panel_ld;        /* = K rounded up to a multiple of 64 */
} i8mm_workspace_layout;

int int8_mixed_matmul_workspace_layout(int M, int N, int K, i8mm_workspace_layout* out);

/*
 * The whole decomposition (AIInfra LLM.int8() section: C_i32 = X_i8 x W_i8,
 * C_normal = C_i32 / (c_x (x) c_w), C_outlier = sum_{h in O} X_f16^h W_f16^h,
 * C_f16 = C_outlier + C_normal).
 *   X          in : fp16 [M][K] activations
 *   Wq,w_scale in : from int8_quantize_weight_rows
 *   Wt_fp16    in : fp16 [K][N], the unquantised weight in the pages' h x o
 *                   orientation (row k holds input feature k for every output
 *                   n; int8_transpose_weight makes it from the [N][K] weight
 *                   once, offline); only the rows of the outlier features are
 *                   read, each contiguously
 *   threshold  in : outlier magnitude threshold (6.0 in the pages)
 *   Y          out: fp16 [M][N], Y = fp16(C_i32*x_scale*w_scale/127^2 + C_outlier),
 *                   the sum formed in fp32 and rounded once
 *   workspace  in : device scratch of at least int8_mixed_matmul_workspace_size(M,N,K)
 *                   bytes, 256-byte aligned; contents on entry are ignored
 * One call launches the detection, quantisation/compaction and GEMM kernels
 * back to back on `stream`; the outlier count never leaves the device.
 */
int int8_mixed_matmul(const void* X, const int8_t* Wq, const float* w_scale,
                      const void* Wt_fp16, int M, int N, int K, float threshold, void* Y,
                      void* workspace, size_t workspace_bytes, i8mm_stream_t stream);

/*
 * Measurement hook: exactly int8_mixed_matmul, and in addition records three
 * CUDA events (cudaEvent_t, created by the caller) on `stream`:
 *   events[0] before the first operation of the call,
 *   events[1] after the detection and quantisation/compaction kernels,
 *   events[2] after the GEMM kernel.
 * The elapsed times events[0]->events[1] and events[1]->events[2] are the
 * device durations of the memory-bound stage and of the tensor-core GEMM.
 */
int int8_mixed_matmul_profiled(const void* X, const int8_t* Wq, const float* w_scale,
                               const void* Wt_fp16, int M, int N, int K, float threshold,
                               void* Y, void* workspace, size_t workspace_bytes,
                               i8mm_stream_t stream, void* const* events);

// ---------------------------------------------------------------- zero-point rows
// [Scholia] "Inference Quantization" notes, section 6: affine codes
// q = clip(round(x/s) + z, qmin, qmax), x_hat = s(q - z), z the integer that
// represents real 0; [AIInfra] "05Quantization01", LLM.int8() section: the
// outliers are one-sided, which is where zeropoint beats absmax. Here the
// non-outlier part of each token is quantised with a zero point: over its
// non-outlier columns lo = min(0, min x), hi = max(0, max x), step =
// fl32(fl32(hi - lo)/255), z = clamp(-128 - rint(fl32(lo/step)), -128, 127),
// q = clamp(rint(fl32(x/step)) + z, -128, 127), and q = z at outlier columns.
// The INT8 product then needs sum_k (q - z) Wq[n,k] = C - z * sum_k Wq[n,k], so
// Y = fp16((C - z*rowsum[n]) * step * w_scale[n] / 127 + X_O.W_O^T).

// rowsum[n] = sum_k Wq[n][k] (int32 [N]), once per weight (offline).
int int8_weight_rowsum(const int8_t* Wq, int N, int K, int32_t* rowsum, i8mm_stream_t stream);

// The decomposition with zero-point codes. Arguments, layout and errors as
// int8_mixed_matmul plus w_rowsum (from int8_weight_rowsum, 16-byte aligned)
// and the larger workspace below. In the workspace x_scale holds the step and
// an int32 [M] array of zero points follows the regular layout (256-byte
// aligned). Always runs the prefill kernels.
size_t int8_mixed_matmul_zp_workspace_size(int M, int N, int K);
int int8_mixed_matmul_zp(const void* X, const int8_t* Wq, const float* w_scale,
                         const int32_t* w_rowsum, const void* Wt_fp16, int M, int N, int K,
                         float threshold, void* Y, void* workspace, size_t workspace_bytes,
                         i8mm_stream_t stream);

// ---------------------------------------------------------------- top-k decomposition
// [AIInfra] "05Quantization01", LLM.int8() section, training notes: raise the
// decomposition ratio by computing the top 1% or 2% largest-magnitude feature
// dimensions in FP16. The outlier set is the k columns of X with the largest
// max |x| over the M tokens (ties to the lower column index; k >= K selects all
// columns); the rest of the path is int8_mixed_matmul with that set (per-token
// absmax codes of the other columns, INT8 product, FP16 product over the set).
// Arguments, layout and errors as int8_mixed_matmul, except k (>= 0) instead
// of the threshold and the larger workspace below; the workspace's bitmap,
// count and list describe the selected set. Always runs the prefill kernels.
size_t int8_mixed_matmul_topk_workspace_size(int M, int N, int K);
int int8_mixed_matmul_topk(const void* X, const int8_t* Wq, const float* w_scale,
                           const void* Wt_fp16, int M, int N, int K, int k, void* Y,
                           void* workspace, size_t workspace_bytes, i8mm_stream_t stream);

// ---------------------------------------------------------------- SmoothQuant W8A8
// [Tanjunchen] "quantization explained part 2", section 4: per input channel i,
// X_i / s_i and W_i * s_i with s_i = max|X_i|^alpha / max|W_i|^(1-alpha) leave
// X.W unchanged (4.2) and make the activations quantisable, so both operands
// are INT8 (W8A8, no outlier split). s is computed offline from calibration
// activations (4.4). Here W is [N][K], so W_i is column i; the INT8 scheme after
// smoothing is per token for X and per output row for W, codes
// clamp(rint(fl32(fl32(v*127)/absmax)), +-127) of the smoothed fp32 values v.

// colmax[k] = max(colmax[k], max over rows of |X[row][k]|) for an fp16 [rows][K]
// matrix (running calibration statistic; also the weight's column maxima).
// colmax: device fp32 [K], 16-byte aligned, initialised by the caller (0 to start).
int int8_column_absmax(const void* X, int rows, int K, float* colmax, i8mm_stream_t stream);

// s[k] = act_absmax[k]^alpha / w_absmax[k]^(1-alpha) (1 where either is 0) and,
// if s_rcp is not null, s_rcp[k] = fl32(1/s[k]) (correctly rounded).
// alpha in [0, 1]. All device fp32 [K].
int int8_smoothquant_factors(const float* act_absmax, const float* w_absmax, int K, float alpha,
                             float* s, float* s_rcp, i8mm_stream_t stream);

// Offline weight side: W_hat = fl32(W[n][k] * s[k]), quantised per output row.
// W fp16 [N][K] -> Wq int8 [N][K], w_scale fp32 [N] (row absmax of W_hat).
int int8_smoothquant_weight_rows(const void* W, const float* s, int N, int K, int8_t* Wq,
                                 float* w_scale, i8mm_stream_t stream);

// Bytes of workspace int8_smoothquant_matmul needs (0 for invalid sizes).
size_t int8_smoothquant_workspace_size(int M, int N, int K);

// Runtime W8A8 path: X_hat = fl32(X[m][k] * s_rcp[k]), per-token absmax codes
// (Xq and x_scale left in the workspace), INT8 x INT8 -> INT32 on the tensor
// cores, Y = fp16(C * x_scale * w_scale / 127^2). X fp16 [M][K], Wq/w_scale from
// int8_smoothquant_weight_rows, s_rcp fp32 [K], Y fp16 [M][N]. Alignment,
// workspace and error rules as int8_mixed_matmul (256-byte aligned workspace).
int int8_smoothquant_matmul(const void* X, const int8_t* Wq, const float* w_scale,
                            const float* s_rcp, int M, int N, int K, void* Y, void* workspace,
                            size_t workspace_bytes, i8mm_stream_t stream);

// ---------------------------------------------------------------- grouped Hadamard rotation
// developer.baidu.com "分组旋转方法从W8A8到W4A4" (grouped rotation from W8A8 to
// W4A4), sections 2, 5.1, 5.2, 5.4: before quantising, both operands are
// multiplied along K by the block-diagonal orthogonal matrix with blocks
// H_G/sqrt(G) (H_G the Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i&j)),
// which leaves X W^T unchanged and spreads an outlier channel over its group.
// G is 16, 32, 64, 128 or 256 and divides K; K <= 32768. The rotated value of an
// fp16 row is r = fl32(fl32(S) * fl32(1/sqrt(G))), S the exact +-1 sum over the
// group. Codes clamp(rint(fl32(fl32(r*qmax)/a)), +-qmax), a the group's absmax
// (0 gives 0), qmax 127 (W8A8) or 7 (W4A4, the symmetric INT4 grid).

// W8A8 side: rotate each row of X fp16 [rows][K], one absmax per row over all K:
// Xq int8 [rows][K], absmax fp32 [rows]; R (optional, may be null) fp32
// [rows][K] receives the rotated values. Serves the weight offline (rows = N)
// and the activations. X, Xq, R 16-byte aligned.
int int8_rotate_quantize_rows(const void* X, int rows, int K, int G, int8_t* Xq, float* absmax,
                              float* R, i8mm_stream_t stream);

// Bytes of workspace int8_rotated_matmul needs (0 for invalid sizes).
size_t int8_rotated_workspace_size(int M, int N, int K);

// Runtime W8A8 path after rotation: rotate and quantise X per token (Xq and
// x_scale left in the workspace: status 16 B, x_scale fp32 [M], Xq int8 [M][K],
// each 256-byte aligned), INT8 x INT8 -> INT32 on the tensor cores, Y =
// fp16(C * x_scale * w_scale / 127^2). Wq int8 [N][K] and w_scale fp32 [N] come
// from int8_rotate_quantize_rows on the weight with the same G. No outlier
// split. Alignment, workspace and error rules as int8_mixed_matmul.
int int8_rotated_matmul(const void* X, const int8_t* Wq, const float* w_scale, int M, int N, int K,
                        int G, void* Y, void* workspace, size_t workspace_bytes,
                        i8mm_stream_t stream);

// W4A4 activation side: rotate, one absmax per (row, group of G columns):
// absmax fp32 [rows][K/G]; Xq (optional) int8 [rows][K] holds the codes one
// per byte (the form the INT8 tensor cores read), Xp (optional) uint32
// [rows][K/8] holds them packed: code j of each run of eight along K in bits
// 4j..4j+3 (two's complement nibble). At least one of Xq, Xp; X, Xq 16-byte
// and Xp 8-byte aligned.
int int4_rotate_quantize_groups(const void* X, int rows, int K, int G, int8_t* Xq, uint32_t* Xp,
                                float* absmax, i8mm_stream_t stream);

// W4A4 weight side (offline): rotate the rows of W fp16 [N][K], one absmax per
// G x G sub-block (G output rows by G columns): absmax fp32 [N/G][K/G]; codes
// packed as in int4_rotate_quantize_groups into Wp uint32 [N][K/8]. N % G == 0.
int int4_rotate_quantize_weight_blocks(const void* W, int N, int K, int G, uint32_t* Wp,
                                       float* absmax, i8mm_stream_t stream);

// Packed 4-bit codes (as written by the two functions above) to one signed
// byte each: P uint32 [rows][K/8] -> Q int8 [rows][K]. K % 32 == 0; P and Q
// 16-byte aligned. The 4-bit product runs on the INT8 tensor cores (sm_100a
// has no 4-bit integer MMA), so the weight is expanded once, at load time.
int int4_unpack(const uint32_t* P, int rows, int K, int8_t* Q, i8mm_stream_t stream);

// Bytes of workspace int4_rotated_matmul needs (0 for invalid sizes).
size_t int4_rotated_workspace_size(int M, int N, int K, int G);

// Runtime W4A4 path after rotation: rotate X and quantise it per (token, group)
// (workspace: status 16 B, x_absmax fp32 [M][K/G], Xq int8 [M][K], each 256-byte
// aligned), then Y = fp16(sum_g C_g * x_absmax[m][g] * w_absmax[n/G][g] / 7^2),
// C_g the INT32 product over group g on the tensor cores. Wq4 int8 [N][K] holds
// the weight's 4-bit codes one per byte (int4_unpack of the packed words of
// int4_rotate_quantize_weight_blocks), w_absmax fp32 [N/G][K/G] its block
// maxima. G in {64, 128, 256}; K % 128 == 0; N % G == 0. Alignment, workspace
// and error rules as int8_mixed_matmul.
int int4_rotated_matmul(const void* X, const int8_t* Wq4, const float* w_absmax, int M, int N,
                        int K, int G, void* Y, void* workspace, size_t workspace_bytes,
                        i8mm_stream_t stream);

// Token-sharded (data-parallel over tokens) form of int8_mixed_matmul, one call
// per rank on that rank's rows of X. AIInfra "05Quantization01", LLM.int8()
// section: the outlier feature dimensions are those where any token of the
// batch exceeds the threshold, so ranks holding parts of one batch must agree
// on one set. Each rank runs int8_find_outlier_cols on its own rows, the ranks
// gather their bitmaps (one collective, ceil(K/32) words per rank), and each
// calls this with all of them: the outlier set is their bitwise OR, and the
// rest (per-token quantisation, INT8 product, outlier product, sum) is exactly
// int8_mixed_matmul restricted to the rank's rows. Concatenating the ranks' Y
// gives, element for element, the Y of one int8_mixed_matmul over the whole batch.
//   X        device fp16 [M][K], this rank's tokens (M may be 0)
//   bitmaps  device u32 [n_bitmaps][ceil(K/32)], read only; 4-byte aligned
//   other arguments, layout, workspace and errors as int8_mixed_matmul; the
//   workspace's bitmap holds the OR afterwards. Always runs the prefill kernels.
int int8_mixed_matmul_sharded(const void* X, const int8_t* Wq, const float* w_scale,
                              const void* Wt_fp16, int M, int N, int K, const uint32_t* bitmaps,
                              int n_bitmaps, void* Y, void* workspace, size_t workspace_bytes,
                              i8mm_stream_t stream);

/*
 * Measurement hook: one stage of int8_mixed_matmul on its own, so that each
 * kernel can be timed back to back.
 *   stage 1: clear the control words and run the detection / quantisation /
 *            compaction kernel (writes the workspace intermediates);
 *   stage 2: run only the GEMM kernel on the intermediates already in the
 *            workspace (a previous stage 1 or full call with the same X, sizes,
 *            threshold and workspace must have completed on the stream).
 * Other arguments as for int8_mixed_matmul; any other stage value is
 * I8MM_ERR_INVALID_ARG.
 */
int int8_mixed_matmul_stage(int stage, const void* X, const int8_t* Wq, const float* w_scale,
                            const void* Wt_fp16, int M, int N, int K, float threshold, void* Y,
                            void* workspace, size_t workspace_bytes, i8mm_stream_t stream);

/*
 * Test hook: the INT8 x INT8 -> INT32 product alone (AIInfra LLM.int8()
 * section, "C_i32 = X_i8 x W_i8", accumulated in INT32), on the same
 * tensor-core kernel the full path uses.
 *   C out: int32 [M][N], C[i][n] = sum_k Xq[i][k] * Wq[n][k]
 */
int int8_debug_gemm_i32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K, int32_t* C,
                        i8mm_stream_t stream);

/*
 * Self-test of the bounded device-side waits: launches one CTA that waits on an
 * mbarrier phase nothing completes; after the library's wait limit (2 s) the
 * wait gives up and the CTA writes I8MM_ERR_TIMEOUT into *status (device int32,
 * cleared first) and exits normally. Returns I8MM_OK once launched; the caller
 * synchronises `stream` and reads *status. Nothing faults or hangs.
 */
int int8_selftest_wait_timeout(int32_t* status, i8mm_stream_t stream);

/*
 * Reads the device status word a previous int8_mixed_matmul left in its
 * workspace (synchronises `stream`). Returns I8MM_OK, I8MM_ERR_TIMEOUT if
 * a bounded device-side wait gave up, or I8MM_ERR_CUDA.
 */
int int8_device_status(const void* workspace, i8mm_stream_t stream);

/*
 * int8_mixed_matmul without a workspace argument, for callers that cannot give
 * the library device memory: for example code whose host framework owns every
 * device allocation and offers it no allocator, or code that must not grow its
 * device memory use while it runs. The paper has no counterpart to this entry
 * point; it is an interface convenience of this library.
 *   Arguments and results are those of int8_mixed_matmul.
 *   Scratch: a fixed device array built into the library,
 *            I8MM_NOALLOC_SCRATCH_BYTES (64 MiB), which every GPU that loads
 *            the library holds until the process exits. Nothing is allocated
 *            or freed by the call.
 *   Limit:   problems with int8_mixed_matmul_workspace_size(M, N, K) larger
 *            than I8MM_NOALLOC_SCRATCH_BYTES return I8MM_ERR_WORKSPACE.
 *   Set-up:  the first call on a device looks up the array's device address
 *            (with that device current) and caches it; make that first call
 *            before any stream capture.
 *   Sharing: all calls on a device use the same array, which keeps the last
 *            call's contents (each call clears the words it needs first).
 *            Calls that can overlap on the GPU (several streams or host
 *            threads) race on the array; the caller must serialise them.
 *   Status:  a bounded device-side wait that gives up writes I8MM_ERR_TIMEOUT
 *            into the array's status word (cleared by every call);
 *            int8_noalloc_device_status reads it.
 *   Errors:  those of int8_mixed_matmul; a device other than sm_100 returns
 *            I8MM_ERR_UNSUPPORTED_DEVICE before the array is looked up.
 */
#define I8MM_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int int8_mixed_matmul_noalloc(const void* X, const int8_t* Wq, const float* w_scale,
                              const void* Wt_fp16, int M, int N, int K, float threshold,
                              void* Y, i8mm_stream_t stream);

/*
 * The device status word of the last int8_mixed_matmul_noalloc call on the
 * current device (synchronises `stream`; reads 4 bytes into host memory, no
 * allocation). Returns I8MM_OK, I8MM_ERR_TIMEOUT if a bounded device-side wait
 * of that call gave up, I8MM_ERR_UNSUPPORTED_DEVICE on a device other than
 * sm_100, or I8MM_ERR_CUDA.
 */
int int8_noalloc_device_status(i8mm_stream_t stream);

/* Static string for a status code. */
const char* int8_status_string(int status);

/*
 * Text of the CUDA error behind the last I8MM_ERR_CUDA returned on the
 * calling host thread (which call failed and the CUDA error name), or "" if
 * none. The pointer stays valid until the thread's next failing call.
 */
const char* int8_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* INT8MM_H_ */

// Tensor-core GEMM of the LLM.int8() path on sm_100a (B200).
//
//   Y[i][n] = fp16( C_i32[i][n] * x_scale[i] * w_scale[n] / 127^2 + C_out[i][n] )
//   C_i32   = Xq . Wq^T          tcgen05.mma kind::i8, INT32 accumulator in TMEM
//   C_out   = X_O . W_O^T        the FP16 product over the outlier columns
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section:
// INT8 matmul accumulated in INT32, dequantisation by the outer product of the
// row and column scales, FP16 matmul over the outlier dimensions, final sum.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles walked with stride
// gridDim.x (M-tile index fastest, so the CTAs in flight share Wq column blocks
// and all of Xq through L2). Warp roles:
//   warp 0      TMA producer: 128-byte-swizzled K-blocks (128 int8 columns of
//               Xq and Wq) into a STAGES-deep shared-memory ring that runs
//               continuously across tiles
//   warp 1      owns the 512-column TMEM allocation; one lane issues the MMAs
//               (4 x K=32 per K-block) and commits
//   warps 2-9   epilogue: tcgen05.ld (thread = output row, two warps per TMEM
//               lane quarter splitting the 256 columns), dequantise, add the
//               outlier product, round to fp16, store
// Two ways of forming C_out, chosen on the device from the outlier count:
//   count <= kCcMax  on CUDA cores in the epilogue (fp16 products are exact in
//                    fp32; <= 16 FMAs per output). The two 256-column INT32
//                    accumulators are double-buffered, so the epilogue of one
//                    tile overlaps the MMAs of the next.
//   count >  kCcMax  on the tensor cores: the compacted fp16 panels X_O, W_O are
//                    streamed through the same ring after the int8 K-blocks and
//                    multiplied with kind::f16 into an FP32 accumulator in the
//                    other half of TMEM (single-buffered).
// The outlier count is read from device memory, so the host never syncs.
// No clusters and no TMA multicast are used. Every mbarrier wait is bounded;
// a wait that gives up records I8MM_ERR_TIMEOUT in the status word and the
// CTA stops issuing work.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int BM = 128;              // rows of the output tile (TMEM lanes)
constexpr int BN = 256;              // columns of the output tile
constexpr int KB_I8 = 128;           // int8 columns per K-block (128 bytes)
constexpr int KB_F16 = 64;           // fp16 columns per panel block (128 bytes)
constexpr int STAGES = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kCcMax = 16;           // outlier counts handled on CUDA cores
constexpr int kStatusTimeout = -5;   // == I8MM_ERR_TIMEOUT

constexpr int A_BYTES = BM * 128;
constexpr int B_BYTES = BN * 128;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int WO_BYTES = kCcMax * BN * 4;   // W_O tile, fp32, [j][column]
constexpr int SW_BYTES = BN * 4;            // w_scale tile
constexpr int BAR_OFF = RING_BYTES + WO_BYTES + SW_BYTES;
constexpr int BAR_BYTES = (2 * STAGES + 4) * 8 + 16;
constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + BAR_OFF + BAR_BYTES;
constexpr uint32_t TMEM_COLS = 512;

__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
}

template <bool OUT_I32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_persistent_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB,
                              const __grid_constant__ CUtensorMap tmXO,
                              const __grid_constant__ CUtensorMap tmWO,
                              const float* __restrict__ x_scale,
                              const float* __restrict__ w_scale,
                              const int32_t* __restrict__ n_outliers,
                              const __half* __restrict__ X_O, const __half* __restrict__ W_O,
                              int ld, void* __restrict__ out, int M, int N, int K,
                              int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* wo_s = reinterpret_cast<float*>(smem + RING_BYTES);            // [kCcMax][BN]
  float* sw_s = reinterpret_cast<float*>(smem + RING_BYTES + WO_BYTES);  // [BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!OUT_I32) {
      tma_prefetch_desc(&tmXO);
      tma_prefetch_desc(&tmWO);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int count = (!OUT_I32 && n_outliers) ? *n_outliers : 0;
  const bool tc_out = count > kCcMax;          // outlier product on the tensor cores
  const int nk = (K + KB_I8 - 1) / KB_I8;
  const int np = tc_out ? (count + KB_F16 - 1) / KB_F16 : 0;
  const int iters = nk + np;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t g = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * BM;
        const int n0 = (tile / m_tiles) * BN;
        for (int it = 0; it < iters; ++it, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            record_error(status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* a = smem + s * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          if (it < nk) {
            tma_load_2d(a, &tmA, &full[s], it * KB_I8, m0);
            tma_load_2d(b, &tmB, &full[s], it * KB_I8, n0);
          } else {
            const int p = it - nk;
            tma_load_2d(a, &tmXO, &full[s], p * KB_F16, m0);
            tma_load_2d(b, &tmWO, &full[s], p * KB_F16, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_i8 = make_idesc(2 /*s32*/, 1 /*signed*/, BM, BN);
      constexpr uint32_t idesc_f16 = make_idesc(1 /*f32*/, 0 /*fp16*/, BM, BN);
      uint32_t g = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x, ++local) {
        const int buf = tc_out ? 0 : (local & 1);
        const uint32_t aph = tc_out ? (local & 1) : ((local >> 1) & 1);
        if (!mbar_wait(&acc_empty[buf], aph ^ 1)) {
          record_error(status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_i32 = tmem + buf * BN;
        const uint32_t d_f32 = tmem + BN;
        bool ok = true;
        for (int it = 0; it < iters; ++it, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&full[s], ph)) {
            record_error(status, kStatusTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_addr(smem + s * STAGE_BYTES);
          const uint32_t b = a + A_BYTES;
          if (it < nk) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(d_i32, sw128_kmajor_desc(a + 32 * kk), sw128_kmajor_desc(b + 32 * kk),
                     idesc_i8, (it | kk) != 0);
          } else {
            const int p = it - nk;
            const int steps = min(4, (count - p * KB_F16 + 15) / 16);
            for (int kk = 0; kk < steps; ++kk)
              mma_f16(d_f32, sw128_kmajor_desc(a + 32 * kk), sw128_kmajor_desc(b + 32 * kk),
                      idesc_f16, (p | kk) != 0);
          }
          mma_commit(&empty[s]);
        }
        mma_commit(&acc_full[buf]);
        if (!ok) break;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;       // which 128 of the 256 columns
    const int et = threadIdx.x - 64;        // 0..255
    const bool cc_out = !OUT_I32 && !tc_out && count > 0;
    const bool vec_ok = (N % 8) == 0;
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int m0 = (tile % m_tiles) * BM;
      const int n0 = (tile / m_tiles) * BN;
      const int buf = tc_out ? 0 : (local & 1);
      const uint32_t aph = tc_out ? (local & 1) : ((local >> 1) & 1);
      const int row = m0 + q * 32 + lane;

      // Per-tile column data (w_scale, W_O tile as fp32) and this row's X_O values.
      if (!OUT_I32) {
        const int n = n0 + et;
        sw_s[et] = (n < N) ? w_scale[n] : 0.0f;
        if (cc_out) {
          for (int j = 0; j < kCcMax; ++j)
            wo_s[j * BN + et] =
                (n < N && j < count) ? __half2float(W_O[static_cast<size_t>(n) * ld + j]) : 0.0f;
        }
      }
      float xo[kCcMax];
      float rs = 0.0f;
      if (!OUT_I32) {
        if (row < M) rs = x_scale[row] * (1.0f / 16129.0f);
#pragma unroll
        for (int j = 0; j < kCcMax; ++j)
          xo[j] = (cc_out && row < M && j < count)
                      ? __half2float(X_O[static_cast<size_t>(row) * ld + j])
                      : 0.0f;
      }
      epi_sync();

      const bool ok = mbar_wait(&acc_full[buf], aph);
      if (!ok) {
        record_error(status, kStatusTimeout);
        *abort_flag = 1;
      }
      tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = half * 128; c < half * 128 + 128 && ok; c += 32) {
        __syncwarp();
        uint32_t acc[32];
        uint32_t oacc[32];
        tmem_ld_32x32b_x32(lane_base + buf * BN + c, acc);
        if (tc_out) tmem_ld_32x32b_x32(lane_base + BN + c, oacc);
        tmem_ld_wait();
        const int col0 = n0 + c;
        if (row < M && col0 < N) {
          if constexpr (OUT_I32) {
            int32_t* orow = reinterpret_cast<int32_t*>(out) + static_cast<size_t>(row) * N;
            if (vec_ok && col0 + 32 <= N) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<uint4*>(orow + col0 + j) =
                    make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) orow[col0 + j] = static_cast<int32_t>(acc[j]);
            }
          } else {
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              y[j] = static_cast<float>(static_cast<int32_t>(acc[j])) * (rs * sw_s[c + j]);
            if (tc_out) {
#pragma unroll
              for (int j = 0; j < 32; ++j) y[j] += __uint_as_float(oacc[j]);
            } else if (cc_out) {
              float o[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = 0.0f;
#pragma unroll
              for (int t = 0; t < kCcMax; ++t) {
                if (t < count) {
                  const float4* w4 = reinterpret_cast<const float4*>(wo_s + t * BN + c);
#pragma unroll
                  for (int j = 0; j < 8; ++j) {
                    const float4 w = w4[j];
                    o[4 * j + 0] = fmaf(xo[t], w.x, o[4 * j + 0]);
                    o[4 * j + 1] = fmaf(xo[t], w.y, o[4 * j + 1]);
                    o[4 * j + 2] = fmaf(xo[t], w.z, o[4 * j + 2]);
                    o[4 * j + 3] = fmaf(xo[t], w.w, o[4 * j + 3]);
                  }
                }
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) y[j] += o[j];
            }
            __half* orow = reinterpret_cast<__half*>(out) + static_cast<size_t>(row) * N;
            if (vec_ok && col0 + 32 <= N) {
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 v;
                __half2* h = reinterpret_cast<__half2*>(&v);
                h[0] = __floats2half2_rn(y[j], y[j + 1]);
                h[1] = __floats2half2_rn(y[j + 2], y[j + 3]);
                h[2] = __floats2half2_rn(y[j + 4], y[j + 5]);
                h[3] = __floats2half2_rn(y[j + 6], y[j + 7]);
                *reinterpret_cast<uint4*>(orow + col0 + j) = v;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) orow[col0 + j] = __float2half_rn(y[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      epi_sync();   // the tile's sw_s / wo_s are no longer read
      if (!ok || *abort_flag) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major [rows][cols] matrix, box of box_rows x (128 bytes), 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
               uint64_t cols, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool OUT_I32>
cudaError_t launch(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap maps[4];
  std::memset(maps, 0, sizeof(maps));
  if (!make_tmap(&maps[0], a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.M, BM) ||
      !make_tmap(&maps[1], a.Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.N, BN))
    return cudaErrorInvalidValue;
  if (!OUT_I32 && a.X_O && a.W_O) {
    if (!make_tmap(&maps[2], a.X_O, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.ld, a.M, BM) ||
        !make_tmap(&maps[3], a.W_O, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.ld, a.N, BN))
      return cudaErrorInvalidValue;
  } else {
    maps[2] = maps[0];
    maps[3] = maps[1];
  }
  auto kern = gemm_i8_persistent_kernel<OUT_I32>;
  static bool attr_set[64] = {};  // per instantiation and device
  static int sm_count[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 64) {
      attr_set[dev] = true;
      sm_count[dev] = sms;
    }
  }
  const int sms = dev < 64 ? sm_count[dev] : 148;
  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = (a.N + BN - 1) / BN;
  const int tiles = m_tiles * n_tiles;
  const int grid = tiles < sms ? tiles : sms;
  kern<<<grid, kThreads, SMEM_BYTES, s>>>(maps[0], maps[1], maps[2], maps[3], a.x_scale,
                                          a.w_scale, OUT_I32 ? nullptr : a.n_outliers, a.X_O,
                                          a.W_O, a.ld, a.out, a.M, a.N, a.K, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_mixed(const GemmArgs& a, cudaStream_t s) { return launch<false>(a, s); }

cudaError_t launch_gemm_i32(const GemmArgs& a, cudaStream_t s) { return launch<true>(a, s); }

}  // namespace i8mm

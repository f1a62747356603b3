// Tensor-core GEMM of the LLM.int8() path on sm_100a (B200).
//
//   Y[i][n] = fp16( C_i32[i][n] * x_scale[i] * w_scale[n] / 127^2 + C_out[i][n] )
//   C_i32   = Xq . Wq^T          (tcgen05.mma kind::i8, INT32 accumulator in TMEM)
//   C_out   = X_O . W_O^T        (tcgen05.mma kind::f16, FP32 accumulator in TMEM)
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section:
// INT8 matmul accumulated in INT32, dequantisation by the outer product of the
// row and column scales, FP16 matmul over the outlier dimensions, final sum.
//
// One CTA computes one 128 x BN output tile:
//   warp 0      TMA producer: 128-byte-swizzled K-blocks of Xq/Wq (128 int8
//               columns), then of the compacted fp16 outlier panels (64 fp16
//               columns), into a STAGES-deep shared-memory ring
//   warp 1      owns the TMEM allocation; one lane issues the MMAs
//               (4 x K=32 int8 steps per int8 block, up to 4 x K=16 fp16 steps
//               per panel block, skipping all-zero padding steps)
//   warps 2-5   epilogue: tcgen05.ld both accumulators (thread = output row),
//               dequantise, add, round to fp16, store
// The outlier count is read from device memory, so the host never syncs.
// No clusters and no TMA multicast are used.
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
constexpr int KB_I8 = 128;           // int8 columns per K-block (128 bytes)
constexpr int KB_F16 = 64;           // fp16 columns per panel block (128 bytes)
constexpr int kThreads = 192;        // 6 warps
constexpr int kStatusTimeout = -5;   // == I8MM_ERR_TIMEOUT

template <int BN, int STAGES>
struct Cfg {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  // barriers: full[STAGES], empty[STAGES], done; then tmem slot + flag; then w_scale tile
  static constexpr int BAR_BYTES = (2 * STAGES + 1) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + RING_BYTES + BAR_BYTES + BN * 4;
  static constexpr uint32_t TMEM_COLS = 2 * BN;  // INT32 acc + FP32 outlier acc
};

__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

template <int BN, int STAGES, bool OUT_I32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_mixed_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmXO,
                         const __grid_constant__ CUtensorMap tmWO,
                         const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                         const int32_t* __restrict__ n_outliers, void* __restrict__ out, int M,
                         int N, int K, int32_t* status) {
  using C = Cfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* sw_tile = reinterpret_cast<float*>(smem + C::RING_BYTES + C::BAR_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int m0 = (blockIdx.x % m_tiles) * BM;
  const int n0 = (blockIdx.x / m_tiles) * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!OUT_I32) {
      tma_prefetch_desc(&tmXO);
      tma_prefetch_desc(&tmWO);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int count = (!OUT_I32 && n_outliers) ? *n_outliers : 0;
  const int nk = (K + KB_I8 - 1) / KB_I8;
  const int np = (count + KB_F16 - 1) / KB_F16;
  const int total = nk + np;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      for (int it = 0; it < total; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          record_error(status, kStatusTimeout);
          break;
        }
        uint8_t* a = smem + s * C::STAGE_BYTES;
        uint8_t* b = a + C::A_BYTES;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
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
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_i8 = make_idesc(2 /*s32*/, 1 /*signed*/, BM, BN);
      constexpr uint32_t idesc_f16 = make_idesc(1 /*f32*/, 0 /*fp16*/, BM, BN);
      for (int it = 0; it < total; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&full[s], ph)) {
          record_error(status, kStatusTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_addr(smem + s * C::STAGE_BYTES);
        const uint32_t b = a + C::A_BYTES;
        if (it < nk) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem, sw128_kmajor_desc(a + 32 * kk), sw128_kmajor_desc(b + 32 * kk),
                   idesc_i8, (it | kk) != 0);
        } else {
          const int p = it - nk;
          const int steps = min(4, (count - p * KB_F16 + 15) / 16);
          for (int kk = 0; kk < steps; ++kk)
            mma_f16(tmem + BN, sw128_kmajor_desc(a + 32 * kk), sw128_kmajor_desc(b + 32 * kk),
                    idesc_f16, (p | kk) != 0);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(done);
    }
  } else {
    // ---------------- epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
    const int et = threadIdx.x - 64;
    if (!OUT_I32)
      for (int j = et; j < BN; j += 128) sw_tile[j] = (n0 + j < N) ? w_scale[n0 + j] : 0.0f;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    if (!mbar_wait(done, 0)) record_error(status, kStatusTimeout);
    tc_fence_after();
    float rs = 0.0f;
    if (!OUT_I32 && row < M) rs = x_scale[row] * (1.0f / 16129.0f);
    const bool vec_ok = (N % 8) == 0;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      __syncwarp();
      uint32_t acc[32];
      uint32_t oacc[32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + c;
      tmem_ld_32x32b_x32(taddr, acc);
      if (!OUT_I32 && count > 0) tmem_ld_32x32b_x32(taddr + BN, oacc);
      tmem_ld_wait();
      const int col0 = n0 + c;
      if (row >= M || col0 >= N) {
        // nothing of this row/column block lies inside Y
      } else if constexpr (OUT_I32) {
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
        for (int j = 0; j < 32; ++j) {
          const float cn = static_cast<float>(static_cast<int32_t>(acc[j])) * (rs * sw_tile[c + j]);
          y[j] = (count > 0) ? cn + __uint_as_float(oacc[j]) : cn;
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
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
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

template <int BN, int STAGES, bool OUT_I32>
cudaError_t launch(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<BN, STAGES>;
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
  auto kern = gemm_i8_mixed_kernel<BN, STAGES, OUT_I32>;
  static bool attr_set[64] = {};  // per instantiation and device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = (a.N + BN - 1) / BN;
  kern<<<m_tiles * n_tiles, kThreads, C::SMEM_BYTES, s>>>(
      maps[0], maps[1], maps[2], maps[3], a.x_scale, a.w_scale, OUT_I32 ? nullptr : a.n_outliers,
      a.out, a.M, a.N, a.K, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_mixed(const GemmArgs& a, cudaStream_t s) {
  return launch<256, 4, false>(a, s);
}

cudaError_t launch_gemm_i32(const GemmArgs& a, cudaStream_t s) {
  return launch<256, 4, true>(a, s);
}

}  // namespace i8mm

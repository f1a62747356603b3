// Group-scaled tensor-core GEMM of the W4A4 path after grouped Hadamard rotation
// ([Baidu] developer.baidu.com "分组旋转方法从W8A8到W4A4", sections 5.1 and 5.4):
//
//   Y[m][n] = fp16( sum_g C_g[m][n] * ax[m][g] * aw[n / G][g] / 7^2 )
//   C_g     = sum over the G columns k of group g of Xq[m][k] * Wq[n][k]   (INT32)
//
// ax: one absmax per (token, group of G columns); aw: one per G x G sub-block
// of the weight. sm_100a has no 4-bit integer MMA kind, so the 4-bit codes
// (held one per byte) run through tcgen05.mma kind::i8. Because the scales
// change every G columns of K, each group's INT32 product leaves TMEM and is
// folded into fp32 accumulators held in registers, while the tensor cores
// compute the next group into the other half of TMEM.
//
// The fold needs no integer-to-float conversion: before a buffer takes its
// group, every element is set to the bit pattern of 1.5 * 2^23 (0x4B400000)
// and all of the group's MMAs accumulate onto it. For |C_g| < 2^22 the INT32
// sum's bits read as the fp32 value 1.5 * 2^23 + C_g, so one exact fp32
// subtraction gives C_g, and one FMA adds C_g * ax * aw to the accumulator
// (both as paired f32x2 operations). The epilogue writes the constant back
// with tcgen05.st before it releases the buffer to the MMA warp.
//
// Persistent, one CTA per SM, 128 x 128 output tiles walked with stride
// gridDim.x (M-tile index fastest). The fold of every group is on the
// epilogue's critical path and its fixed cost (wait, fence, release) is paid
// per warp, so few warps with many columns each do it best: eight epilogue
// warps of 64 columns (64 fp32 accumulators and one group's 64 INT32 values
// per thread), in a CTA of ten warps that can give each thread ~200 registers.
// Warp roles:
//   warp 0      TMA producer: 128-byte-swizzled K-blocks (128 int8 columns of
//               Xq and Wq) into a 6-deep shared-memory ring
//   warp 1      owns the 512-column TMEM allocation (four 128-column buffers,
//               so the MMAs run up to three groups ahead of the fold) and
//               issues the MMAs (G/32 per group, K = 32 each)
//   warps 2-9   epilogue: warp w reads TMEM lane quarter (w % 4) and the 64
//               columns [64 p, 64 p + 64) of the tile, p = (w - 2) / 4
// Every mbarrier wait is bounded; a wait that gives up records
// I8MM_ERR_TIMEOUT in the status word and the CTA stops issuing work.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace i8mm {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NBUF = 4;                // TMEM accumulator buffers of BN columns
constexpr int KB = 128;                // int8 columns per K-block
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * KB;
constexpr int B_BYTES = BN * KB;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int BAR_BYTES = (2 * STAGES + 2 * NBUF) * 8 + 16;
constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kStatusTimeout = -5;     // == I8MM_ERR_TIMEOUT
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kMagicBits = 0x4B400000u;   // 1.5 * 2^23

__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_groups_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const float* __restrict__ x_absmax,   // [M][K/G]
                       const float* __restrict__ w_absmax,   // [N/G][K/G]
                       __half* __restrict__ Y, int M, int N, int K, int32_t* status) {
  constexpr int kPerGroup = G / 32;   // MMAs (K = 32) per group
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [NBUF]
  uint64_t* acc_free = acc_full + NBUF;  // [NBUF]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_free + NBUF);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int nk = K / KB;                 // K % G == 0 and G divides or is a multiple of KB
  const int ng = K / G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_free[b], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- producer
      uint32_t g = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * BM;
        const int n0 = (tile / m_tiles) * BN;
        for (int it = 0; it < nk; ++it, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            record_error(status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* a = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(a, &tmA, &full[s], it * KB, m0);
          tma_load_2d(a + A_BYTES, &tmB, &full[s], it * KB, n0);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (waits are warp-uniform through __all_sync)
    // and one elected lane issues each MMA and commit: a converged warp issues
    // MMAs faster than a lone lane of a diverged branch.
    constexpr uint32_t idesc = make_idesc(2 /*s32*/, 1 /*signed*/, BM, BN);
    uint32_t g = 0;    // K-blocks consumed (ring position)
    uint32_t u = 0;    // groups issued (buffer u % NBUF, its use u / NBUF)
    int mm = 0;        // MMAs issued into the current group
    uint32_t d = tmem;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok && !*abort_flag; tile += gridDim.x) {
      for (int it = 0; it < nk && ok; ++it, ++g) {
        const int s = g % STAGES;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (g / STAGES) & 1));
        if (!ok) break;
        const uint32_t a = smem_addr(smem + s * STAGE_BYTES);
        const uint32_t b = a + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (mm == 0) {
            // The buffer holds the 1.5 * 2^23 pattern again (written by the
            // epilogue after its previous group). The fence that orders those
            // stores before the MMAs stalls the issue for several hundred
            // cycles, so the buffers are claimed two groups at a time, with one
            // fence. (A claim past the last group waits for a release that
            // still comes: the epilogue frees every buffer it reads.)
            if ((u & 1) == 0) {
              ok = __all_sync(0xffffffffu,
                              mbar_wait(&acc_free[u % NBUF], (u / NBUF) & 1) &&
                                  mbar_wait(&acc_free[(u + 1) % NBUF], ((u + 1) / NBUF) & 1));
              if (!ok) break;
              tc_fence_after();
            }
            d = tmem + (u % NBUF) * BN;
          }
          mma_i8_elect(d, sw128_kmajor_desc(a + 32 * kk), sw128_kmajor_desc(b + 32 * kk), idesc,
                       1u);
          if (++mm == kPerGroup) {
            mma_commit_elect(&acc_full[u % NBUF]);
            mm = 0;
            ++u;
          }
        }
        if (!ok) break;
        mma_commit_elect(&empty[s]);
      }
    }
    if (!ok && lane == 0) {
      record_error(status, kStatusTimeout);
      *abort_flag = 1;
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    const int col_lo = part * 64;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    // Every buffer starts as the 1.5 * 2^23 pattern.
#pragma unroll
    for (int b = 0; b < NBUF; ++b)
#pragma unroll
      for (int c = 0; c < 64; c += 16)
        tmem_st_32x32b_x16_fill(lane_base + b * BN + col_lo + c, kMagicBits);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < NBUF; ++b) mbar_arrive(&acc_free[b]);
    }
    const uint64_t magic2 = f2pack(12582912.0f, 12582912.0f);
    uint32_t u = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * BM;
      const int n0 = (tile / m_tiles) * BN;
      const int row = m0 + q * 32 + lane;
      const int col0 = n0 + col_lo;
      const bool live_r = row < M;
      const bool live_c = col0 < N;          // N % 64 == 0: a warp's 64 columns are all in or out
      const int xoff = (live_r ? row : 0) * ng;            // < 2^31: M * K / G elements
      const int woff = (live_c ? col0 / G : 0) * ng;
      uint64_t acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0ull;
      float sx = live_r ? __ldg(x_absmax + xoff) : 0.0f;
      float sw = live_c ? __ldg(w_absmax + woff) : 0.0f;
      for (int gi = 0; gi < ng; ++gi, ++u) {
        const float sc = __fmul_rn(sx, sw);
        if (gi + 1 < ng) {                    // next group's scales, loaded under the wait
          sx = live_r ? __ldg(x_absmax + xoff + gi + 1) : 0.0f;
          sw = live_c ? __ldg(w_absmax + woff + gi + 1) : 0.0f;
        }
        const uint64_t sc2 = f2pack(sc, sc);
        const uint32_t buf = u % NBUF;
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (u / NBUF) & 1));
        if (!ok) {
          record_error(status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t base = lane_base + buf * BN + col_lo;
        uint32_t v[64];
        tmem_ld_32x32b_x32(base, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_32x32b_x32(base + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint64_t cg = sub2(static_cast<uint64_t>(v[2 * j]) |
                                       (static_cast<uint64_t>(v[2 * j + 1]) << 32),
                                   magic2);
          acc[j] = fma2(cg, sc2, acc[j]);
        }
#pragma unroll
        for (int c = 0; c < 64; c += 16) tmem_st_32x32b_x16_fill(base + c, kMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_free[buf]);
      }
      if (!ok) break;
      if (live_r && live_c) {
        constexpr float kInv49 = 1.0f / 49.0f;
        uint4* dst = reinterpret_cast<uint4*>(Y + static_cast<size_t>(row) * N + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t h[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint64_t p = acc[4 * j + i];
            const __half2 y2 = __floats2half2_rn(lo(p) * kInv49, hi(p) * kInv49);
            h[i] = *reinterpret_cast<const uint32_t*>(&y2);
          }
          dst[j] = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int sm_count_groups(int dev) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

template <int G>
cudaError_t launch_g(const int8_t* Xq, const int8_t* Wq, const float* xa, const float* wa,
                     __half* Y, int M, int N, int K, int32_t* status, cudaStream_t s) {
  CUtensorMap maps[2];
  std::memset(maps, 0, sizeof(maps));
  if (!make_tmap_sw128(&maps[0], Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, BM) ||
      !make_tmap_sw128(&maps[1], Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, BN))
    return cudaErrorInvalidValue;
  auto kern = gemm_groups_kernel<G>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int sms = sm_count_groups(dev);
  const int grid = tiles < sms ? tiles : sms;
  kern<<<grid, kThreads, SMEM_BYTES, s>>>(maps[0], maps[1], xa, wa, Y, M, N, K, status);
  return cudaGetLastError();
}

}  // namespace

// G in {64, 128, 256}; K % G == 0 and K % 128 == 0; N % G == 0.
cudaError_t launch_gemm_groups(const int8_t* Xq, const int8_t* Wq, const float* x_absmax,
                               const float* w_absmax, __half* Y, int M, int N, int K, int G,
                               int32_t* status, cudaStream_t s) {
  switch (G) {
    case 64: return launch_g<64>(Xq, Wq, x_absmax, w_absmax, Y, M, N, K, status, s);
    case 128: return launch_g<128>(Xq, Wq, x_absmax, w_absmax, Y, M, N, K, status, s);
    case 256: return launch_g<256>(Xq, Wq, x_absmax, w_absmax, Y, M, N, K, status, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace i8mm

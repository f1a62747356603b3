// Tensor-core GEMM of the LLM.int8() path on sm_100a (B200).
//
//   Y[i][n] = fp16( C_i32[i][n] * x_scale[i] * w_scale[n] / 127^2 + C_out[i][n] )
//   C_i32   = Xq . Wq^T          tcgen05.mma kind::i8, INT32 accumulator in TMEM
//   C_out   = X_O . W_O^T        the FP16 product over the outlier columns,
//                                tcgen05.mma kind::f16, FP32 accumulator in TMEM
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section:
// INT8 matmul accumulated in INT32, dequantisation by the outer product of the
// row and column scales, FP16 matmul over the outlier dimensions, final sum.
//
// Persistent kernel, one CTA per SM, output tiles walked with stride over the
// grid (M-tile index fastest, so the CTAs in flight share Wq column blocks and
// all of Xq through L2). With more than 128 rows the CTAs run as pairs (2-CTA
// clusters, tcgen05 cta_group::2) on 256 x 256 tiles, each CTA staging its 128
// rows of Xq and 128 of the 256 rows of Wq; otherwise one CTA takes a 128 x 256
// tile. Warp roles:
//   warp 0      TMA producer: 128-byte-swizzled K-blocks (128 int8 columns of
//               Xq and Wq) into a STAGES-deep shared-memory ring that runs
//               continuously across tiles
//   warp 1      owns the 512-column TMEM allocation; one lane issues the MMAs
//               (4 x K=32 per K-block) and commits
//   warps 2-17  epilogue: tcgen05.ld (thread = output row, four warps per TMEM
//               lane quarter splitting the 256 columns), dequantise, add the
//               outlier product, round to fp16, store
// The mode is chosen on the device from the outlier count:
//   count == 0  INT8 only; the two 256-column INT32 accumulators are
//               double-buffered, so the epilogue of one tile overlaps the MMAs
//               of the next.
//   count >  0  the compacted fp16 panels X_O, W_O (64-column blocks) are
//               streamed through the same ring after the int8 K-blocks and
//               multiplied with kind::f16 into an FP32 accumulator in the other
//               half of TMEM (single-buffered). Measured on B200 with 6-7
//               outlier columns, this beat forming the outlier product on CUDA
//               cores in a double-buffered epilogue (OPT-6.7B FFN-up GEMM
//               101 against 108 us): the CUDA-core work and its gathers slowed
//               the main loop more than the lost overlap costs.
// The outlier count is read from device memory, so the host never syncs.
// No TMA load uses cluster multicast: both CTAs of a pair load their own halves,
// completing on the even CTA's barrier. Every mbarrier wait is bounded;
// a wait that gives up records I8MM_ERR_TIMEOUT in the status word and the
// CTA stops issuing work.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8mm {

namespace {

constexpr int BM = 128;              // output rows per CTA (TMEM lanes)
constexpr int BN = 256;              // columns of the output tile
constexpr int KB_I8 = 128;           // int8 columns per K-block (128 bytes)
constexpr int KB_F16 = 64;           // fp16 columns per panel block (128 bytes)
constexpr int kEpiWarps = 16;          // four per TMEM lane quarter, 64 columns each
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kStatusTimeout = -5;   // == I8MM_ERR_TIMEOUT
constexpr uint32_t TMEM_COLS = 512;

// PAIR: a CTA pair (cta_group::2) computes a 256 x 256 tile; each CTA stages its
// 128 rows of A and 128 of the 256 rows of B, so a stage is 32 KB; five fit next
// to the output staging buffers. Single CTA: 128 x 256 tiles, 48 KB stages, three.
// Output staging: two 1 KB buffers per epilogue warp (32 rows x 16 fp16 columns,
// 32-byte swizzle) drained by TMA stores.
constexpr int STG_BUF_BYTES = 32 * 16 * 2;

template <bool PAIR>
struct Cfg {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;
  static constexpr int STAGES = PAIR ? 5 : 3;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int STG_BYTES = kEpiWarps * 2 * STG_BUF_BYTES;
  static constexpr int SW_BYTES = BN * 4;            // w_scale tile
  static constexpr int ZS_BYTES = BN * 4;            // weight row sums (zero-point mode)
  static constexpr int BAR_OFF = RING_BYTES + STG_BYTES + SW_BYTES + ZS_BYTES;
  static constexpr int BAR_BYTES = (2 * STAGES + 4) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + BAR_OFF + BAR_BYTES;
};

__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
}

// 18 warps: two of the four SM sub-partitions hold five warps, so the register
// budget is 96 per thread (16K registers per sub-partition).
// ZP: the activation codes carry a per-token zero point z (scholia section 6);
// the epilogue forms (C - z * sum_k Wq[n, k]) * step * w_scale / 127.
template <bool OUT_I32, bool PAIR, bool ZP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_persistent_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB,
                              const __grid_constant__ CUtensorMap tmXO,
                              const __grid_constant__ CUtensorMap tmWO,
                              const __grid_constant__ CUtensorMap tmY, int y_tma,
                              const float* __restrict__ x_scale,
                              const float* __restrict__ w_scale,
                              const int32_t* __restrict__ x_zero,
                              const int32_t* __restrict__ w_rowsum,
                              const int32_t* __restrict__ n_outliers, void* __restrict__ out,
                              int M, int N, int K, int32_t* status) {
  using C = Cfg<PAIR>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (swizzle atoms). Derived by an offset from the
  // shared array, not through an integer cast, so every pointer below stays in
  // the shared state space and compiles to shared-memory loads and stores.
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* stg = smem + C::RING_BYTES;                                          // staging
  float* sw_s = reinterpret_cast<float*>(stg + C::STG_BYTES);                  // [BN]
  int32_t* zs_s = reinterpret_cast<int32_t*>(stg + C::STG_BYTES + C::SW_BYTES);  // [BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // A pair walks the tiles as one unit; rank 0 of the pair issues the MMAs.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int m_tiles = (M + C::TILE_M - 1) / C::TILE_M;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], (PAIR ? 2 : 1) * kEpiWarps);   // epilogue warps of the pair
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
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // barriers and TMEM of both CTAs are ready
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Set-up above overlaps the tail of the previous kernel (the quantisation
  // kernel); nothing it writes is read before this point.
  griddep_launch_dependents();
  griddep_wait();

  const int count = (!OUT_I32 && n_outliers) ? *n_outliers : 0;
  const bool tc_out = count > 0;               // outlier product on the tensor cores
  // With every column an outlier (threshold 0 on data without zeros) all INT8
  // codes and row scales are 0: the INT8 K-blocks are skipped and the epilogue
  // takes C_i32 as 0.
  const bool no_i8 = !OUT_I32 && count >= K;
  const int nk = no_i8 ? 0 : (K + KB_I8 - 1) / KB_I8;
  const int np = tc_out ? (count + KB_F16 - 1) / KB_F16 : 0;
  const int iters = nk + np;


  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t g = 0;
      for (int tile = unit; tile < num_tiles && !*abort_flag; tile += units) {
        const int m0 = (tile % m_tiles) * C::TILE_M + static_cast<int>(rank) * BM;
        const int n0 = (tile / m_tiles) * BN + static_cast<int>(rank) * C::B_ROWS;
        for (int it = 0; it < iters; ++it, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            record_error(status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* a = smem + s * C::STAGE_BYTES;
          uint8_t* b = a + C::A_BYTES;
          const bool panel = it >= nk;
          const CUtensorMap* ta = panel ? &tmXO : &tmA;
          const CUtensorMap* tb = panel ? &tmWO : &tmB;
          const int x = panel ? (it - nk) * KB_F16 : it * KB_I8;
          if constexpr (PAIR) {
            // Both CTAs' loads complete on the full barrier of rank 0, which waits
            // for the bytes of the whole pair.
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
            const uint32_t bar0 = cluster_addr(&full[s], 0);
            tma_load_2d_pair(a, ta, bar0, x, m0);
            tma_load_2d_pair(b, tb, bar0, x, n0);
          } else {
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
            tma_load_2d(a, ta, &full[s], x, m0);
            tma_load_2d(b, tb, &full[s], x, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_i8 = make_idesc(2 /*s32*/, 1 /*signed*/, C::TILE_M, BN);
      constexpr uint32_t idesc_f16 = make_idesc(1 /*f32*/, 0 /*fp16*/, C::TILE_M, BN);
      uint32_t g = 0;
      int local = 0;
      for (int tile = unit; tile < num_tiles && !*abort_flag; tile += units, ++local) {
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
          // The stage was written by TMA and is ordered by its mbarrier alone;
          // a tcgen05 fence here would stall the issue of every stage.
          const uint32_t a = smem_addr(smem + s * C::STAGE_BYTES);
          const uint32_t b = a + C::A_BYTES;
          if (it < nk) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(a + 32 * kk);
              const uint64_t bd = sw128_kmajor_desc(b + 32 * kk);
              if constexpr (PAIR)
                mma_i8_pair(d_i32, ad, bd, idesc_i8, (it | kk) != 0);
              else
                mma_i8(d_i32, ad, bd, idesc_i8, (it | kk) != 0);
            }
          } else {
            const int p = it - nk;
            const int steps = min(4, (count - p * KB_F16 + 15) / 16);
            for (int kk = 0; kk < steps; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(a + 32 * kk);
              const uint64_t bd = sw128_kmajor_desc(b + 32 * kk);
              if constexpr (PAIR)
                mma_f16_pair(d_f32, ad, bd, idesc_f16, (p | kk) != 0);
              else
                mma_f16(d_f32, ad, bd, idesc_f16, (p | kk) != 0);
            }
          }
          if constexpr (PAIR)
            mma_commit_pair(&empty[s], 0x3);
          else
            mma_commit(&empty[s]);
        }
        if constexpr (PAIR)
          mma_commit_pair(&acc_full[buf], 0x3);
        else
          mma_commit(&acc_full[buf]);
        if (!ok) break;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Warp w reads TMEM lane quarter (w % 4) and the 64 columns [part*64, part*64+64)
    // of the tile. The per-tile scales of the epilogue are fetched one tile ahead
    // into registers; the column scales are staged in shared memory.
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    const int et = threadIdx.x - 64;        // 0 .. 32*kEpiWarps-1
    const bool vec_ok = (N % 8) == 0;
    const int col_lo = part * (BN / 4);

    float sw_next = 0.0f;
    int32_t ws_next = 0, zr_next = 0;
    float rs_next = 0.0f;
    auto prefetch = [&](int tile) {
      if (OUT_I32 || tile >= num_tiles) return;
      const int m0 = (tile % m_tiles) * C::TILE_M + static_cast<int>(rank) * BM;
      const int n0 = (tile / m_tiles) * BN;
      const int row = m0 + q * 32 + lane;
      // absmax codes: x_absmax * w_absmax / 127^2; zero-point codes: step * w_absmax / 127
      rs_next = (row < M) ? x_scale[row] * (ZP ? (1.0f / 127.0f) : (1.0f / 16129.0f)) : 0.0f;
      if constexpr (ZP) zr_next = (row < M) ? x_zero[row] : 0;
      if (et < BN) {
        const int n = n0 + et;
        sw_next = (n < N) ? w_scale[n] : 0.0f;
        if constexpr (ZP) ws_next = (n < N) ? w_rowsum[n] : 0;
      }
    };
    prefetch(unit);

    int local = 0;
    uint32_t sc = 0;   // chunks stored by this warp (selects the staging buffer)
    for (int tile = unit; tile < num_tiles; tile += units, ++local) {
      const int m0 = (tile % m_tiles) * C::TILE_M + static_cast<int>(rank) * BM;
      const int n0 = (tile / m_tiles) * BN;
      const int buf = tc_out ? 0 : (local & 1);
      const uint32_t aph = tc_out ? (local & 1) : ((local >> 1) & 1);
      const int row = m0 + q * 32 + lane;

      // Stage this tile's column scales in shared memory; the row scale stays in a register.
      const float rs = rs_next;
      const int32_t zr = zr_next;
      if (!OUT_I32 && et < BN) {
        sw_s[et] = sw_next;
        if constexpr (ZP) zs_s[et] = ws_next;
      }
      epi_sync();

      // Warp-uniform, so that a timed-out wait can never split the warp before
      // the warp-collective TMEM loads below.
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], aph));
      if (!ok) {
        record_error(status, kStatusTimeout);
        *abort_flag = 1;
      }
      tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      // The chunk loop is instantiated separately for the two outlier modes so that
      // each keeps only its own registers live.
      auto chunks = [&](auto tc_tag) {
        constexpr bool TC = decltype(tc_tag)::value;
#pragma unroll 1
        for (int c = col_lo; c < col_lo + BN / 4 && ok; c += 16, ++sc) {
          if (!OUT_I32 && y_tma) {
            // The staging buffer of this chunk was last drained two stores ago.
            if (lane == 0) bulk_wait_group_read<1>();
          }
          __syncwarp();
          // tcgen05.ld is warp-collective: issued by all 32 lanes, outside any
          // per-row condition (tc_out and ok are uniform across the warp).
          uint32_t acc[16];
          uint32_t oacc[TC ? 16 : 1];
          if (!no_i8) {
            tmem_ld_32x32b_x16(lane_base + buf * BN + c, acc);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0u;
          }
          if constexpr (TC) tmem_ld_32x32b_x16(lane_base + BN + c, oacc);
          tmem_ld_wait();
          const int col0 = n0 + c;
          if (row < M && col0 < N) {
            if constexpr (OUT_I32) {
              int32_t* orow = reinterpret_cast<int32_t*>(out) + static_cast<size_t>(row) * N;
              if (vec_ok && col0 + 16 <= N) {
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                  *reinterpret_cast<uint4*>(orow + col0 + j) =
                      make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  if (col0 + j < N) orow[col0 + j] = static_cast<int32_t>(acc[j]);
              }
            } else {
              float y[16];
              const float4* sw4 = reinterpret_cast<const float4*>(sw_s + c);
              if constexpr (ZP) {
                // C - z * sum_k Wq[n, k], exact in int32 (|.| <= 2 * 128 * 127 * K)
                const int4* zs4 = reinterpret_cast<const int4*>(zs_s + c);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const int4 zw = zs4[j];
                  acc[4 * j + 0] = static_cast<uint32_t>(static_cast<int32_t>(acc[4 * j + 0]) - zr * zw.x);
                  acc[4 * j + 1] = static_cast<uint32_t>(static_cast<int32_t>(acc[4 * j + 1]) - zr * zw.y);
                  acc[4 * j + 2] = static_cast<uint32_t>(static_cast<int32_t>(acc[4 * j + 2]) - zr * zw.z);
                  acc[4 * j + 3] = static_cast<uint32_t>(static_cast<int32_t>(acc[4 * j + 3]) - zr * zw.w);
                }
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 w = sw4[j];
                y[4 * j + 0] = static_cast<float>(static_cast<int32_t>(acc[4 * j + 0])) * (rs * w.x);
                y[4 * j + 1] = static_cast<float>(static_cast<int32_t>(acc[4 * j + 1])) * (rs * w.y);
                y[4 * j + 2] = static_cast<float>(static_cast<int32_t>(acc[4 * j + 2])) * (rs * w.z);
                y[4 * j + 3] = static_cast<float>(static_cast<int32_t>(acc[4 * j + 3])) * (rs * w.w);
              }
              if constexpr (TC) {
#pragma unroll
                for (int j = 0; j < 16; ++j) y[j] += __uint_as_float(oacc[j]);
              }
              __half* orow = reinterpret_cast<__half*>(out) + static_cast<size_t>(row) * N;
              if (y_tma) {
                // Row `lane` of this warp's 32 x 16 staging block, 16-byte chunks
                // XOR-swizzled by bit 2 of the row (the TMA 32-byte swizzle).
                uint8_t* buf_row = stg + ((warp - 2) * 2 + (sc & 1)) * STG_BUF_BYTES + lane * 32;
                const int sw = (lane >> 2) & 1;
#pragma unroll
                for (int j = 0; j < 16; j += 8) {
                  uint4 v;
                  __half2* h = reinterpret_cast<__half2*>(&v);
                  h[0] = __floats2half2_rn(y[j], y[j + 1]);
                  h[1] = __floats2half2_rn(y[j + 2], y[j + 3]);
                  h[2] = __floats2half2_rn(y[j + 4], y[j + 5]);
                  h[3] = __floats2half2_rn(y[j + 6], y[j + 7]);
                  *reinterpret_cast<uint4*>(buf_row + (((j >> 3) ^ sw) << 4)) = v;
                }
              } else if (vec_ok && col0 + 16 <= N) {
#pragma unroll
                for (int j = 0; j < 16; j += 8) {
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
                for (int j = 0; j < 16; ++j)
                  if (col0 + j < N) orow[col0 + j] = __float2half_rn(y[j]);
              }
            }
          }
          if (!OUT_I32 && y_tma) {
            // Rows >= M are staged too (as anything) and clipped by the TMA store.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && col0 < N) {
              tma_store_2d(&tmY, stg + ((warp - 2) * 2 + (sc & 1)) * STG_BUF_BYTES, col0,
                           m0 + q * 32);
              bulk_commit_group();
            }
          }
        }
      };
      if (tc_out)
        chunks(std::true_type{});
      else
        chunks(std::false_type{});
      // The next tile's operands: issued now, so that their registers are not
      // live during the chunk loop; the wait for the next accumulator covers
      // their latency.
      prefetch(tile + units);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(cluster_addr(&acc_empty[buf], 0));
        else
          mbar_arrive(&acc_empty[buf]);
      }
      epi_sync();   // the tile's sw_s / zs_s are no longer read
      if (!ok || *abort_flag) break;
    }
    if (!OUT_I32 && y_tma && lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the peer may still read our shared memory
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, TMEM_COLS);
    else
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

// Row-major [rows][cols] matrix, box of box_rows x box_bytes (one swizzle span).
bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
               uint64_t cols, uint64_t rows, uint32_t box_rows, uint32_t box_bytes = 128,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes / elem_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count(int dev) {
  static int cached[64] = {};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2) n = 2;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

template <bool OUT_I32, bool PAIR, bool ZP>
cudaError_t launch(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<PAIR>;
  CUtensorMap maps[5];
  std::memset(maps, 0, sizeof(maps));
  if (!make_tmap(&maps[0], a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.M, BM) ||
      !make_tmap(&maps[1], a.Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.N, C::B_ROWS))
    return cudaErrorInvalidValue;
  if (!OUT_I32 && a.X_O && a.W_O) {
    if (!make_tmap(&maps[2], a.X_O, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.ld, a.M, BM) ||
        !make_tmap(&maps[3], a.W_O, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.ld, a.N, C::B_ROWS))
      return cudaErrorInvalidValue;
  } else {
    maps[2] = maps[0];
    maps[3] = maps[1];
  }
  // fp16 Y leaves through TMA stores when its row stride allows (N % 8 == 0).
  int y_tma = 0;
  if (!OUT_I32 && a.N % 8 == 0 &&
      make_tmap(&maps[4], a.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.M, 32, 32,
                CU_TENSOR_MAP_SWIZZLE_32B))
    y_tma = 1;
  if (!y_tma) maps[4] = maps[0];
  auto kern = gemm_i8_persistent_kernel<OUT_I32, PAIR, ZP>;
  static bool attr_set[64] = {};  // per instantiation and device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const int sms = sm_count(dev);
  const int m_tiles = (a.M + C::TILE_M - 1) / C::TILE_M;
  const int n_tiles = (a.N + BN - 1) / BN;
  const int tiles = m_tiles * n_tiles;
  const int max_units = PAIR ? sms / 2 : sms;
  const int units = tiles < max_units ? tiles : max_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(PAIR ? 2 * units : units);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (PAIR) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], y_tma,
                         a.x_scale, a.w_scale, a.x_zero, a.w_rowsum,
                         OUT_I32 ? nullptr : a.n_outliers, a.out, a.M, a.N, a.K, a.status);
  if (e != cudaSuccess) (void)cudaGetLastError();   // do not leave it for the next launch
  return e;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint32_t box_rows, uint32_t box_bytes,
                  CUtensorMapSwizzle swz) {
  return make_tmap(m, base, dt, elem_bytes, cols, rows, box_rows, box_bytes, swz);
}

// CTA pairs whenever there is more than one 128-row block of output rows.
cudaError_t launch_gemm_mixed(const GemmArgs& a, cudaStream_t s) {
  if (a.x_zero && a.w_rowsum)
    return a.M > BM ? launch<false, true, true>(a, s) : launch<false, false, true>(a, s);
  return a.M > BM ? launch<false, true, false>(a, s) : launch<false, false, false>(a, s);
}

cudaError_t launch_gemm_i32(const GemmArgs& a, cudaStream_t s) {
  return a.M > BM ? launch<true, true, false>(a, s) : launch<true, false, false>(a, s);
}

}  // namespace i8mm

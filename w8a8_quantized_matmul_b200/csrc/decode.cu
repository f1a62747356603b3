// Decode-shape path (M <= 16 tokens) of the LLM.int8() matmul, one launch.
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier detection by threshold, vector-wise absmax INT8 quantisation of the
// rest, INT8 matmul with INT32 accumulation, dequantisation by the outer product
// of the scales, FP16 product over the outlier columns, final sum); tanjunchen
// "quantization explained part 2" section 1.2 (threshold 6.0).
//
// With at most 16 tokens the work is bound by reading Wq once. The grid is
// made of clusters of S CTAs; a cluster owns 128 output features (rows of Wq)
// and its CTAs split K, so every CTA streams a 128 x (K/S) slice of Wq:
//   * the producer TMA-loads the whole slice at kernel start (up to 8 stages of
//     128 x 128 bytes, no reuse), before anything else;
//   * all threads bulk-copy the CTA's K-range of every token row of X into
//     shared memory. Every CTA sees all tokens, so the outlier flags of its
//     columns are exact locally; each computes per-token maxima over its
//     non-outlier columns and the cluster exchanges them through distributed
//     shared memory to form each token's absmax;
//   * the CTA writes the INT8 codes of its X range straight into the 128-byte
//     swizzled K-major layout the tensor core reads (16 token rows) and one
//     thread issues tcgen05.mma kind::i8 with M = 128 weight rows, N = 16 tokens;
//   * the outlier product of the CTA's own outlier columns is formed on CUDA
//     cores (fp16 products are exact in fp32);
//   * INT32 partials (exact, order free) and fp32 outlier partials are summed
//     across the cluster in a fixed rank order through distributed shared
//     memory; each CTA finishes 128/S rows and writes Y.
// Cluster 0 also writes the intermediates the workspace documents (bitmap,
// count, ascending outlier list, x_scale, Xq). No TMA multicast is used.
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

constexpr int kRows = 128;       // Wq rows (output features) per cluster
constexpr int kKB = 128;         // int8 columns per K-block
constexpr int kMaxBlocks = 8;    // K-blocks per CTA (all in flight at once)
constexpr int kTok = 16;         // MMA N: tokens, zero-padded
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCluster = 8;
constexpr int kStatusTimeout = -5;

struct DecodeSmem {
  static constexpr int RING = 0;                                   // [8][128][128] i8
  static constexpr int BOP = RING + kMaxBlocks * kRows * kKB;      // [8][16][128] i8
  static constexpr int XS = BOP + kMaxBlocks * kTok * kKB;         // [16][1024] f16
  static constexpr int PI = XS + kTok * kMaxBlocks * kKB * 2;      // [128][16] i32
  static constexpr int PF = PI + kRows * kTok * 4;                 // [128][16] f32
  static constexpr int XMAX = PF + kRows * kTok * 4;               // [8 ranks][16] f32
  static constexpr int XCNT = XMAX + kMaxCluster * kTok * 4;       // [8 ranks] i32
  static constexpr int BITS = XCNT + kMaxCluster * 4;              // [32] u32
  static constexpr int LIDX = BITS + 32 * 4;                       // [1024] u16
  static constexpr int RED = LIDX + kMaxBlocks * kKB * 2;          // [8 warps][16] f32
  static constexpr int AMAX = RED + kWarps * kTok * 4;             // [16] f32
  static constexpr int MISC = AMAX + kTok * 4;                     // [4] i32
  static constexpr int BARS = MISC + 16;                           // full[8], done, xbar
  static constexpr int TSLOT = BARS + (kMaxBlocks + 2) * 8;
  static constexpr int TOTAL = TSLOT + 16;
  static constexpr int BYTES = TOTAL + 1024;                       // alignment slack
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_s32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmWq, DecodeArgs a) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  using L = DecodeSmem;
  uint8_t* ring = sm + L::RING;
  uint8_t* bop = sm + L::BOP;
  __half* xs = reinterpret_cast<__half*>(sm + L::XS);
  int32_t* p_i32 = reinterpret_cast<int32_t*>(sm + L::PI);
  float* p_f32 = reinterpret_cast<float*>(sm + L::PF);
  float* xmax = reinterpret_cast<float*>(sm + L::XMAX);
  int32_t* xcnt = reinterpret_cast<int32_t*>(sm + L::XCNT);
  uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L::BITS);
  uint16_t* lidx = reinterpret_cast<uint16_t*>(sm + L::LIDX);
  float* red = reinterpret_cast<float*>(sm + L::RED);
  float* amax = reinterpret_cast<float*>(sm + L::AMAX);
  int32_t* misc = reinterpret_cast<int32_t*>(sm + L::MISC);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::BARS);
  uint64_t* done = full + kMaxBlocks;
  uint64_t* xbar = done + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::TSLOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int tile = blockIdx.x / S;
  const int n0 = tile * kRows;
  const int M = a.M, N = a.N, K = a.K;
  const int nkb = (K + kKB - 1) / kKB;
  const int bper = (nkb + S - 1) / S;
  const int kb0 = min(nkb, rank * bper);
  const int nb = min(nkb, kb0 + bper) - kb0;            // K-blocks of this CTA (0..8)
  const int k0 = min(K, kb0 * kKB);
  const int k1 = min(K, (kb0 + nb) * kKB);
  const int kw = k1 - k0;                               // columns of this CTA
  const bool writer = (tile == 0);                      // cluster 0 writes intermediates

  if (tid == 0) {
    for (int b = 0; b < kMaxBlocks; ++b) mbar_init(&full[b], 1);
    mbar_init(done, 1);
    mbar_init(xbar, 1);
    fence_mbarrier_init();
    tma_prefetch_desc(&tmWq);
    if (blockIdx.x == 0 && a.status) *a.status = 0;
  }
  if (warp == 1) {
    tmem_alloc(tslot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // every CTA's barriers and buffers exist before any remote access
  const uint32_t tmem = *tslot;

  // ---- weight stream first: the whole slice is requested at once
  if (warp == 0 && lane == 0) {
    for (int b = 0; b < nb; ++b) {
      mbar_arrive_expect_tx(&full[b], kRows * kKB);
      tma_load_2d(ring + b * kRows * kKB, &tmWq, &full[b], (kb0 + b) * kKB, n0);
    }
  }
  // ---- this CTA's K-range of every token row of X
  bool ok = true;
  if (kw > 0) {
    if (tid == 0) {
      mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(M * kw * 2));
      for (int t = 0; t < M; ++t)
        bulk_load(xs + t * kw, a.X + static_cast<size_t>(t) * K + k0,
                  static_cast<uint32_t>(kw * 2), xbar);
    }
    if (!mbar_wait(xbar, 0)) ok = false;
  }

  // ---- outlier flags of the CTA's columns (exact: every token is here) and
  //      per-token maxima over its non-outlier columns
  const int nvec = kw >> 3;                              // 16-byte vectors per row
  float part[kTok];
#pragma unroll
  for (int t = 0; t < kTok; ++t) part[t] = 0.0f;
  if (tid < 128) {                                       // 128 vectors cover 1024 columns
    const int v = tid;
    uint32_t m8 = 0;
    if (v < nvec) {
      float cm[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cm[i] = 0.0f;
      for (int t = 0; t < M; ++t) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(xs + t * kw + v * 8), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) cm[i] = fmaxf(cm[i], fabsf(f[i]));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) m8 |= (cm[i] > a.threshold ? 1u : 0u) << i;
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
        if (t < M) {
          float f[8];
          unpack8(*reinterpret_cast<const uint4*>(xs + t * kw + v * 8), f);
          float pm = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (!((m8 >> i) & 1u)) pm = fmaxf(pm, fabsf(f[i]));
          part[t] = pm;
        }
      }
    }
    uint32_t word = m8 << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if ((lane & 3) == 0) bits[v >> 2] = (v < nvec) ? word : 0u;
  }
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    const float m = warp_max(part[t]);
    if (lane == 0) red[warp * kTok + t] = m;
  }
  __syncthreads();
  if (tid < kTok) {
    float m = 0.0f;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w * kTok + tid]);
    // Publish to every CTA of the cluster (slot = this CTA's rank).
    for (int r = 0; r < S; ++r)
      st_cluster_f32(cluster_addr(&xmax[rank * kTok + tid], r), m);
  }
  // Local outlier list in ascending order (one warp, 32 bitmap words at most).
  if (warp == 0) {
    const int words = (kw + 31) >> 5;
    const uint32_t bw = (lane < words) ? bits[lane] : 0u;
    const int c = __popc(bw);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    uint32_t b = bw;
    int p = incl - c;
    while (b) {
      const int j = __ffs(b) - 1;
      b &= b - 1;
      lidx[p++] = static_cast<uint16_t>(lane * 32 + j);
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
      misc[0] = total;
      for (int r = 0; r < S; ++r) st_cluster_s32(cluster_addr(&xcnt[rank], r), total);
    }
  }
  __syncthreads();
  cluster_sync();   // maxima and counts of every rank have arrived

  // ---- token absmax, global outlier positions, intermediates (cluster 0)
  const int lcount = misc[0];
  int prefix = 0, total = 0;
  for (int r = 0; r < S; ++r) {
    const int c = xcnt[r];
    if (r < rank) prefix += c;
    total += c;
  }
  if (tid < kTok) {
    float m = 0.0f;
    for (int r = 0; r < S; ++r) m = fmaxf(m, xmax[r * kTok + tid]);
    amax[tid] = m;
    if (writer && rank == 0 && tid < M) a.x_scale[tid] = m;
  }
  if (writer) {
    for (int w = tid; w < ((kw + 31) >> 5); w += kThreads) a.bitmap[(k0 >> 5) + w] = bits[w];
    for (int i = tid; i < lcount; i += kThreads) a.col_idx[prefix + i] = k0 + lidx[i];
    if (rank == 0 && tid == 0) *a.n_outliers = total;
  }
  __syncthreads();

  // ---- INT8 codes of the X range into the swizzled K-major B operand (16 rows)
  //      and, in cluster 0, into Xq
  for (int e = tid; e < kTok * nb * 8; e += kThreads) {
    const int t = e / (nb * 8);
    const int c = e - t * (nb * 8);                      // 16-byte chunk along K
    const int b = c >> 3, cc = c & 7;
    uint4 q = make_uint4(0, 0, 0, 0);
    const int kc = c * 16;                                // first column of the chunk
    if (t < M && kc < kw) {
      const float am = amax[t];
      const float inv = quant_inv(am);
      const uint32_t wbits = bits[kc >> 5] >> (kc & 31);  // 16 flag bits of the chunk
      uint32_t* qw = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(xs + t * kw + kc + h * 8), f);
        int code[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          code[i] = ((wbits >> (h * 8 + i)) & 1u) ? 0 : quant_code_fast(f[i], am, inv);
        qw[2 * h] = pack4(code[0], code[1], code[2], code[3]);
        qw[2 * h + 1] = pack4(code[4], code[5], code[6], code[7]);
      }
      if (writer)
        *reinterpret_cast<uint4*>(a.Xq + static_cast<size_t>(t) * K + k0 + kc) = q;
    }
    uint8_t* dst = bop + b * (kTok * kKB) + (t >> 3) * 1024 + (t & 7) * 128 + ((cc ^ (t & 7)) << 4);
    *reinterpret_cast<uint4*>(dst) = q;
  }
  fence_proxy_async_smem();   // generic writes above are read by the tensor core
  __syncthreads();

  // ---- MMA: D[128 weight rows][16 tokens] += Wq_slice . Xq_range^T
  if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = make_idesc(2 /*s32*/, 1 /*signed*/, kRows, kTok);
    for (int b = 0; b < nb; ++b) {
      if (!mbar_wait(&full[b], 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ad = smem_addr(ring + b * kRows * kKB);
      const uint32_t bd = smem_addr(bop + b * kTok * kKB);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_i8(tmem, sw128_kmajor_desc(ad + 32 * kk), sw128_kmajor_desc(bd + 32 * kk), idesc,
               (b | kk) != 0);
    }
    mma_commit(done);
  }

  // ---- fp32 outlier partials of this CTA's outlier columns (CUDA cores)
  if (tid < kRows) {
    float o[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) o[t] = 0.0f;
    const int n = n0 + tid;
    if (n < N) {
      const __half* wrow = a.W + static_cast<size_t>(n) * K + k0;
      for (int i = 0; i < lcount; ++i) {
        const int j = lidx[i];
        const float w = __half2float(wrow[j]);
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t < M) o[t] = fmaf(__half2float(xs[t * kw + j]), w, o[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < kTok; ++t) p_f32[tid * kTok + t] = o[t];
  }

  // ---- INT32 partials from TMEM (warps 4..7: lane quarters 0..3)
  if (warp >= 4) {
    const int q = warp & 3;
    uint32_t acc[16];
    bool got = true;
    if (nb > 0) got = __all_sync(0xffffffffu, mbar_wait(done, 0));
    if (nb > 0 && got) {
      tc_fence_after();
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16), acc);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) acc[t] = 0u;
    }
    if (!got) ok = false;
    const int r = q * 32 + lane;
#pragma unroll
    for (int t = 0; t < kTok; ++t) p_i32[r * kTok + t] = static_cast<int32_t>(acc[t]);
  }
  if (!ok && a.status) atomicExch(a.status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // every rank's partials are complete

  // ---- sum the partials of all ranks (fixed order) for this CTA's share of rows
  const int rpr = (kRows + S - 1) / S;
  for (int e = tid; e < rpr * kTok; e += kThreads) {
    const int t = e / rpr;
    const int rl = rank * rpr + (e - t * rpr);
    const int n = n0 + rl;
    if (t < M && rl < kRows && n < N) {
      int32_t c = 0;
      float o = 0.0f;
      for (int r = 0; r < S; ++r) {
        c += ld_cluster_s32(cluster_addr(&p_i32[rl * kTok + t], r));
        o += ld_cluster_f32(cluster_addr(&p_f32[rl * kTok + t], r));
      }
      const float rs = amax[t] * (1.0f / 16129.0f);
      const float y = static_cast<float>(c) * (rs * a.w_scale[n]) + o;
      a.Y[static_cast<size_t>(t) * N + n] = __float2half_rn(y);
    }
  }
  __syncthreads();
  cluster_sync();   // no CTA leaves while a peer may still read its partials
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

}  // namespace

bool decode_supported(int M, int K) { return M >= 1 && M <= kTok && K <= kMaxCluster * kMaxBlocks * kKB; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  CUtensorMap tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!make_tmap_sw128(&tm, a.Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.N, kRows))
    return cudaErrorInvalidValue;
  const int nkb = (a.K + kKB - 1) / kKB;
  int S = (nkb + kMaxBlocks - 1) / kMaxBlocks;          // CTAs per cluster
  if (S < 1) S = 1;
  if (S > kMaxCluster) return cudaErrorInvalidValue;
  const int tiles = (a.N + kRows - 1) / kRows;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecodeSmem::BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = DecodeSmem::BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  DecodeArgs args = a;
  e = cudaLaunchKernelEx(&cfg, decode_kernel, tm, args);
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

}  // namespace i8mm

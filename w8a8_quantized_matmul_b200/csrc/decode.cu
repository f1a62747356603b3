// Decode-shape path (M <= 16 tokens) of the LLM.int8() matmul, one launch.
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier detection by threshold, vector-wise absmax INT8 quantisation of the
// rest, INT8 matmul with INT32 accumulation, dequantisation by the outer product
// of the scales, FP16 product over the outlier columns, final sum); tanjunchen
// "quantization explained part 2" section 1.2 (threshold 6.0).
//
// With at most 16 tokens the work is bound by reading Wq once; everything else
// is arranged to finish while that stream is in flight. The grid is made of
// clusters of S CTAs; a cluster owns 128 output features (rows of Wq) and its
// CTAs split K, so every CTA reads a 128 x (K/S) slice of Wq (at most 8 blocks
// of 128 x 128 bytes, all requested at kernel start).
//
// Warp roles (320 threads):
//   warp 0     producer: bulk-copies the CTA's K-range of every token row of X
//              (first, it is small and L2-resident), then TMA-loads the Wq slice
//   warp 1     TMEM allocator and MMA issuer: tcgen05.mma kind::i8 with
//              M = 128 weight rows, N = 16 tokens, one K-block as it lands
//   warps 2-9  X workers, 4 columns per thread, all 16 tokens held in registers:
//              exact outlier flags of their columns (every token is here),
//              per-token maxima over the non-outlier columns, and after the
//              cluster exchange of those maxima the INT8 codes, written straight
//              into the 128-byte-swizzled K-major B operand of the MMA
//   warps 4-7  also the epilogue: the fp32 outlier partials of the CTA's own
//              outlier columns on CUDA cores (fp16 products are exact in fp32),
//              the INT32 partials from TMEM, and the cross-CTA sum.
//
// Cross-CTA traffic uses st.async into the peer's shared memory, counted in
// bytes on the peer's mbarrier: one 80-byte message per CTA pair with the
// per-token maxima and the outlier count, then each CTA pushes every row's
// 16 INT32 + 16 fp32 partials to the CTA that finishes that row, which sums the
// S partials in rank order and writes Y. A split cluster barrier only publishes
// the mbarrier initialisation and keeps every CTA alive until its peers have
// issued their last store into it. Cluster 0 also writes the intermediates the
// workspace documents (bitmap, count, ascending outlier list, x_scale, Xq).
// No TMA multicast is used.
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

constexpr int kRows = 128;                    // Wq rows (output features) per cluster = MMA M
constexpr int kKB = 128;                      // int8 columns per K-block (one swizzle row)
constexpr int kMaxBlocks = 8;                 // K-blocks per CTA, all in flight at once
constexpr int kCols = kMaxBlocks * kKB;       // columns per CTA at most
constexpr int kTok = 16;                      // MMA N: tokens, zero-padded
constexpr int kMaxCluster = 8;
constexpr int kXWarps = 8;                    // X workers: 4 columns per thread
constexpr int kXThreads = kXWarps * 32;
constexpr int kThreads = 64 + kXThreads;
constexpr int kMsgWords = 20;                 // exchange message: 16 maxima, count, pad
constexpr int kRecvRows = kRows + kMaxCluster;   // S * ceil(128 / S) <= 135
constexpr int kWPrefetch = 8;                 // outlier weights gathered ahead per row
constexpr int kStatusTimeout = -5;

static_assert(kXThreads * 4 == kCols, "X workers cover the CTA's columns");

// Named barriers (0 is __syncthreads).
constexpr uint32_t kBarX = 1;       // the X workers
constexpr uint32_t kBarList = 2;    // warp 2 publishes the local outlier list to warps 4-7
constexpr uint32_t kBarEpi = 3;     // warps 4-7

struct DecodeSmem {
  static constexpr int RING = 0;                                // [8][128][128] i8 (swizzled)
  static constexpr int BOP = RING + kMaxBlocks * kRows * kKB;   // [8][16][128] i8 (swizzled)
  static constexpr int XS = BOP + kMaxBlocks * kTok * kKB;      // [16][kw] f16
  static constexpr int RECV = XS + kTok * kCols * 2;            // [kRecvRows][8][16 B]
  static constexpr int MSG = RECV + kRecvRows * 128;            // [8 ranks][20] words
  static constexpr int BITS = MSG + kMaxCluster * kMsgWords * 4;   // [32] u32
  static constexpr int LIDX = BITS + 32 * 4;                    // [1024] u16
  static constexpr int RED = LIDX + kCols * 2;                  // [8 warps][16] f32
  static constexpr int TOK = RED + kXWarps * kTok * 4;          // amax[16], inv[16] f32
  static constexpr int WSC = TOK + 2 * kTok * 4;                // [128] f32 w_scale of owned rows
  static constexpr int MISC = WSC + kRows * 4;                  // lcount, prefix
  static constexpr int BARS = MISC + 16;                        // full[8] xbar codes done xchg red
  static constexpr int TSLOT = BARS + (kMaxBlocks + 5) * 8;
  static constexpr int TOTAL = TSLOT + 16;
  static constexpr int BYTES = TOTAL + 1024;                    // alignment slack
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Rows finished (owned) by `rank` when 128 rows are dealt out rpr at a time.
__device__ __forceinline__ int owned_rows(int rank, int rpr) {
  return max(0, min(rpr, kRows - rank * rpr));
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmWq, DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  // 1024-byte aligned base (swizzle atoms). Derived by an offset from the
  // shared array, not through an integer cast, so every pointer below stays in
  // the shared state space and compiles to shared-memory loads and stores.
  uint8_t* sm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  using L = DecodeSmem;
  uint8_t* ring = sm + L::RING;
  uint8_t* bop = sm + L::BOP;
  __half* xs = reinterpret_cast<__half*>(sm + L::XS);
  uint8_t* recv = sm + L::RECV;
  uint32_t* msg = reinterpret_cast<uint32_t*>(sm + L::MSG);
  uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L::BITS);
  uint16_t* lidx = reinterpret_cast<uint16_t*>(sm + L::LIDX);
  float* red = reinterpret_cast<float*>(sm + L::RED);
  float* amax_s = reinterpret_cast<float*>(sm + L::TOK);
  float* inv_s = amax_s + kTok;
  float* wsc = reinterpret_cast<float*>(sm + L::WSC);
  int32_t* misc = reinterpret_cast<int32_t*>(sm + L::MISC);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::BARS);
  uint64_t* xbar = full + kMaxBlocks;
  uint64_t* codes_bar = xbar + 1;
  uint64_t* done = xbar + 2;
  uint64_t* xchg = xbar + 3;
  uint64_t* redbar = xbar + 4;
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
  const int nb = min(nkb, kb0 + bper) - kb0;            // K-blocks of this CTA (1..8)
  const int k0 = min(K, kb0 * kKB);
  const int kw = min(K, (kb0 + nb) * kKB) - k0;         // columns of this CTA
  const int rpr = (kRows + S - 1) / S;                  // rows finished per rank
  const bool writer = (tile == 0);                      // cluster 0 writes intermediates

  if (tid == 0) {
    for (int b = 0; b < kMaxBlocks; ++b) mbar_init(&full[b], 1);
    mbar_init(xbar, 1);
    mbar_init(codes_bar, kXWarps);
    mbar_init(done, 1);
    mbar_init(xchg, 1);
    mbar_init(redbar, 1);
    // The peers' stores are counted in bytes; the one local arrival is made now.
    mbar_arrive_expect_tx(xchg, static_cast<uint32_t>(S * kMsgWords * 4));
    mbar_arrive_expect_tx(redbar, static_cast<uint32_t>(S * owned_rows(rank, rpr) * 128));
    fence_mbarrier_init();
    if (blockIdx.x == 0 && a.status) *a.status = 0;
    // Producer: X first (small, L2-resident after the first cluster), then the
    // whole Wq slice. Issued before the CTA barrier: only this thread has used
    // the barriers so far.
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(M * kw * 2));
    for (int t = 0; t < M; ++t)
      bulk_load(xs + t * kw, a.X + static_cast<size_t>(t) * K + k0, static_cast<uint32_t>(kw * 2),
                xbar);
    for (int b = 0; b < nb; ++b) {
      mbar_arrive_expect_tx(&full[b], kRows * kKB);
      tma_load_2d(ring + b * kRows * kKB, &tmWq, &full[b], (kb0 + b) * kKB, n0);
    }
  }
  if (warp == 1) {
    tmem_alloc(tslot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_arrive_relaxed();   // phase 1: this CTA's barriers are initialised
  const uint32_t tmem = *tslot;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (done)
    cluster_wait();
    cluster_arrive();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop; one elected lane issues each MMA.
    cluster_wait();
    ok = __all_sync(0xffffffffu, mbar_wait(codes_bar, 0));
    constexpr uint32_t idesc = make_idesc(2 /*s32*/, 1 /*signed*/, kRows, kTok);
    const uint64_t a0 = sw128_kmajor_desc(smem_addr(ring));
    const uint64_t b0 = sw128_kmajor_desc(smem_addr(bop));
    for (int b = 0; b < nb && ok; ++b) {
      ok = __all_sync(0xffffffffu, mbar_wait(&full[b], 0));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_i8_elect(tmem, a0 + static_cast<uint64_t>((b * kRows * kKB + 32 * kk) >> 4),
                     b0 + static_cast<uint64_t>((b * kTok * kKB + 32 * kk) >> 4), idesc,
                     (b | kk) != 0);
    }
    // Always committed, so the epilogue's wait ends even after a failed wait here.
    mma_commit_elect(done);
    cluster_arrive();
  } else {
    // ---------------------------------------------------------------- X workers
    // Loops over tokens stay rolled: this code runs once per launch, and
    // straight-line code would be bound by instruction fetch.
    const int xw = warp - 2;                 // 0..7
    const int xi = tid - 64;                 // 0..255
    const int c0 = 4 * xi;                   // first of the thread's 4 columns (CTA-local)
    const bool cv = c0 < kw;                 // kw is a multiple of 16
    const float thr = a.threshold;
    const bool epi = (warp >= 4 && warp < 8);
    const int r = (warp & 3) * 32 + lane;    // epilogue: tile row = TMEM lane
    const uint2* xrow = reinterpret_cast<const uint2*>(xs) + xi;   // + t * (kw / 4)
    const int xstride = kw >> 2;             // uint2 per token row

    ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0));

    // Outlier flags of the 4 columns: the max of |x| over all tokens against the threshold.
    __half2 m01 = __float2half2_rn(0.0f), m23 = m01;
    if (cv) {
#pragma unroll 4
      for (int t = 0; t < M; ++t) {
        const uint2 v = xrow[t * xstride];
        m01 = __hmax2(m01, habs2_bits(v.x));
        m23 = __hmax2(m23, habs2_bits(v.y));
      }
    }
    const float2 f01 = __half22float2(m01), f23 = __half22float2(m23);
    const uint32_t f4 = (f01.x > thr ? 1u : 0u) | (f01.y > thr ? 2u : 0u) |
                        (f23.x > thr ? 4u : 0u) | (f23.y > thr ? 8u : 0u);
    const uint32_t keep0 = ((f4 & 1u) ? 0u : 0x0000FFFFu) | ((f4 & 2u) ? 0u : 0xFFFF0000u);
    const uint32_t keep1 = ((f4 & 4u) ? 0u : 0x0000FFFFu) | ((f4 & 8u) ? 0u : 0xFFFF0000u);
    // Bitmap word of 32 columns = 8 threads x 4 flags.
    {
      uint32_t word = f4 << (4 * (lane & 7));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      word |= __shfl_xor_sync(0xffffffffu, word, 4);
      if ((lane & 7) == 0) bits[xi >> 3] = word;
    }
    // Per-token max of |x| over the non-outlier columns: per thread, then over
    // the warp (non-negative floats order like their bit patterns).
#pragma unroll 2
    for (int t = 0; t < M; ++t) {
      const uint2 v = cv ? xrow[t * xstride] : make_uint2(0u, 0u);
      const __half2 m = __hmax2(habs2_bits(v.x & keep0), habs2_bits(v.y & keep1));
      const float pm = fmaxf(__low2float(m), __high2float(m));
      const uint32_t wm = __reduce_max_sync(0xffffffffu, __float_as_uint(pm));
      if (lane == 0) red[xw * kTok + t] = __uint_as_float(wm);
    }
    named_bar_sync(kBarX, kXThreads);

    if (xw == 0) {
      // Local outlier list (ascending) and count; then the message to every rank.
      const int words = (kw + 31) >> 5;
      const uint32_t bw = (lane < words) ? bits[lane] : 0u;
      const int c = __popc(bw);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      uint32_t bb = bw;
      int p = incl - c;
      while (bb) {
        const int j = __ffs(bb) - 1;
        bb &= bb - 1;
        lidx[p++] = static_cast<uint16_t>(lane * 32 + j);
      }
      const int lcount = __shfl_sync(0xffffffffu, incl, 31);
      // CTA maxima of the tokens (0 for the padding tokens).
      float cm = 0.0f;
      if (lane < M) {
        for (int w = 0; w < kXWarps; ++w) cm = fmaxf(cm, red[w * kTok + lane]);
      }
      if (lane == 0) misc[0] = lcount;
      __syncwarp();
      // Lane l alone read red[w][l]; its CTA maximum replaces red[0][l].
      if (lane < kTok) red[lane] = cm;
      __syncwarp();
      named_bar_arrive(kBarList, 32 + 128);
      cluster_wait();   // every CTA's barriers are initialised
      for (int i = lane; i < S * 5; i += 32) {
        const int dst = i / 5, ch = i - dst * 5;
        uint32_t v[4] = {static_cast<uint32_t>(lcount), 0u, 0u, 0u};
        if (ch < 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(red + 4 * ch);
          v[0] = __float_as_uint(m4.x);
          v[1] = __float_as_uint(m4.y);
          v[2] = __float_as_uint(m4.z);
          v[3] = __float_as_uint(m4.w);
        }
        st_async_v4(cluster_addr(&msg[rank * kMsgWords + 4 * ch], dst), v[0], v[1], v[2], v[3],
                    cluster_addr(xchg, dst));
      }
    } else {
      cluster_wait();
    }

    // Epilogue warps: start the gathers of the outlier weights now, they have
    // the whole exchange and the code pass to land.
    int lcount = 0;
    __half wv[kWPrefetch];
    if (epi) {
      named_bar_sync(kBarList, 32 + 128);
      lcount = misc[0];
      const int n = n0 + r;
      const __half* wrow = a.W + static_cast<size_t>(min(n, N - 1)) * K + k0;
#pragma unroll
      for (int j = 0; j < kWPrefetch; ++j)
        wv[j] = (j < lcount && n < N) ? wrow[lidx[j]] : __float2half(0.0f);
      const int owned = owned_rows(rank, rpr);
      if (r < owned) {
        const int nr = n0 + rank * rpr + r;
        wsc[r] = (nr < N) ? a.w_scale[nr] : 0.0f;
      }
    }

    // Token absmax over the whole cluster, its inverse, the outlier prefix.
    ok = __all_sync(0xffffffffu, mbar_wait(xchg, 0)) && ok;
    if (xw == 0) {
      if (lane < kTok) {
        float m = 0.0f;
        for (int s2 = 0; s2 < S; ++s2) m = fmaxf(m, __uint_as_float(msg[s2 * kMsgWords + lane]));
        amax_s[lane] = m;
        inv_s[lane] = quant_inv(m);
        if (writer && rank == 0 && lane < M) a.x_scale[lane] = m;
      }
      if (lane == 0) {
        int prefix = 0, total = 0;
        for (int s2 = 0; s2 < S; ++s2) {
          const int cs = static_cast<int>(msg[s2 * kMsgWords + 16]);
          if (s2 < rank) prefix += cs;
          total += cs;
        }
        misc[1] = prefix;
        if (writer && rank == 0) *a.n_outliers = total;
      }
    }
    named_bar_sync(kBarX, kXThreads);

    if (writer) {
      if (xi < ((kw + 31) >> 5)) a.bitmap[(k0 >> 5) + xi] = bits[xi];
      const int lc = misc[0], prefix = misc[1];
      for (int i = xi; i < lc; i += kXThreads) a.col_idx[prefix + i] = k0 + lidx[i];
    }

    // INT8 codes of the 4 columns for every token, into the B operand (and Xq).
    if (c0 < nb * kKB) {
      const uint32_t kc = static_cast<uint32_t>(c0) & 127u;
      uint8_t* dst = bop + (c0 >> 7) * (kTok * kKB) + (kc & 15u);
      const uint32_t keepq = keep_bytes(f4);
      int8_t* xq = a.Xq + k0 + c0;
#pragma unroll 2
      for (int t = 0; t < kTok; ++t) {
        uint32_t q = 0u;
        if (cv && t < M) {
          q = codes4(xrow[t * xstride], amax_s[t], inv_s[t]) & keepq;
          if (writer) *reinterpret_cast<uint32_t*>(xq + static_cast<size_t>(t) * K) = q;
        }
        const uint32_t off = (t >> 3) * 1024 + (t & 7) * 128 + (((kc >> 4) ^ (t & 7)) << 4);
        *reinterpret_cast<uint32_t*>(dst + off) = q;
      }
    }
    fence_proxy_async_smem();   // the tensor core reads what the generic proxy wrote
    __syncwarp();
    if (lane == 0) mbar_arrive(codes_bar);

    if (!epi) {
      cluster_arrive();
    } else {
      // fp32 outlier partials of this row over the CTA's outlier columns.
      float o[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) o[t] = 0.0f;
      const int n = n0 + r;
      const __half* wrow = a.W + static_cast<size_t>(min(n, N - 1)) * K + k0;
#pragma unroll 1
      for (int j = 0; j < lcount; ++j) {
        const int col = lidx[j];
        __half wh = __float2half(0.0f);
#pragma unroll
        for (int i = 0; i < kWPrefetch; ++i)
          if (i == j) wh = wv[i];
        if (j >= kWPrefetch && n < N) wh = wrow[col];
        const float w = __half2float(wh);
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t < M) o[t] = fmaf(__half2float(xs[t * kw + col]), w, o[t]);
      }

      // INT32 partials of the row from TMEM.
      uint32_t acc[kTok];
      const bool got = __all_sync(0xffffffffu, mbar_wait(done, 0));
      if (got) {
        tc_fence_after();
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), acc);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int t = 0; t < kTok; ++t) acc[t] = 0u;
      }
      ok = ok && got;

      // Push the row's partials to the rank that finishes it: 8 chunks of 16 B,
      // chunk c at position c ^ (row & 7) to spread the banks of the final reads.
      {
        const int own = r / rpr, rl = r - own * rpr;
        const uint32_t base = cluster_addr(recv + (rank * rpr + rl) * 128, own);
        const uint32_t bar = cluster_addr(redbar, own);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t pos = static_cast<uint32_t>(ch ^ (rl & 7)) << 4;
          if (ch < 4)
            st_async_v4(base + pos, acc[4 * ch], acc[4 * ch + 1], acc[4 * ch + 2], acc[4 * ch + 3],
                        bar);
          else
            st_async_v4(base + pos, __float_as_uint(o[4 * (ch - 4)]),
                        __float_as_uint(o[4 * (ch - 4) + 1]), __float_as_uint(o[4 * (ch - 4) + 2]),
                        __float_as_uint(o[4 * (ch - 4) + 3]), bar);
        }
      }
      cluster_arrive();

      // Finish the owned rows: sum the S partials in rank order, dequantise, add.
      ok = __all_sync(0xffffffffu, mbar_wait(redbar, 0)) && ok;
      named_bar_sync(kBarEpi, 128);   // wsc of all owned rows is written
      const int owned = owned_rows(rank, rpr);
      const int32_t* ri = reinterpret_cast<const int32_t*>(recv);
      const float* rf = reinterpret_cast<const float*>(recv);
#pragma unroll 1
      for (int e = (warp & 3) * 32 + lane; e < owned * kTok; e += 128) {
        const int t = e / owned;
        const int rl = e - t * owned;
        const int nn = n0 + rank * rpr + rl;
        if (t < M && nn < N) {
          const int pi = (((t >> 2) ^ (rl & 7)) << 2) + (t & 3);
          const int pf = (((4 + (t >> 2)) ^ (rl & 7)) << 2) + (t & 3);
          int32_t c = 0;
          float of = 0.0f;
          for (int s2 = 0; s2 < S; ++s2) {
            const int row = (s2 * rpr + rl) * 32;
            c += ri[row + pi];
            of += rf[row + pf];
          }
          const float rs = amax_s[t] * (1.0f / 16129.0f);
          const float y = static_cast<float>(c) * (rs * wsc[rl]) + of;
          a.Y[static_cast<size_t>(t) * N + nn] = __float2half_rn(y);
        }
      }
    }
  }

  if (!ok && lane == 0 && a.status) atomicExch(a.status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  cluster_wait();   // no CTA leaves while a peer may still store into it
}

}  // namespace

bool decode_supported(int M, int K) {
  return M >= 1 && M <= kTok && K <= kMaxCluster * kMaxBlocks * kKB;
}

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

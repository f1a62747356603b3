// Decode-shape path (M <= 16 tokens) of the LLM.int8() matmul, one launch.
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier detection by threshold, vector-wise absmax INT8 quantisation of the
// rest, INT8 matmul with INT32 accumulation, dequantisation by the outer product
// of the scales, FP16 product over the outlier columns, final sum); tanjunchen
// "quantization explained part 2" section 1.2 (threshold 6.0).
//
// With at most 16 tokens the work is bound by reading Wq once; everything else
// is arranged to finish while that stream is in flight, and the per-CTA work on
// the critical path is kept small because it runs on few warps.
//
// The grid is made of clusters of S <= 8 CTAs. A cluster owns 128 output
// features (rows of Wq) and its CTAs split K, so every CTA reads a 128 x (K/S)
// slice of Wq as nbox = 8 TMA boxes of 128 rows x 128 bytes, all requested at
// kernel start (K = 4096: clusters of 4, one CTA per SM, all resident at once).
// The layout also supports nbox = 4 (about 100 KB, two CTAs per SM, clusters of
// 8); that variant measured slower because the launch of its 256 CTAs spread
// over about 2 us.
//
// Warp roles (64 + 32*nxw threads, nxw = 2*nbox X workers):
//   warp 0        barrier set-up and the copies: the CTA's K-range of X (2-D
//                 boxes; tokens past M read as zeros), then the Wq slice
//   warp 1        TMEM allocator and MMA issuer: tcgen05.mma kind::i8,
//                 M = 128 weight rows, N = 16 tokens, issued by an elected lane
//   X workers     2 columns per thread, loops over the tokens: exact outlier
//                 flags (every token is here), per-token maxima over the
//                 non-outlier columns (one redux per token and warp), and after
//                 the cluster exchange of those maxima the INT8 codes, written
//                 into the 128-byte-swizzled K-major B operand of the MMA
//   warps 4-7     (X workers too) the epilogue: the fp32 outlier partials of the
//                 CTA's own outlier columns on CUDA cores (fp16 products are
//                 exact in fp32), the INT32 partials from TMEM dequantised with
//                 the row and column scales, and the cross-CTA sum.
//
// Cross-CTA traffic uses st.async into the peer's shared memory, counted in
// bytes on the peer's mbarrier: one 80-byte message per CTA pair with the
// per-token maxima and the outlier count; then each CTA pushes every row's 16
// fp32 partial results to the CTA that finishes that row, which adds the S
// partials in rank order and writes Y. A split cluster barrier publishes the
// mbarrier initialisation and keeps every CTA alive until its peers have issued
// their last store into it. Cluster 0 also writes the intermediates the
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

constexpr int kTileRows = 128;                // MMA M = output rows per cluster
constexpr int kKB = 128;                      // int8 columns per K-block (one swizzle row)
constexpr int kMaxBoxes = 8;                  // Wq boxes (128 x 128 B) per CTA, all in flight
constexpr int kBoxBytes = kTileRows * kKB;
constexpr int kTok = 16;                      // MMA N: tokens, zero-padded
constexpr int kMaxCluster = 8;
constexpr int kMaxCols = kMaxBoxes * kKB;     // columns per CTA at most
constexpr int kXBox = 256;                    // fp16 columns per X box
constexpr int kMaxXWarps = kMaxCols / 64;     // 2 columns per thread
constexpr int kMsgWords = 20;                 // exchange message: 16 maxima, count, pad
constexpr int kRecvRows = kTileRows + kMaxCluster;   // S * ceil(128 / S) <= 128 + S - 1
constexpr int kWPrefetch = 8;                 // outlier weights gathered ahead per row
constexpr int kStatusTimeout = -5;

// Named barriers (0 is __syncthreads).
constexpr uint32_t kBarX = 1;       // the X workers
constexpr uint32_t kBarList = 2;    // the first X warp publishes the outlier list to warps 4-7
constexpr uint32_t kBarCodes = 3;   // the X workers' codes are in the B operand (MMA warps wait)

// Shared-memory layout for nbox Wq boxes per CTA (offsets from a 1024-byte
// aligned base).
struct DecodeSmem {
  int ring, bop, xs, recv, cm, msg, bits, lidx, red, tok, misc, bars, tslot, bytes;
};
__host__ __device__ inline DecodeSmem decode_layout(int nbox) {
  DecodeSmem L;
  int off = 0;
  L.ring = off;  off += nbox * kBoxBytes;                 // [nbox] Wq boxes (swizzled)
  L.bop = off;   off += nbox * kTok * kKB;                // [nbox][16][128] i8 (swizzled)
  L.xs = off;    off += nbox * kKB * kTok * 2;            // [nbox/2][16][256] f16
  L.recv = off;  off += kRecvRows * 64;                   // [rows][4][16 B] fp32 partials
  L.cm = off;    off += 4 * 128 * 16;                     // [4 token quarters][128 groups] column maxima
  L.msg = off;   off += kMaxCluster * kMsgWords * 4;      // [8 ranks][20] words
  L.bits = off;  off += 32 * 4;                           // outlier bitmap of the columns
  L.lidx = off;  off += kMaxCols * 2;                     // ascending outlier list
  L.red = off;   off += kMaxXWarps * kTok * 4;            // [warps][16] f32
  L.tok = off;   off += 3 * kTok * 4;                     // amax, amax/127^2, 1/amax
  L.misc = off;  off += 16;                               // lcount, prefix
  L.bars = off;  off += (2 * kMaxBoxes + 5) * 8;          // full[8] codes[8] xbar - done xchg red
  L.tslot = off; off += 16;
  L.bytes = off + 1024;                                   // alignment slack
  return L;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Rows finished (owned) by `rank` when the 128 rows are dealt out rpr at a time.
__device__ __forceinline__ int owned_rows(int rank, int rpr) {
  return max(0, min(rpr, kTileRows - rank * rpr));
}

__global__ void __launch_bounds__(64 + 32 * kMaxXWarps, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmWq, const __grid_constant__ CUtensorMap tmX,
                  DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  // 1024-byte aligned base, derived by an offset so pointers stay in the shared space.
  uint8_t* sm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  const int nbox = a.nbox;                              // 4 or 8
  const DecodeSmem L = decode_layout(nbox);
  uint8_t* ring = sm + L.ring;
  uint8_t* bop = sm + L.bop;
  __half* xs = reinterpret_cast<__half*>(sm + L.xs);
  uint8_t* recv = sm + L.recv;
  uint8_t* cmx_s = sm + L.cm;
  uint32_t* msg = reinterpret_cast<uint32_t*>(sm + L.msg);
  uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L.bits);
  uint16_t* lidx = reinterpret_cast<uint16_t*>(sm + L.lidx);
  float* red = reinterpret_cast<float*>(sm + L.red);
  float* amax_s = reinterpret_cast<float*>(sm + L.tok);
  float* rs_s = amax_s + kTok;
  float* ra_s = amax_s + 2 * kTok;
  int32_t* misc = reinterpret_cast<int32_t*>(sm + L.misc);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* cbar = full + kMaxBoxes;        // codes of K-block b written
  uint64_t* xbar = cbar + kMaxBoxes;
  uint64_t* done = xbar + 2;
  uint64_t* xchg = xbar + 3;
  uint64_t* redbar = xbar + 4;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L.tslot);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  griddep_launch_dependents();
  const int S = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int nxw = 2 * nbox;                             // X worker warps
  const int nxt = 32 * nxw;
  const int tile = blockIdx.x / S;
  const int n0 = tile * kTileRows;
  const int M = a.M, N = a.N, K = a.K;
  const int nkb = (K + kKB - 1) / kKB;
  const int bper = (nkb + S - 1) / S;
  const int kb0 = min(nkb, rank * bper);
  const int nb = min(nkb, kb0 + bper) - kb0;            // K-blocks of this CTA (1..nbox)
  const int k0 = min(K, kb0 * kKB);
  const int kw = min(K, (kb0 + nb) * kKB) - k0;         // columns of this CTA
  const int nbx = (kw + kXBox - 1) / kXBox;             // X boxes
  const int rpr = (kTileRows + S - 1) / S;              // rows finished per rank
  const bool writer = (tile == 0);                      // cluster 0 writes intermediates

  if (tid == 0) {
    for (int b = 0; b < kMaxBoxes; ++b) mbar_init(&full[b], 1);
    mbar_init(xbar, 1);

    mbar_init(done, 2);   // the two MMA-issuing warps commit
    mbar_init(xchg, 1);
    mbar_init(redbar, 1);
    // The peers' stores are counted in bytes; the one local arrival is made now.
    mbar_arrive_expect_tx(xchg, static_cast<uint32_t>(S * kMsgWords * 4));
    mbar_arrive_expect_tx(redbar, static_cast<uint32_t>(S * owned_rows(rank, rpr) * 64));
    fence_mbarrier_init();
    // Launched with programmatic stream serialization: the set-up above overlaps
    // the previous kernel; every global access comes after this wait.
    griddep_wait();
    if (blockIdx.x == 0 && a.status) *a.status = 0;
    // X first (small, L2-resident after the first cluster), then the Wq slice.
    // Issued before the CTA barrier: only this thread has used the barriers.
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(nbx * kTok * kXBox * 2));
    for (int j = 0; j < nbx; ++j)
      tma_load_2d(xs + j * kTok * kXBox, &tmX, xbar, k0 + j * kXBox, 0);
    for (int b = 0; b < nb; ++b) {
      mbar_arrive_expect_tx(&full[b], kBoxBytes);
      tma_load_2d(ring + b * kBoxBytes, &tmWq, &full[b], (kb0 + b) * kKB, n0);
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
  if (tid != 0) griddep_wait();
  const uint32_t tmem = *tslot;
  bool ok = true;

  if (warp <= 1) {
    // ---------------------------------------------------------------- MMA issuers
    // Two warps issue the MMAs, each into its own 16-column TMEM accumulator:
    // warp 1 the first ceil(nb/2) K-blocks, warp 0 the rest (one issuing lane
    // of a converged warp issues an MMA every few tens of cycles; two halve the
    // issue time). The epilogue adds the two accumulators.
    cluster_wait();
    const int half = nb - nb / 2;
    const int b_lo = warp == 1 ? 0 : half;
    const int b_hi = warp == 1 ? half : nb;
    const uint32_t acc = tmem + (warp == 1 ? 0u : static_cast<uint32_t>(kTok));
    // The X workers' code stores are fenced to the async proxy and released
    // through named barrier kBarCodes (a thread sync); the Wq boxes come from
    // TMA and need only their mbarrier.
    named_bar_sync(kBarCodes, 64 + nxt);
    tc_fence_after();
    constexpr uint32_t idesc = make_idesc(2 /*s32*/, 1 /*signed*/, kTileRows, kTok);
    const uint64_t a0 = sw128_kmajor_desc(smem_addr(ring));
    const uint64_t b0 = sw128_kmajor_desc(smem_addr(bop));
    for (int b = b_lo; b < b_hi && ok; ++b) {
      ok = __all_sync(0xffffffffu, mbar_wait(&full[b], 0));
      if (!ok) break;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_i8_elect(acc, a0 + static_cast<uint64_t>((b * kBoxBytes + 32 * kk) >> 4),
                     b0 + static_cast<uint64_t>((b * kTok * kKB + 32 * kk) >> 4), idesc,
                     ((b - b_lo) | kk) != 0);
    }
    // Always committed, so the epilogue's wait ends even after a failed wait here.
    mma_commit_elect(done);
    cluster_arrive();
  } else if (warp - 2 >= nxw) {
    cluster_wait();
    cluster_arrive();
  } else {
    // ---------------------------------------------------------------- X workers
    // Loops over tokens stay rolled: this code runs once per launch on few
    // warps, and straight-line code would be bound by instruction fetch.
    const int xw = warp - 2;
    const int xi = tid - 64;
    const float thr = a.threshold;
    const bool epi = (warp >= 4 && warp < 8);
    constexpr int xvs = kXBox / 8;           // 16-byte vectors per token row of an X box
    const int ng = kw >> 3;                  // 8-column groups of this CTA's slice
    // Group g of the slice: box g / 32, columns 8g % 256 .. +7.
    auto xgroup = [&](int g) -> const uint4* {
      return reinterpret_cast<const uint4*>(xs + (g >> 5) * (kTok * kXBox) + ((8 * g) & (kXBox - 1)));
    };

    ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0));

    // Thread (g, tq): the 8 columns of group g = xi % 128 for the tokens
    // 4tq .. 4tq+3, tq = xi / 128 (one token quarter per warp).
    const int g = xi & 127;
    const int tq = xi >> 7;
    const bool gv = g < ng;
    uint4 xv[4];
    {
      __half2 cm[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) cm[k] = __float2half2_rn(0.0f);
      const uint4* xg = xgroup(gv ? g : 0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = 4 * tq + j;
        xv[j] = (gv && t < M) ? xg[t * xvs] : make_uint4(0, 0, 0, 0);
        const uint32_t* wd = reinterpret_cast<const uint32_t*>(&xv[j]);
#pragma unroll
        for (int k = 0; k < 4; ++k) cm[k] = __hmax2(cm[k], habs2_bits(wd[k]));
      }
      reinterpret_cast<uint4*>(cmx_s)[tq * 128 + g] = *reinterpret_cast<const uint4*>(cm);
    }
    named_bar_sync(kBarX, nxt);
    // Outlier flags of the 8 columns: the max of |x| over all tokens against the threshold.
    uint32_t f8 = 0;
    {
      __half2 cm[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) cm[k] = __float2half2_rn(0.0f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = reinterpret_cast<const uint4*>(cmx_s)[q * 128 + g];
        const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int k = 0; k < 4; ++k) cm[k] = __hmax2(cm[k], h[k]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 m = __half22float2(cm[k]);
        f8 |= (m.x > thr ? 1u : 0u) << (2 * k);
        f8 |= (m.y > thr ? 1u : 0u) << (2 * k + 1);
      }
      if (!gv) f8 = 0;
    }
    if (tq == 0) {
      // Bitmap word of 32 columns = 4 consecutive groups.
      uint32_t word = f8 << (8 * (lane & 3));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      if ((lane & 3) == 0 && gv) bits[g >> 2] = word;
    }
    // Per-token max of |x| over the non-outlier columns, per warp with one
    // redux (non-negative floats order like their bit patterns); the warp's
    // slots of the other quarters' tokens hold 0.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t* wd = reinterpret_cast<const uint32_t*>(&xv[j]);
      __half2 h = __float2half2_rn(0.0f);
#pragma unroll
      for (int k = 0; k < 4; ++k) h = __hmax2(h, habs2_bits(wd[k] & keep_half2(f8, k)));
      const float2 f = __half22float2(h);
      const uint32_t wm = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(f.x, f.y)));
      if (lane == 0) red[xw * kTok + 4 * tq + j] = __uint_as_float(wm);
    }
    if (lane < kTok && (lane >> 2) != tq) red[xw * kTok + lane] = 0.0f;
    named_bar_sync(kBarX, nxt);

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
      float cmx = 0.0f;
      if (lane < M) {
        for (int w = 0; w < nxw; ++w) cmx = fmaxf(cmx, red[w * kTok + lane]);
      }
      if (lane == 0) misc[0] = lcount;
      __syncwarp();
      // Lane l alone read red[w][l]; its CTA maximum replaces red[0][l].
      if (lane < kTok) red[lane] = cmx;
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

    // Epilogue warps: start the gathers of the outlier weights and the column
    // scales now; they have the exchange and the code pass to land.
    const int q = warp & 3;
    const int r = q * 32 + lane;             // epilogue: row of the cluster = TMEM lane
    const int n = n0 + r;
    int lcount = 0;
    __half wv[kWPrefetch];
    float wsr = 0.0f;
    if (epi) {
      named_bar_sync(kBarList, 32 + 128);
      lcount = misc[0];
      // Outlier feature k of the weight is row k of Wt ([K][N]): consecutive
      // threads read consecutive n.
      const __half* wcol = a.W + static_cast<size_t>(k0) * N + (n < N ? n : 0);
#pragma unroll
      for (int i = 0; i < kWPrefetch; ++i)
        wv[i] = (n < N && i < lcount) ? wcol[static_cast<size_t>(lidx[i]) * N] : __float2half(0.0f);
      wsr = (n < N) ? a.w_scale[n] : 0.0f;
    }

    // Token absmax over the whole cluster, its inverse, the outlier prefix
    // (for the epilogue, x_scale and the outlier list; the code warps take
    // their tokens' absmax from the messages themselves).
    ok = __all_sync(0xffffffffu, mbar_wait(xchg, 0)) && ok;
    if (xw == 0) {
      if (lane < kTok) {
        float m = 0.0f;
        for (int s2 = 0; s2 < S; ++s2) m = fmaxf(m, __uint_as_float(msg[s2 * kMsgWords + lane]));
        amax_s[lane] = m;
        rs_s[lane] = m * (1.0f / 16129.0f);
        ra_s[lane] = quant_rcp(m);
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
    // INT8 codes into the B operand (and Xq): thread xi takes K-block
    // b = xi / 64, group gi = xi % 16 of the block's 16, and the tokens
    // 4tc .. 4tc+3, tc = (xi / 16) % 4.
    {
      const int b = xi >> 6;
      const int gi = xi & 15;
      const int tc = (xi >> 4) & 3;
      const int gg = b * 16 + gi;
      if (b < nb) {
        const bool live = gg < ng;
        const uint32_t m8 = live ? (bits[gg >> 2] >> (8 * (gg & 3))) & 0xFFu : 0xFFu;
        const uint4* xg = xgroup(live ? gg : 0);
        uint8_t* dst = bop + b * (kTok * kKB) + (gi & 1) * 8;
        int8_t* xq = a.Xq + k0 + 8 * gg;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = 4 * tc + j;
          uint2 qv = make_uint2(0u, 0u);
          if (live && t < M) {
            float am = 0.0f;
            for (int s2 = 0; s2 < S; ++s2) am = fmaxf(am, __uint_as_float(msg[s2 * kMsgWords + t]));
            qv = codes8(xg[t * xvs], am, quant_rcp(am));
            if (m8) {
              qv.x &= keep_bytes(m8 & 0xFu);
              qv.y &= keep_bytes(m8 >> 4);
            }
            if (writer) *reinterpret_cast<uint2*>(xq + static_cast<size_t>(t) * K) = qv;
          }
          // Row t of the 128-byte-swizzled K-major operand: 16-byte chunk gi/2
          // of the block's 128 columns, XOR the row's position in its 8-row group.
          const uint32_t off = (t >> 3) * 1024 + (t & 7) * 128 + ((((gi >> 1) ^ (t & 7))) << 4);
          *reinterpret_cast<uint2*>(dst + off) = qv;
        }
        fence_proxy_async_smem();   // the tensor core reads what the generic proxy wrote
      }
    }
    named_bar_arrive(kBarCodes, 64 + nxt);
    named_bar_sync(kBarX, nxt);   // amax_s, rs_s and the prefix of the first X warp

    if (writer) {
      if (xi < ((kw + 31) >> 5)) a.bitmap[(k0 >> 5) + xi] = bits[xi];
      const int lc = misc[0], prefix = misc[1];
      for (int i = xi; i < lc; i += nxt) a.col_idx[prefix + i] = k0 + lidx[i];
    }

    if (!epi) {
      cluster_arrive();
    } else {
      // fp32 outlier partials of this row over the CTA's outlier columns.
      float o[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) o[t] = 0.0f;
      const __half* wcol = a.W + static_cast<size_t>(k0) * N + (n < N ? n : 0);
#pragma unroll 1
      for (int jj = 0; jj < lcount; ++jj) {
        const int col = lidx[jj];
        __half wh = __float2half(0.0f);
#pragma unroll
        for (int i = 0; i < kWPrefetch; ++i)
          if (i == jj) wh = wv[i];
        if (jj >= kWPrefetch && n < N) wh = wcol[static_cast<size_t>(col) * N];
        const float w = __half2float(wh);
        const __half* xc = xs + (col >> 8) * (kTok * kXBox) + (col & (kXBox - 1));
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t < M) o[t] = fmaf(__half2float(xc[t * kXBox]), w, o[t]);
      }
      // INT32 partials of the row from TMEM, dequantised with the scales.
      const bool got = __all_sync(0xffffffffu, mbar_wait(done, 0));
      ok = ok && got;
      uint32_t acc[kTok];
      if (got) {
        tc_fence_after();
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16), acc);
        if (nb >= 2) {
          uint32_t acc2[kTok];
          tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + kTok, acc2);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < kTok; ++t)
            acc[t] = static_cast<uint32_t>(static_cast<int32_t>(acc[t]) + static_cast<int32_t>(acc2[t]));
        }
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int t = 0; t < kTok; ++t) acc[t] = 0u;
      }
      float y[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t)
        y[t] = static_cast<float>(static_cast<int32_t>(acc[t])) * (rs_s[t] * wsr) + o[t];
      // Push to the rank that finishes the row: 4 chunks of 16 B, chunk c at
      // position c ^ (row & 3) to spread the banks of the final reads.
      {
        const int own = r / rpr, rl = r - own * rpr;
        const uint32_t base = cluster_addr(recv + (rank * rpr + rl) * 64, own);
        const uint32_t bar = cluster_addr(redbar, own);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          st_async_v4(base + (static_cast<uint32_t>(ch ^ (rl & 3)) << 4),
                      __float_as_uint(y[4 * ch]), __float_as_uint(y[4 * ch + 1]),
                      __float_as_uint(y[4 * ch + 2]), __float_as_uint(y[4 * ch + 3]), bar);
      }
      cluster_arrive();

      // Finish the owned rows: add the S partials in rank order, write Y.
      ok = __all_sync(0xffffffffu, mbar_wait(redbar, 0)) && ok;
      const int owned = owned_rows(rank, rpr);
      const float4* rv = reinterpret_cast<const float4*>(recv);
#pragma unroll 1
      for (int e = q * 32 + lane; e < owned * 4; e += 128) {
        const int tg = e / owned;               // tokens 4tg..4tg+3
        const int rl = e - tg * owned;
        const int nn = n0 + rank * rpr + rl;
        float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int s2 = 0; s2 < S; ++s2) {
          const float4 v = rv[(s2 * rpr + rl) * 4 + (tg ^ (rl & 3))];
          sum.x += v.x;
          sum.y += v.y;
          sum.z += v.z;
          sum.w += v.w;
        }
        if (nn < N) {
          const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (4 * tg + i < M) a.Y[static_cast<size_t>(4 * tg + i) * N + nn] = __float2half_rn(sv[i]);
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
  return M >= 1 && M <= kTok && K <= kMaxCluster * kMaxBoxes * kKB;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const int nkb = (a.K + kKB - 1) / kKB;
  // Eight boxes per CTA: clusters of 4 (K = 4096) are all resident with one CTA
  // per SM and start together; four boxes per CTA (clusters of 8, two CTAs per
  // SM) measured slower, their launch spread over about 2 us.
  const int nbox = kMaxBoxes;
  const int S = max(1, (nkb + nbox - 1) / nbox);        // CTAs per cluster
  if (S > kMaxCluster) return cudaErrorInvalidValue;
  const int tiles = (a.N + kTileRows - 1) / kTileRows;
  CUtensorMap tmw, tmx;
  std::memset(&tmw, 0, sizeof(tmw));
  std::memset(&tmx, 0, sizeof(tmx));
  if (!make_tmap_sw128(&tmw, a.Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.N, kTileRows))
    return cudaErrorInvalidValue;
  // X boxes: 16 token rows (rows past M read as zeros) x 256 fp16 columns.
  if (!make_tmap_2d(&tmx, a.X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.K, a.M, kTok, kXBox * 2,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int smem = decode_layout(nbox).bytes;
  static int attr_bytes[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || attr_bytes[dev] < smem) {
    e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode_layout(kMaxBoxes).bytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_bytes[dev] = decode_layout(kMaxBoxes).bytes;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * S);
  cfg.blockDim = dim3(64 + 32 * 2 * nbox);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  DecodeArgs args = a;
  args.nbox = nbox;
  e = cudaLaunchKernelEx(&cfg, decode_kernel, tmw, tmx, args);
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

}  // namespace i8mm

// Fused detection + quantisation + compaction for the full LLM.int8() path,
// one cooperative launch (all CTAs co-resident), in its two-pass form. The
// library uses it for the zero-point codes (scholia section 6); the absmax
// codes run the single-pass kernel of stream_quant.cu.
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier feature dimensions by a magnitude threshold, vector-wise absmax INT8
// quantisation of the remaining dimensions, the outlier dimensions kept in
// fp16); tanjunchen "quantization explained part 2", section 1.2 (threshold 6.0;
// once the outlier dimension is split out the scale comes from the rest).
//
// The outlier set O is a property of the whole batch, so no code is final
// before every CTA has looked at its rows. The kernel does not wait for that:
// each CTA quantises its rows against its OWN outlier set (the columns where
// one of its rows exceeds the threshold, a subset of O) while the other CTAs
// are still reading, and checks afterwards. A CTA whose rows show every column
// of O (with outliers on most tokens and several rows per CTA, nearly always)
// is done; the others redo their rows with O. The results are the same either
// way; only the time differs.
//
// Each CTA owns a contiguous block of R rows of X and of the rows of W.
//   pass A   all 16 warps: the rows stream through a ring of S row slots in
//            shared memory (bulk copies, one mbarrier per slot; a chunk's slots
//            are refilled with the rows S further on once every thread is done
//            with it). Thread t owns the 16-byte vectors v = t + 512*c of every
//            row and keeps a packed-fp16 running max of |x| per owned column;
//            the column maxima against the threshold give the CTA's outlier
//            flags, ORed into the batch bitmap (atomics only for non-zero
//            words). Afterwards the slots hold the last min(R, S) rows.
//   pass B   warps 0-14: per row the absmax over the non-outlier columns of the
//            CTA's own set (redux per warp; teams of warps share a row through
//            named barrier 1) and the INT8 codes with paired fp32 arithmetic;
//            the rows still in their slots are read from shared memory, the
//            others again from L2 into registers, a few rows per round.
//   control  warp 15, meanwhile: arrives at the grid barrier, builds the CTA's
//            ascending outlier list, waits at the barrier (bounded) and compares
//            the batch bitmap with the CTA's.
//   redo     only if the batch has a column the CTA's rows missed: pass B and
//            the list again with the batch's set.
//   panels   with any outlier column, by the workers right after pass B (with
//            the CTA's list; again after a redo): the CTA's rows of the
//            compacted fp16 panels X_O (from the slots or L2) and W_O (gathered
//            from the rows of the transposed weight Wt [K][N] that the list
//            names), a multiple of 64 columns wide and zero-padded. The GEMM
//            multiplies them on the tensor cores.

// The code of x is rint(fl32(fl32(x*127)/a)) clamped to +-127. The correctly
// rounded quotient is formed without a division (codes8 in quant_common.cuh:
// Markstein's FMA-corrected product with fl(1/a), exact for every pair of fp16
// values with |x| <= a) and rounded with the 1.5*2^23 trick (ties to even in
// one add; the code lands in the low byte).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace i8mm {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
// After pass A the last warp is the control warp (grid-barrier arrival and
// wait, the outlier list, the check); the others quantise, synchronising among
// themselves on named barrier 1.
constexpr int kWorkers = kWarps - 1;
constexpr uint32_t kWorkBar = 1;
constexpr uint32_t kListBar = 2;   // the control warp has built the CTA's list
constexpr int kMaxSlots = 16;                 // row slots in shared memory
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace

// Shared-memory layout of one CTA (16-byte aligned pieces):
//   rows    [S][K] fp16        row slots, filled by bulk copies
//   lbits   [words] u32        the CTA's own outlier bitmap
//   gbits   [words] u32        the global bitmap, after the grid barrier
//   red     [2][2][kWarps] f32 per-warp partial row maxima (and of -x, zero point),
//                              alternating between consecutive rounds
//   misc    [4] i32            outlier count of the current list
//   idx     [K] u16            ascending outlier columns of the current list
//   bar     [S] u64            one mbarrier per slot
struct FusedSmem {
  size_t rows, lbits, gbits, red, misc, idx, bar, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

__host__ __device__ inline FusedSmem fused_smem_layout(int K, int S) {
  FusedSmem L;
  const size_t words = static_cast<size_t>((K + 31) / 32);
  size_t off = 0;
  L.rows = off;   off = align16(off + static_cast<size_t>(S) * K * 2);
  L.lbits = off;  off = align16(off + words * 4);
  L.gbits = off;  off = align16(off + words * 4);
  L.red = off;    off = align16(off + 4 * kWarps * 4);
  L.misc = off;   off = align16(off + 16);
  L.idx = off;    off = align16(off + static_cast<size_t>(K) * 2);
  L.bar = off;    off = align16(off + static_cast<size_t>(kMaxSlots) * 8);
  L.total = off;
  return L;
}

template <int VPT, bool ZP>
__global__ void __launch_bounds__(kThreads, VPT <= 2 ? 2 : 1)
    detect_quantize_compact_kernel(FusedArgs a, int S) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int K = a.K;
  const int words = (K + 31) >> 5;
  const int nv = K >> 3;
  const size_t row_bytes = static_cast<size_t>(K) * 2;
  const __half* __restrict__ X = a.X;
  const __half* __restrict__ W = a.W;
  int8_t* __restrict__ Xq = a.Xq;

  const FusedSmem L = fused_smem_layout(K, S);
  uint8_t* s_rows = fsm + L.rows;
  uint32_t* s_lbits = reinterpret_cast<uint32_t*>(fsm + L.lbits);
  uint32_t* s_gbits = reinterpret_cast<uint32_t*>(fsm + L.gbits);
  float* s_red = reinterpret_cast<float*>(fsm + L.red);        // [2 rounds][2][kWarps]
  int32_t* s_misc = reinterpret_cast<int32_t*>(fsm + L.misc);
  uint16_t* s_idx = reinterpret_cast<uint16_t*>(fsm + L.idx);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(fsm + L.bar);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int rows_per = (a.M + gridDim.x - 1) / gridDim.x;
  const int r0 = min(a.M, static_cast<int>(blockIdx.x) * rows_per);
  const int R = min(a.M, r0 + rows_per) - r0;

  // The GEMM that follows may launch now; it waits for this grid's completion
  // before reading anything written here.
  griddep_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&s_bar[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  bool ok = true;

  // ------------------------------------------------------------ pass A
  // Rows stream through S slots (row r in slot r % S); after a chunk of rows
  // every thread is done with their slots and the rows S further on are loaded
  // into them. Each thread waits for each row itself (one mbarrier per slot).
  {
    uint32_t par = 0;   // bit s: parity of the next completion of slot s
    auto issue = [&](int row) {   // thread 0 only
      uint64_t* bar = &s_bar[row % S];
      // Order earlier generic-proxy reads of the slot before the async-proxy write.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(row_bytes));
      bulk_load(s_rows + static_cast<size_t>(row % S) * row_bytes,
                X + static_cast<size_t>(r0 + row) * K, static_cast<uint32_t>(row_bytes), bar);
    };
    if (tid == 0)
      for (int r = 0; r < min(R, S); ++r) issue(r);
    __half2 cmax[VPT][4];
#pragma unroll
    for (int c = 0; c < VPT; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) cmax[c][i] = __float2half2_rn(0.0f);
    const int step = R <= S ? max(R, 1) : max(1, S / 2);
    for (int i0 = 0; i0 < R; i0 += step) {
      const int i1 = min(R, i0 + step);
      for (int r = i0; r < i1; ++r) {
        const int sl = r % S;
        if (ok && !mbar_wait(&s_bar[sl], (par >> sl) & 1u)) {
          ok = false;
          atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
        }
        par ^= 1u << sl;
        const uint4* row = reinterpret_cast<const uint4*>(s_rows + static_cast<size_t>(sl) * row_bytes);
#pragma unroll
        for (int c = 0; c < VPT; ++c) {
          const int v = tid + kThreads * c;
          if (v < nv) {
            const uint4 u = row[v];
            const uint32_t* wd = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
            for (int k = 0; k < 4; ++k) cmax[c][k] = __hmax2(cmax[c][k], habs2_bits(wd[k]));
          }
        }
      }
      if (i1 < R) {
        __syncthreads();
        if (tid == 0)
          for (int r = i0; r < i1; ++r)
            if (r + S < R) issue(r + S);
      }
    }
#pragma unroll
    for (int c = 0; c < VPT; ++c) {
      const int v = tid + kThreads * c;
      uint32_t flags = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 m = __half22float2(cmax[c][k]);
        flags |= (m.x > a.threshold ? 1u : 0u) << (2 * k);
        flags |= (m.y > a.threshold ? 1u : 0u) << (2 * k + 1);
      }
      uint32_t word = flags << (8 * (lane & 3));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      if ((lane & 3) == 0 && v < nv) {
        s_lbits[v >> 2] = word;
        if (word != 0) atomicOr(a.bitmap + (v >> 2), word);
      }
    }
    __syncthreads();
  }

  // ------------------------------------------------------------ pass B
  // After pass A the slots hold rows [R - nres, R) ("resident"); the others are
  // read again from global memory (L2) into registers.
  const int nres = min(R, S);
  int round = 0;   // selects the half of s_red a round of partial maxima uses

  // Row absmax over the non-outlier columns (zero-point codes: the largest x
  // and the largest -x, both at least 0 so that 0 stays inside the range),
  // reduced over the warp; non-negative floats order like their bit patterns.
  auto mask8 = [&](const uint32_t* mbits, int v) -> uint32_t {
    return (mbits[v >> 2] >> (8 * (v & 3))) & 0xFFu;
  };
  auto fold = [&](const uint4& u, uint32_t m8, __half2& h, __half2& g) {
    const uint32_t* wd = reinterpret_cast<const uint32_t*>(&u);
    if constexpr (!ZP) {
      if (m8 == 0u) {
#pragma unroll
        for (int k = 0; k < 4; ++k) h = __hmax2(h, habs2_bits(wd[k]));
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) h = __hmax2(h, habs2_bits(wd[k] & keep_half2(m8, k)));
      }
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t kw = wd[k] & keep_half2(m8, k);
        const uint32_t nw = kw ^ 0x80008000u;
        h = __hmax2(h, *reinterpret_cast<const __half2*>(&kw));
        g = __hmax2(g, *reinterpret_cast<const __half2*>(&nw));
      }
    }
  };
  auto warp_max = [&](__half2 h, __half2 g, float& hm, float& hn) {
    const float2 hf = __half22float2(h);
    hm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fmaxf(hf.x, hf.y), 0.0f))));
    hn = 0.0f;
    if constexpr (ZP) {
      const float2 gf = __half22float2(g);
      hn = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fmaxf(gf.x, gf.y), 0.0f))));
    }
  };
  // Per-row code parameters: absmax and 1/absmax, or step and zero point.
  struct RowQ {
    float am, ra;
    int z;
  };
  auto row_params = [&](int row, float hm, float hn, bool writer) -> RowQ {
    RowQ q{hm, 0.0f, 0};
    if constexpr (!ZP) {
      q.ra = quant_rcp(hm);
      if (writer) a.x_scale[r0 + row] = hm;
    } else {
      // hi = hm, lo = -hn; step = fl(fl(hi - lo) / 255); z = -128 - rint(lo / step)
      q.am = __fdiv_rn(__fadd_rn(hm, hn), 255.0f);
      if (q.am > 0.0f) q.z = max(-128, min(127, -128 - __float2int_rn(__fdiv_rn(-hn, q.am))));
      if (writer) {
        a.x_scale[r0 + row] = q.am;
        a.x_zero[r0 + row] = q.z;
      }
    }
    return q;
  };
  // Eight codes of vector u (0 at outlier columns; z for zero-point codes).
  auto code8 = [&](const uint4& u, uint32_t m8, const RowQ& q) -> uint2 {
    if constexpr (!ZP) {
      uint2 c = codes8(u, q.am, q.ra);
      if (m8) {
        c.x &= keep_bytes(m8 & 0xFu);
        c.y &= keep_bytes(m8 >> 4);
      }
      return c;
    } else {
      float f[8];
      unpack8(u, f);
      uint32_t b[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qv = 0;
        if ((m8 >> i) & 1u) {
          qv = q.z;
        } else if (q.am > 0.0f) {
          qv = max(-128, min(127, __float2int_rn(__fdiv_rn(f[i], q.am)) + q.z));
        }
        b[i >> 2] |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * (i & 3));
      }
      return make_uint2(b[0], b[1]);
    }
  };

  // Run by the kWorkers worker warps only (their barriers are named barrier 1).
  auto quantise = [&](const uint32_t* mbits) {
    // (1) resident rows, read from their slots: a team of T warps per row
    // (T a power of two, nres * T <= kWorkers), one barrier for the maxima.
    if (nres > 0) {
      int T = 1;
      while (nres * T * 2 <= kWorkers) T *= 2;
      const int seg = warp % T;
      if (T == 1) {
        for (int i = warp; i < nres; i += kWorkers) {
          const int row = R - nres + i;
          const uint4* src = reinterpret_cast<const uint4*>(s_rows + static_cast<size_t>(row % S) * row_bytes);
          __half2 h = __float2half2_rn(0.0f), g = h;
          for (int v = lane; v < nv; v += 32) fold(src[v], mask8(mbits, v), h, g);
          float hm, hn;
          warp_max(h, g, hm, hn);
          const RowQ q = row_params(row, hm, hn, lane == 0);
          uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(r0 + row) * K);
          for (int v = lane; v < nv; v += 32) dst[v] = code8(src[v], mask8(mbits, v), q);
        }
      } else {
        const int t = warp / T;
        const bool live = t < nres && (t + 1) * T <= kWorkers;
        const int row = R - nres + t;
        const uint4* src = reinterpret_cast<const uint4*>(s_rows + static_cast<size_t>((live ? row : 0) % S) * row_bytes);
        float* red = s_red + (round & 1) * 2 * kWarps;
        float hm = 0.0f, hn = 0.0f;
        if (live) {
          __half2 h = __float2half2_rn(0.0f), g = h;
          for (int v = seg * 32 + lane; v < nv; v += 32 * T) fold(src[v], mask8(mbits, v), h, g);
          warp_max(h, g, hm, hn);
          if (lane == 0) {
            red[warp] = hm;
            red[kWarps + warp] = hn;
          }
        }
        named_bar_sync(kWorkBar, 32 * kWorkers);
        ++round;
        if (live) {
          for (int k = 0; k < T; ++k) {
            hm = fmaxf(hm, red[t * T + k]);
            hn = fmaxf(hn, red[kWarps + t * T + k]);
          }
          const RowQ q = row_params(row, hm, hn, seg == 0 && lane == 0);
          uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(r0 + row) * K);
          for (int v = seg * 32 + lane; v < nv; v += 32 * T) dst[v] = code8(src[v], mask8(mbits, v), q);
        }
      }
    }
    // (2) the other rows, from global memory: rounds of kWorkers/TB rows, a
    // team of TB warps per row, each lane keeping its VL vectors in registers.
    constexpr int TB = VPT <= 2 ? 5 : kWorkers;
    constexpr int VL = (kThreads * VPT + 32 * TB - 1) / (32 * TB);
    constexpr int RPR = kWorkers / TB;
    const int nstream = R - nres;
    const int t = warp / TB;
    const int lt = (warp % TB) * 32 + lane;
    for (int b0 = 0; b0 < nstream; b0 += RPR) {
      const int row = b0 + t;
      const bool live = row < nstream && t < RPR;
      const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<size_t>(r0 + (live ? row : 0)) * K);
      uint4 val[VL];
      __half2 h = __float2half2_rn(0.0f), g = h;
#pragma unroll
      for (int c = 0; c < VL; ++c) {
        const int v = lt + 32 * TB * c;
        val[c] = (live && v < nv) ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int c = 0; c < VL; ++c) {
        const int v = lt + 32 * TB * c;
        if (v < nv) fold(val[c], mask8(mbits, v), h, g);
      }
      float hm, hn;
      warp_max(h, g, hm, hn);
      float* red = s_red + (round & 1) * 2 * kWarps;
      if (lane == 0) {
        red[warp] = hm;
        red[kWarps + warp] = hn;
      }
      named_bar_sync(kWorkBar, 32 * kWorkers);
      ++round;
      if (live) {
        for (int k = 0; k < TB; ++k) {
          hm = fmaxf(hm, red[t * TB + k]);
          hn = fmaxf(hn, red[kWarps + t * TB + k]);
        }
        const RowQ q = row_params(row, hm, hn, lt == 0);
        uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(r0 + row) * K);
#pragma unroll
        for (int c = 0; c < VL; ++c) {
          const int v = lt + 32 * TB * c;
          if (v < nv) dst[v] = code8(val[c], mask8(mbits, v), q);
        }
      }
    }
  };

  // ------------------------------------------------------------ list (control warp)
  // Warp `cw` builds the ascending list of a bitmap and its count (lane l
  // scans a contiguous run of words); its readers synchronise with it.
  auto build_list = [&](const uint32_t* bits) {
    const int lper = (words + 31) >> 5;
    const int lw0 = min(words, lane * lper), lw1 = min(words, lw0 + lper);
    int cnt = 0;
    for (int w = lw0; w < lw1; ++w) cnt += __popc(bits[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tt = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += tt;
    }
    int p = incl - cnt;
    for (int w = lw0; w < lw1; ++w) {
      uint32_t b = bits[w];
      while (b) {
        const int j = __ffs(b) - 1;
        b &= b - 1;
        s_idx[p++] = static_cast<uint16_t>(w * 32 + j);
      }
    }
    if (lane == 31) s_misc[0] = incl;
  };

  // ------------------------------------------------------------ panels
  // The CTA's rows of the compacted fp16 panels for the list in s_idx, a
  // multiple of 64 columns wide and zero-padded: X_O (from the slots or L2)
  // and W_O (gathered from Wt). Run by the threads [t0, t0 + nt).
  const int nper = (a.N + gridDim.x - 1) / gridDim.x;
  const int wn0 = min(a.N, static_cast<int>(blockIdx.x) * nper);
  const int wn1 = min(a.N, wn0 + nper);
  auto panels = [&](int count, int t0, int nt) {
    if (count == 0) return;
    const int pw = (count + 63) & ~63;
    for (int e = tid - t0; e < R * pw; e += nt) {
      const int row = e / pw;
      const int p = e - row * pw;
      __half v = __float2half_rn(0.0f);
      if (p < count) {
        v = (row >= R - nres)
                ? reinterpret_cast<const __half*>(s_rows + static_cast<size_t>(row % S) * row_bytes)[s_idx[p]]
                : X[static_cast<size_t>(r0 + row) * K + s_idx[p]];
      }
      a.X_O[static_cast<size_t>(r0 + row) * a.ld + p] = v;
    }
    const int chunks = pw >> 3;
    const int items = (wn1 - wn0) * chunks;
    // One item = 8 consecutive panel columns of one weight row n, read from the
    // rows idx[p] of Wt ([K][N]); consecutive items are consecutive n, so the
    // loads are coalesced across a warp. One 16-byte store.
    const int nr = wn1 - wn0;
    for (int it = tid - t0; it < items; it += nt) {
      const int ch = it / nr;
      const int n = wn0 + (it - ch * nr);
      const __half* wcol = W + n;
      uint4 o;
      __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int p = ch * 8 + i;
        h[i] = (p < count) ? wcol[static_cast<size_t>(s_idx[p]) * a.N] : __float2half_rn(0.0f);
      }
      reinterpret_cast<uint4*>(a.W_O + static_cast<size_t>(n) * a.ld)[ch] = o;
    }
  };

  if (warp < kWorkers) {
    quantise(s_lbits);
    // The panels with the CTA's own list (the batch's, unless the check below
    // finds a column the CTA's rows missed), while the control warp waits.
    named_bar_sync(kListBar, kThreads);
    panels(s_misc[0], 0, 32 * kWorkers);
  } else {
    // Control warp: arrive at the grid barrier, build this CTA's list (the
    // batch's list unless the check below finds a column it lacks), wait at the
    // barrier, then read the batch's bitmap and compare.
    if (lane == 0) {
      __threadfence();
      atomicAdd(a.sync_ctr, 1);
    }
    __syncwarp();
    build_list(s_lbits);
    __syncwarp();
    named_bar_arrive(kListBar, kThreads);
    int extra = 0;
    {
      if (lane == 0) {
        const uint64_t t0 = gtimer();
        while (ld_acquire(a.sync_ctr) < static_cast<int>(gridDim.x)) {
          __nanosleep(64);
          if (gtimer() - t0 > kBarrierLimitNs) {
            atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
            break;
          }
        }
        __threadfence();
      }
      __syncwarp();
      for (int w = lane; w < words; w += 32) {
        const uint32_t g = __ldcg(a.bitmap + w);
        s_gbits[w] = g;
        extra |= (g & ~s_lbits[w]) != 0u;
      }
      extra = __any_sync(0xffffffffu, extra);
    }
    if (lane == 0) s_misc[1] = extra;
  }
  __syncthreads();
  if (s_misc[1]) {
    // This CTA's rows missed an outlier column of the batch: codes, list and
    // panels again with the batch's set.
    if (warp < kWorkers)
      quantise(s_gbits);
    else
      build_list(s_gbits);
    __syncthreads();
    panels(s_misc[0], 0, kThreads);
  }
  const int count = s_misc[0];
  if (blockIdx.x == 0) {
    for (int p = tid; p < count; p += kThreads) a.col_idx[p] = s_idx[p];
    if (tid == 0) *a.n_outliers = count;
  }
  (void)ok;
}

int fused_vpt(int K) {
  const int nv = K / 8;
  if (nv <= kThreads) return 1;
  if (nv <= 2 * kThreads) return 2;
  if (nv <= 4 * kThreads) return 4;
  if (nv <= 8 * kThreads) return 8;
  return 16;
}

cudaError_t launch_detect_quantize_compact(const FusedArgs& a, cudaStream_t s) {
  // Absmax codes (with detection or a given set): the single-pass kernel of
  // stream_quant.cu. This kernel serves the zero-point codes with detection.
  if (a.x_zero == nullptr) return launch_detect_quantize_stream(a, s);
  if (a.given != nullptr) return cudaErrorInvalidValue;
  const int vpt = fused_vpt(a.K);
  const void* fn = nullptr;
  switch (vpt) {
    case 1: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<1, true>); break;
    case 2: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<2, true>); break;
    case 4: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<4, true>); break;
    case 8: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<8, true>); break;
    default: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<16, true>); break;
  }
  // Row slots: about 110 KB when two CTAs share an SM (vpt <= 2), 220 KB otherwise.
  const size_t row_bytes = static_cast<size_t>(a.K) * 2;
  const size_t budget = (vpt <= 2 ? 110u : 220u) * 1024u;
  const size_t fixed = fused_smem_layout(a.K, 0).total;
  int S = static_cast<int>((budget > fixed ? budget - fixed : 0) / row_bytes);
  S = max(1, min(S, kMaxSlots));
  const size_t smem = fused_smem_layout(a.K, S).total;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0, sms = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // Enough CTAs to keep every SM streaming, but not more than can be co-resident.
  int grid = per_sm * sms;
  const int want = max((a.M + 1) / 2, (a.N + 15) / 16);
  grid = max(1, min(grid, want));
  FusedArgs args = a;
  void* params[] = {&args, &S};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), params, smem, s);
}

}  // namespace i8mm

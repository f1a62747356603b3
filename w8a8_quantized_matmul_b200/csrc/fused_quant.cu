// Fused detection + quantisation + compaction for the full LLM.int8() path,
// one cooperative launch (all CTAs co-resident).
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier feature dimensions by a magnitude threshold, vector-wise absmax INT8
// quantisation of the remaining dimensions, the outlier dimensions kept in
// fp16); tanjunchen "quantization explained part 2", section 1.2 (threshold 6.0;
// once the outlier dimension is split out the scale comes from the rest).
//
// Each CTA owns a contiguous block of rows of X and a contiguous block of rows
// of W. Thread t of the 512 owns the 16-byte vectors v = t + 512*c (c < VPT)
// of every row it touches, i.e. the same 8*VPT columns in every row.
//   phase A  stream the CTA's rows of X once from HBM, keeping a packed-fp16
//            running max of |x| per owned column; compare the column maxima
//            with the threshold once and OR the flags into the global bitmap
//            (atomics only for non-zero words)
//   barrier  grid-wide arrival counter with a bounded wait
//   phase B  bitmap -> per-word prefix counts and the ascending outlier list in
//            shared memory (CTA 0 also publishes the count and the list); re-read
//            the rows (now L2-resident): per-row absmax over the non-outlier
//            columns in packed fp16, INT8 codes with paired fp32 arithmetic; the
//            outlier columns of the rows are compacted into the fp16 panel X_O,
//            and those of the CTA's W rows gathered into W_O. The panels are
//            kCcMaxOutliers columns wide (zero-padded) when the GEMM epilogue adds
//            the outlier product, or a multiple of 64 wide when the GEMM
//            multiplies them on the tensor cores.
//
// The code of x is rint(fl32(fl32(x*127)/a)) clamped to +-127. The correctly
// rounded quotient is formed without a division (codes8 in quant_common.cuh:
// the FMA-corrected product with fl(1/a), exact for every pair of fp16 values
// with |x| <= a) and rounded with the 1.5*2^23 trick (ties to even in one add;
// the code lands in the low byte).
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
constexpr int kMaxGroup = 16;                 // rows per reduction group (and per wave)
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
//   rows    [nb][K] fp16       the rows of the current wave, filled by bulk copies
//   bits    [words] u32        outlier bitmap
//   prefix  [words] i32        outliers before each bitmap word
//   red     [2*kWarps+3][kMaxGroup] f32 per-warp row maxima (and, for zero-point codes,
//                                      of -x); then row absmax or step, 1/absmax, zero point
//   misc    [4] i32            running count during the scan
//   idx     [K] u16            ascending outlier columns
//   bar     u64                mbarrier of the bulk copies
struct FusedSmem {
  size_t rows, bits, prefix, red, misc, idx, bar, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

__host__ __device__ inline FusedSmem fused_smem_layout(int K, int nb) {
  FusedSmem L;
  const size_t words = static_cast<size_t>((K + 31) / 32);
  size_t off = 0;
  L.rows = off;   off = align16(off + static_cast<size_t>(nb) * K * 2);
  L.bits = off;   off = align16(off + words * 4);
  L.prefix = off; off = align16(off + words * 4);
  L.red = off;    off = align16(off + static_cast<size_t>(2 * kWarps + 3) * kMaxGroup * 4);
  L.misc = off;   off = align16(off + 16);
  L.idx = off;    off = align16(off + static_cast<size_t>(K) * 2);
  L.bar = off;    off = align16(off + 8);
  L.total = off;
  return L;
}

template <int VPT, bool ZP>
__global__ void __launch_bounds__(kThreads, VPT == 1 ? 2 : 1)
    detect_quantize_compact_kernel(FusedArgs a, int nb) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int K = a.K;
  const int words = (K + 31) >> 5;
  const int nv = K >> 3;
  const size_t row_bytes = static_cast<size_t>(K) * 2;
  const __half* __restrict__ X = a.X;
  const __half* __restrict__ W = a.W;
  int8_t* __restrict__ Xq = a.Xq;
  __half* __restrict__ X_O = a.X_O;
  __half* __restrict__ W_O = a.W_O;

  const FusedSmem L = fused_smem_layout(K, nb);
  uint8_t* s_rows = fsm + L.rows;
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(fsm + L.bits);
  int32_t* s_prefix = reinterpret_cast<int32_t*>(fsm + L.prefix);
  float* s_red = reinterpret_cast<float*>(fsm + L.red);
  float* s_row = s_red + kWarps * kMaxGroup;
  float* s_rcp = s_row + kMaxGroup;
  float* s_nred = s_rcp + kMaxGroup;                      // [kWarps][kMaxGroup] max of -x
  int32_t* s_zero = reinterpret_cast<int32_t*>(s_nred + kWarps * kMaxGroup);
  constexpr bool zp = ZP;   // zero-point codes
  int32_t* s_misc = reinterpret_cast<int32_t*>(fsm + L.misc);
  uint16_t* s_idx = reinterpret_cast<uint16_t*>(fsm + L.idx);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(fsm + L.bar);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int rows_per = (a.M + gridDim.x - 1) / gridDim.x;
  const int r0 = min(a.M, static_cast<int>(blockIdx.x) * rows_per);
  const int r1 = min(a.M, r0 + rows_per);
  const int R = r1 - r0;
  // Waves of at most nb rows, as equal as possible; the last one stays resident.
  const int nwaves = (R + nb - 1) / nb;
  const int wave_rows = nwaves ? (R + nwaves - 1) / nwaves : 0;

  // The GEMM that follows may launch now; it waits for this grid's completion
  // before reading anything written here.
  griddep_launch_dependents();
  if (tid == 0) {
    mbar_init(s_bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  uint32_t parity = 0;
  bool ok = true;

  // Bulk-copies the rows of wave w into the row buffer and waits for them.
  auto fetch = [&](int w) -> int {
    const int wb = r0 + w * wave_rows;
    const int n = min(wave_rows, r1 - wb);
    if (tid == 0) {
      // Order earlier generic-proxy reads of the buffer before the async-proxy writes.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(s_bar, static_cast<uint32_t>(n * row_bytes));
      for (int g = 0; g < n; ++g)
        bulk_load(s_rows + g * row_bytes, X + static_cast<size_t>(wb + g) * K,
                  static_cast<uint32_t>(row_bytes), s_bar);
    }
    if (!mbar_wait(s_bar, parity)) {
      ok = false;
      if (tid == 0) atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
    }
    parity ^= 1u;
    return n;
  };

  // ---------------- phase A: per-column max |x| over this CTA's rows
  __half2 cmax[VPT][4];
#pragma unroll
  for (int c = 0; c < VPT; ++c)
#pragma unroll
    for (int i = 0; i < 4; ++i) cmax[c][i] = __float2half2_rn(0.0f);
  const bool given = a.given != nullptr;   // outlier set supplied (token-sharded mode)
  for (int w = 0; w < nwaves; ++w) {
    if (w > 0) __syncthreads();   // everyone is done with the previous wave
    const int n = fetch(w);
    if (given) continue;
    for (int g = 0; g < n; ++g) {
      const uint4* srow = reinterpret_cast<const uint4*>(s_rows + g * row_bytes);
#pragma unroll
      for (int c = 0; c < VPT; ++c) {
        const int v = tid + kThreads * c;
        if (v < nv) {
          const uint4 u = srow[v];
          const uint32_t* wd = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
          for (int i = 0; i < 4; ++i) cmax[c][i] = __hmax2(cmax[c][i], habs2_bits(wd[i]));
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    const int v = tid + kThreads * c;
    uint32_t flags = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 m = __half22float2(cmax[c][i]);
      flags |= (m.x > a.threshold ? 1u : 0u) << (2 * i);
      flags |= (m.y > a.threshold ? 1u : 0u) << (2 * i + 1);
    }
    uint32_t word = flags << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if (!given && (lane & 3) == 0 && v < nv && word != 0) atomicOr(a.bitmap + (v >> 2), word);
  }

  // ---------------- grid barrier (bounded); not needed when the set is given
  __syncthreads();
  if (tid == 0 && !given) {
    __threadfence();
    atomicAdd(a.sync_ctr, 1);
    const uint64_t t0 = gtimer();
    while (ld_acquire(a.sync_ctr) < static_cast<int>(gridDim.x)) {
      __nanosleep(32);
      if (gtimer() - t0 > kBarrierLimitNs) {
        atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();

  // ---------------- phase B.1: outlier masks of this thread's columns (the same
  // for every row), straight from the global bitmap. Warp 0 also builds the
  // per-word prefix counts and the ascending outlier list in shared memory; the
  // other warps start on the row maxima meanwhile.
  // Word w of the outlier bitmap: the global bitmap, or the OR of the given ones.
  auto bitmap_word = [&](int w) -> uint32_t {
    if (!given) return __ldcg(a.bitmap + w);
    uint32_t b = 0;
    for (int r = 0; r < a.given_n; ++r) b |= __ldg(a.given + static_cast<size_t>(r) * words + w);
    return b;
  };
  uint32_t m8[VPT];
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    const int v = tid + kThreads * c;
    m8[c] = (v < nv) ? (bitmap_word(v >> 2) >> (8 * (v & 3))) & 0xFFu : 0u;
  }
  // Warp 0 also builds the per-word prefix counts and the ascending outlier
  // list in shared memory (build_list); its bitmap words are copied to shared
  // memory now (cp.async: no registers held) so that their L2 round trip
  // overlaps the row maxima below.
  const int lper = (words + 31) >> 5;                  // words per lane
  const int lw0 = min(words, lane * lper), lw1 = min(words, lw0 + lper);
  if (warp == 0 && !given) {
    for (int w = lw0; w < lw1; ++w)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(s_bits + w)),
                   "l"(a.bitmap + w)
                   : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  bool listed = false;
  auto build_list = [&]() {
    // Lane l scans the words [lw0, lw1).
    int cnt = 0;
    if (!given) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      for (int w = lw0; w < lw1; ++w) cnt += __popc(s_bits[w]);
    } else {
      for (int w = lw0; w < lw1; ++w) {
        const uint32_t b = bitmap_word(w);
        s_bits[w] = b;
        cnt += __popc(b);
      }
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int p = incl - cnt;
    for (int w = lw0; w < lw1; ++w) {
      uint32_t b = s_bits[w];
      s_prefix[w] = p;
      while (b) {
        const int j = __ffs(b) - 1;
        b &= b - 1;
        s_idx[p++] = static_cast<uint16_t>(w * 32 + j);
      }
    }
    if (lane == 31) s_misc[0] = incl;
    if (given && blockIdx.x == 0)
      for (int w = lw0; w < lw1; ++w) a.bitmap[w] = s_bits[w];
  };

  // ---------------- phase B.2: quantise, the resident wave first, then re-fetch the rest
  int count = -1, pw = 0;
  bool compact = false;
  int items = 0, wn0 = 0, chunks = 0;
  constexpr int kEarly = 2;   // W_O items per thread gathered before the quantisation
  __half early[kEarly][8];    // kept as halves: packed only when stored, after the codes
  // Panel geometry, the published list and the early W_O gathers, once the
  // outlier list is complete (warp 0 wrote it before the first group barrier).
  // The early gathers' latency overlaps the quantisation; their stores follow it.
  auto setup_panels = [&]() {
    count = s_misc[0];
    compact = count > 0;
    // Compacted fp16 outlier panels: kCcMaxOutliers columns wide (zero-padded)
    // when the GEMM epilogue adds the outlier product itself, a multiple of 64
    // wide when the GEMM multiplies the panels on the tensor cores.
    pw = count > kCcMaxOutliers ? ((count + 63) & ~63) : kCcMaxOutliers;
    if (blockIdx.x == 0) {
      for (int p = tid; p < count; p += kThreads) a.col_idx[p] = s_idx[p];
      if (tid == 0) *a.n_outliers = count;
    }
    const int nper = (a.N + gridDim.x - 1) / gridDim.x;
    wn0 = min(a.N, static_cast<int>(blockIdx.x) * nper);
    const int wn1 = min(a.N, wn0 + nper);
    chunks = pw >> 3;
    items = compact ? (wn1 - wn0) * chunks : 0;
#pragma unroll
    for (int e = 0; e < kEarly; ++e) {
      const int it = tid + e * kThreads;
      const bool live = it < items;
      const int n2 = live ? wn0 + it / chunks : wn0;
      const int ch = live ? it - (n2 - wn0) * chunks : 0;
      const __half* wrow = W + static_cast<size_t>(n2) * K;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int pidx = ch * 8 + i;
        early[e][i] = (live && pidx < count) ? wrow[s_idx[pidx]] : __float2half_rn(0.0f);
      }
    }
  };

  for (int k = 0; k < nwaves; ++k) {
    const int w = (k == 0) ? nwaves - 1 : k - 1;
    const int wb = r0 + w * wave_rows;
    int n = min(wave_rows, r1 - wb);
    if (k > 0) {
      __syncthreads();
      n = fetch(w);
    }
    for (int gb = 0; gb < n; gb += kMaxGroup) {
      const int ng = min(kMaxGroup, n - gb);
      // Row absmax over the non-outlier columns: per thread, then per warp with
      // one redux (non-negative floats order like their bit patterns). Zero-point
      // codes need the largest x and the largest -x instead (both >= 0 with the
      // outlier columns zeroed, which keeps 0 inside the range).
#pragma unroll 1
      for (int g = 0; g < ng; ++g) {
        const uint4* srow = reinterpret_cast<const uint4*>(s_rows + (gb + g) * row_bytes);
        __half2 h = __float2half2_rn(0.0f), hn = h;
#pragma unroll
        for (int c = 0; c < VPT; ++c) {
          const int v = tid + kThreads * c;
          if (v < nv) {
            const uint4 u = srow[v];
            const uint32_t* wd = reinterpret_cast<const uint32_t*>(&u);
            if constexpr (!zp) {
              if (m8[c] == 0u) {
#pragma unroll
                for (int i = 0; i < 4; ++i) h = __hmax2(h, habs2_bits(wd[i]));
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) h = __hmax2(h, habs2_bits(wd[i] & keep_half2(m8[c], i)));
              }
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t kw = wd[i] & keep_half2(m8[c], i);
                const uint32_t nw = kw ^ 0x80008000u;
                h = __hmax2(h, *reinterpret_cast<const __half2*>(&kw));
                hn = __hmax2(hn, *reinterpret_cast<const __half2*>(&nw));
              }
            }
          }
        }
        const float2 hf = __half22float2(h);
        if constexpr (!zp) {
          const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(hf.x, hf.y)));
          if (lane == 0) s_red[warp * kMaxGroup + g] = __uint_as_float(mx);
        } else {
          // x and -x may be negative: clamp at 0 (0 stays inside the range)
          const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fmaxf(hf.x, hf.y), 0.0f)));
          if (lane == 0) s_red[warp * kMaxGroup + g] = __uint_as_float(mx);
          const float2 nf = __half22float2(hn);
          const uint32_t mn = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fmaxf(nf.x, nf.y), 0.0f)));
          if (lane == 0) s_nred[warp * kMaxGroup + g] = __uint_as_float(mn);
        }
      }
      if (warp == 0 && !listed) build_list();
      listed = true;
      __syncthreads();
      if (tid < ng) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, s_red[i * kMaxGroup + tid]);
        if constexpr (!zp) {
          s_row[tid] = m;
          s_rcp[tid] = quant_rcp(m);
          a.x_scale[wb + gb + tid] = m;
        } else {
          // hi = m, lo = -nlo; step = fl(fl(hi - lo) / 255); z = -128 - rint(lo / step)
          float nlo = 0.0f;
#pragma unroll
          for (int i = 0; i < kWarps; ++i) nlo = fmaxf(nlo, s_nred[i * kMaxGroup + tid]);
          const float step = __fdiv_rn(__fadd_rn(m, nlo), 255.0f);
          int z = 0;
          if (step > 0.0f) z = max(-128, min(127, -128 - __float2int_rn(__fdiv_rn(-nlo, step))));
          s_row[tid] = step;
          s_zero[tid] = z;
          a.x_scale[wb + gb + tid] = step;
          a.x_zero[wb + gb + tid] = z;
        }
      }
      __syncthreads();
      if (count < 0) setup_panels();
      // Codes of the group's rows (0 at the outlier columns).
#pragma unroll 1
      for (int g = 0; g < ng; ++g) {
        const int row = wb + gb + g;
        const float am = s_row[g];
        const float ra = s_rcp[g];
        const uint4* srow = reinterpret_cast<const uint4*>(s_rows + (gb + g) * row_bytes);
        uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(row) * K);
        if constexpr (zp) {
          // q = clamp(rint(x / step) + z, -128, 127); z at the outlier columns
          const int z = s_zero[g];
#pragma unroll
          for (int c = 0; c < VPT; ++c) {
            const int v = tid + kThreads * c;
            if (v < nv) {
              float f[8];
              unpack8(srow[v], f);
              uint32_t b[2] = {0u, 0u};
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                int qv = 0;
                if ((m8[c] >> i) & 1u) {
                  qv = z;
                } else if (am > 0.0f) {
                  qv = max(-128, min(127, __float2int_rn(__fdiv_rn(f[i], am)) + z));
                }
                b[i >> 2] |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * (i & 3));
              }
              dst[v] = make_uint2(b[0], b[1]);
            }
          }
          continue;
        }
#pragma unroll
        for (int c = 0; c < VPT; ++c) {
          const int v = tid + kThreads * c;
          if (v < nv) {
            uint2 q = codes8(srow[v], am, ra);
            if (m8[c]) {
              q.x &= keep_bytes(m8[c] & 0xFu);
              q.y &= keep_bytes(m8[c] >> 4);
            }
            dst[v] = q;
          }
        }
      }
      // The group's rows of the compacted panel X_O (outlier columns, then zeros).
      if (compact) {
        for (int e = tid; e < ng * pw; e += kThreads) {
          const int g = e / pw;
          const int p2 = e - g * pw;
          const __half* hrow = reinterpret_cast<const __half*>(s_rows + (gb + g) * row_bytes);
          X_O[static_cast<size_t>(wb + gb + g) * a.ld + p2] =
              (p2 < count) ? hrow[s_idx[p2]] : __float2half_rn(0.0f);
        }
      }
      __syncthreads();   // s_red / s_row / s_rcp are reused by the next group
    }
  }

  if (count < 0) {   // no rows of X here: the W_O rows are still this CTA's
    if (warp == 0) build_list();
    __syncthreads();
    setup_panels();
  }

  // ---------------- phase B.3: W_O rows of this CTA (outlier columns of W)
  // One thread per 8-column chunk of a row: up to 8 independent gathers, one
  // 16-byte store; the first kEarly*kThreads items were gathered before B.2.
#pragma unroll
  for (int k = 0; k < kEarly; ++k) {
    const int it = tid + k * kThreads;
    if (it < items) {
      const int n = wn0 + it / chunks;
      const int ch = it - (n - wn0) * chunks;
      uint4 o;
      __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = early[k][i];
      reinterpret_cast<uint4*>(W_O + static_cast<size_t>(n) * a.ld)[ch] = o;
    }
  }
  for (int it = tid + kEarly * kThreads; it < items; it += kThreads) {
    const int n = wn0 + it / chunks;
    const int ch = it - (n - wn0) * chunks;
    const __half* wrow = W + static_cast<size_t>(n) * K;
    uint4 o;
    __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int pidx = ch * 8 + i;
      h[i] = (pidx < count) ? wrow[s_idx[pidx]] : __float2half_rn(0.0f);
    }
    reinterpret_cast<uint4*>(W_O + static_cast<size_t>(n) * a.ld)[ch] = o;
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
  const int vpt = fused_vpt(a.K);
  const void* fn = nullptr;
  const bool zp = a.x_zero != nullptr;
  switch (vpt) {
    case 1: fn = zp ? reinterpret_cast<const void*>(detect_quantize_compact_kernel<1, true>)
                    : reinterpret_cast<const void*>(detect_quantize_compact_kernel<1, false>); break;
    case 2: fn = zp ? reinterpret_cast<const void*>(detect_quantize_compact_kernel<2, true>)
                    : reinterpret_cast<const void*>(detect_quantize_compact_kernel<2, false>); break;
    case 4: fn = zp ? reinterpret_cast<const void*>(detect_quantize_compact_kernel<4, true>)
                    : reinterpret_cast<const void*>(detect_quantize_compact_kernel<4, false>); break;
    case 8: fn = zp ? reinterpret_cast<const void*>(detect_quantize_compact_kernel<8, true>)
                    : reinterpret_cast<const void*>(detect_quantize_compact_kernel<8, false>); break;
    default: fn = zp ? reinterpret_cast<const void*>(detect_quantize_compact_kernel<16, true>)
                     : reinterpret_cast<const void*>(detect_quantize_compact_kernel<16, false>); break;
  }
  // Row buffer: ~96 KB when two CTAs share an SM (vpt 1), ~180 KB otherwise.
  const size_t row_bytes = static_cast<size_t>(a.K) * 2;
  const size_t budget = (vpt == 1 ? 96u : 180u) * 1024u;
  const size_t fixed = fused_smem_layout(a.K, 0).total;
  int nb = static_cast<int>((budget > fixed ? budget - fixed : 0) / row_bytes);
  nb = max(1, min(nb, kMaxGroup));
  const size_t smem = fused_smem_layout(a.K, nb).total;
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
  void* params[] = {&args, &nb};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), params, smem, s);
}

}  // namespace i8mm

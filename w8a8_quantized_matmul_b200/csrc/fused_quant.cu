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
// The code of x is rint(fl32(fl32(x*127)/a)) clamped to +-127. It is computed as
// y = fl32(x * fl32(127/a)) rounded with the 1.5*2^23 trick (round to nearest
// even in one add; the code lands in the low byte). y is within 2.3e-5 of the
// correctly rounded quotient, so the two round alike unless y lies within
// 6.2e-5 of a half-integer; such vectors are recomputed with the division.
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
//   red     [kWarps+1][kMaxGroup] f32   per-warp row maxima; last line = row absmax
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
  L.red = off;    off = align16(off + static_cast<size_t>(kWarps + 1) * kMaxGroup * 4);
  L.misc = off;   off = align16(off + 16);
  L.idx = off;    off = align16(off + static_cast<size_t>(K) * 2);
  L.bar = off;    off = align16(off + 8);
  L.total = off;
  return L;
}

template <int VPT>
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
  for (int w = 0; w < nwaves; ++w) {
    if (w > 0) __syncthreads();   // everyone is done with the previous wave
    const int n = fetch(w);
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
    if ((lane & 3) == 0 && v < nv && word != 0) atomicOr(a.bitmap + (v >> 2), word);
  }

  // ---------------- grid barrier (bounded)
  __syncthreads();
  if (tid == 0) {
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

  // ---------------- phase B.1: bitmap, prefix counts and outlier list in shared memory
  if (tid == 0) s_misc[0] = 0;
  __syncthreads();
  for (int base = 0; base < words; base += kThreads) {
    const int w = base + tid;
    const uint32_t bits = (w < words) ? __ldcg(a.bitmap + w) : 0u;
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_red[warp] = __int_as_float(incl);
    __syncthreads();
    int wsum = 0;
    for (int i = 0; i < warp; ++i) wsum += __float_as_int(s_red[i]);
    const int excl = s_misc[0] + wsum + incl - cnt;
    if (w < words) {
      s_bits[w] = bits;
      s_prefix[w] = excl;
      uint32_t b = bits;
      int p = excl;
      while (b) {
        const int j = __ffs(b) - 1;
        b &= b - 1;
        s_idx[p++] = static_cast<uint16_t>(w * 32 + j);
      }
    }
    __syncthreads();
    if (tid == kThreads - 1) s_misc[0] = excl + cnt;
    __syncthreads();
  }
  const int count = s_misc[0];
  const int pad = (count + 63) & ~63;
  if (blockIdx.x == 0) {
    for (int p = tid; p < count; p += kThreads) a.col_idx[p] = s_idx[p];
    if (tid == 0) *a.n_outliers = count;
  }
  // Compacted fp16 outlier panels: kCcMaxOutliers columns wide (zero-padded) when
  // the GEMM epilogue adds the outlier product itself, a multiple of 64 wide when
  // the GEMM multiplies the panels on the tensor cores.
  const bool compact = count > 0;
  const int pw = count > kCcMaxOutliers ? pad : kCcMaxOutliers;

  // Outlier masks of this thread's columns (the same for every row).
  uint32_t m8[VPT];
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    const int v = tid + kThreads * c;
    m8[c] = (v < nv) ? (s_bits[v >> 2] >> (8 * (v & 3))) & 0xFFu : 0u;
  }

  // W_O gather items of this CTA (row n, 8-column chunk): the loads are issued
  // now so that their latency overlaps the quantisation below; the stores follow it.
  const int nper = (a.N + gridDim.x - 1) / gridDim.x;
  const int wn0 = min(a.N, static_cast<int>(blockIdx.x) * nper);
  const int wn1 = min(a.N, wn0 + nper);
  const int chunks = pw >> 3;
  const int items = compact ? (wn1 - wn0) * chunks : 0;
  constexpr int kEarly = 2;   // items per thread gathered before the quantisation
  uint4 early[kEarly];
#pragma unroll
  for (int k = 0; k < kEarly; ++k) {
    const int it = tid + k * kThreads;
    early[k] = make_uint4(0, 0, 0, 0);
    if (it < items) {
      const int n = wn0 + it / chunks;
      const int ch = it - (n - wn0) * chunks;
      const __half* wrow = W + static_cast<size_t>(n) * K;
      __half* h = reinterpret_cast<__half*>(&early[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int pidx = ch * 8 + i;
        h[i] = (pidx < count) ? wrow[s_idx[pidx]] : __float2half_rn(0.0f);
      }
    }
  }

  // ---------------- phase B.2: quantise, the resident wave first, then re-fetch the rest
  for (int k = 0; k < nwaves; ++k) {
    const int w = (k == 0) ? nwaves - 1 : k - 1;
    const int wb = r0 + w * wave_rows;
    int n = min(wave_rows, r1 - wb);
    if (k > 0) {
      __syncthreads();
      n = fetch(w);
    }
    // Row absmax over the non-outlier columns, for up to kMaxGroup rows at once.
    for (int gb = 0; gb < n; gb += kMaxGroup) {
      const int ng = min(kMaxGroup, n - gb);
      float part[kMaxGroup];
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) {
        part[g] = 0.0f;
        if (g < ng) {
          const uint4* srow = reinterpret_cast<const uint4*>(s_rows + (gb + g) * row_bytes);
          __half2 h = __float2half2_rn(0.0f);
#pragma unroll
          for (int c = 0; c < VPT; ++c) {
            const int v = tid + kThreads * c;
            if (v < nv) {
              const uint4 u = srow[v];
              const uint32_t* wd = reinterpret_cast<const uint32_t*>(&u);
              if (m8[c] == 0u) {
#pragma unroll
                for (int i = 0; i < 4; ++i) h = __hmax2(h, habs2_bits(wd[i]));
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) h = __hmax2(h, habs2_bits(wd[i] & keep_half2(m8[c], i)));
              }
            }
          }
          const float2 hf = __half22float2(h);
          part[g] = fmaxf(hf.x, hf.y);
        }
      }
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) {
        if (g < ng) {
          const float m = warp_max(part[g]);
          if (lane == 0) s_red[warp * kMaxGroup + g] = m;
        }
      }
      __syncthreads();
      if (tid < ng) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, s_red[i * kMaxGroup + tid]);
        s_row[tid] = m;
      }
      __syncthreads();
      for (int g = 0; g < ng; ++g) {
        const int row = wb + gb + g;
        const float am = s_row[g];
        const float inv = quant_inv(am);
        const uint4* srow = reinterpret_cast<const uint4*>(s_rows + (gb + g) * row_bytes);
        uint2* dst = reinterpret_cast<uint2*>(Xq + static_cast<size_t>(row) * K);
        __half* xo_row = X_O + static_cast<size_t>(row) * a.ld;
#pragma unroll
        for (int c = 0; c < VPT; ++c) {
          const int v = tid + kThreads * c;
          if (v < nv) {
            const uint4 u = srow[v];
            uint2 q = codes8(u, am, inv);
            if (m8[c]) {
              q.x &= keep_bytes(m8[c] & 0xFu);
              q.y &= keep_bytes(m8[c] >> 4);
              if (compact) {
                const uint32_t wbits = s_bits[v >> 2];
                const int base = s_prefix[v >> 2];
                const __half* hv = reinterpret_cast<const __half*>(&u);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  if ((m8[c] >> i) & 1u) {
                    const int bit = 8 * (v & 3) + i;
                    xo_row[base + __popc(wbits & ((1u << bit) - 1u))] = hv[i];
                  }
                }
              }
            }
            dst[v] = q;
          }
        }
        if (compact)
          for (int p = count + tid; p < pw; p += kThreads) xo_row[p] = __float2half_rn(0.0f);
        if (tid == 0) a.x_scale[row] = am;
      }
      __syncthreads();   // s_red / s_row are reused by the next group
    }
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
      reinterpret_cast<uint4*>(W_O + static_cast<size_t>(n) * a.ld)[ch] = early[k];
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
  switch (vpt) {
    case 1: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<1>); break;
    case 2: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<2>); break;
    case 4: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<4>); break;
    case 8: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<8>); break;
    default: fn = reinterpret_cast<const void*>(detect_quantize_compact_kernel<16>); break;
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

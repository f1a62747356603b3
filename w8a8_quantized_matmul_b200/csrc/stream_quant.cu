// Single-pass detection + quantisation + compaction of the LLM.int8() path,
// one cooperative launch (all CTAs co-resident).
//
// Method: AIInfra "05Infer/06CompDistill/05Quantization01", LLM.int8() section
// (outlier feature dimensions by a magnitude threshold, vector-wise absmax INT8
// codes of the remaining dimensions, the outlier dimensions kept in fp16);
// tanjunchen "quantization explained part 2", section 1.2 (threshold 6.0; once
// the outlier dimension is split out the scale comes from the rest).
//
// Why one pass over X is enough. Every entry of a row with |x| > threshold
// lies in an outlier column by definition. So the absmax m1 of a row over the
// columns the row does not flag itself can differ from its absmax m over the
// non-outlier columns of the batch only through entries |x| <= threshold in
// columns that OTHER rows flag: m1 = max(m, mO), mO the row's largest such
// entry, and m1 == m whenever mO < m1. The kernel codes each row with m1 as
// soon as the row is in shared memory; once the outlier columns are known it
// zeroes the codes there and codes again only the rows with mO >= m1 > 0 (with
// the outliers in a few fixed columns, almost never).
//
// Each CTA (one per SM, 16 warps) owns a contiguous block of R rows of X and
// of the rows of W. Its warps form NG groups of GW warps; GW is chosen so that
// a warp's piece of a row is at most 256 vectors of 8 fp16 values (8 per lane,
// held in registers): GW = 1 up to K = 2048, K/2048 beyond.
//   stream   group g takes rows g, g + NG, ... of the block; each warp bulk-
//            copies its piece of a row into its own slot in shared memory (one
//            mbarrier per slot), reads it into registers and at once refills
//            the slot with its piece of the group's next row, so that the load
//            overlaps the coding. From the registers: the maximum |x| of each
//            vector and of the lane (only a lane whose maximum exceeds the
//            threshold, rarely, takes the per-entry flags of its vectors above
//            it, a shared-memory atomicOr into the CTA's column bitmap, and the
//            maximum over its unflagged entries), the row maximum m1 (warp
//            reduction, then one named barrier of the group), and the codes
//            with m1, stored straight to Xq. Groups never wait for one another.
//   list     after the last row: warp 0 builds the ascending list L of the
//            CTA's flagged columns (a subset of the batch's outlier set O; equal
//            to it unless the CTA's rows miss a column that other rows flag);
//            meanwhile the last warp ORs the CTA's bitmap into the batch bitmap
//            and arrives at the grid barrier (its memory fence is off the
//            other warps' path).
//   fix-up   with L, by the other warps, every (row, listed column) pair in
//            parallel: the code zeroed, the entry copied into the fp16 panel
//            X_O, the row's largest such |x| <= threshold (mO) by a shared-
//            memory atomicMax; the CTA's rows of W_O gathered from the rows of
//            the transposed weight Wt ([K][N]) that the list names, contiguous
//            reads issued first so that the latencies overlap; then the rows
//            with mO >= m1 coded again from X (L2) with L masked out.
//   check    wait at the grid barrier (bounded) and compare the batch bitmap
//            with L; if the batch has a column the CTA's rows lack, every row of
//            the CTA, X_O and W_O again with the batch's set.
// With a given outlier set (the OR of the bitmaps of a token-sharded batch's
// ranks, or a top-k selection) nothing is speculative: the given columns are
// masked out of the row maximum and the codes from the start, and the list, the
// panels and the bitmap follow with no check and no grid barrier.
// The panels are zero-padded to a multiple of 16 columns (one kind::f16 K step
// of the GEMM, which multiplies only the K steps that hold columns).
//
// Codes: rint(fl32(fl32(x*127)/a)) for |x| <= a (so within +-127 without a
// clamp) from the FMA-corrected quotient of quant_common.cuh, with x*127 formed
// by a mixed-precision FMA (codes8_h). The threshold test |x| > t is taken on
// fp16 values against the largest fp16 value not above t, which selects the
// same entries as the fp32 comparison.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace i8mm {

namespace {

constexpr int kMaxWarps = 16;     // warps per CTA
constexpr int kMaxGroups = 8;     // warp groups per CTA (named barriers 1..8)
constexpr int kRowBlock = 64;     // rows of the fix-up per round (shared row maxima)
constexpr int kMaxRedo = 32;      // rows of one CTA listed for a second coding
constexpr uint32_t kFixBar = 9;   // named barrier of the fix-up warps
constexpr uint64_t kGridWaitNs = 2000000000ull;

__device__ __forceinline__ int load_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t hmax2_bits(uint32_t x, uint32_t y) {
  const __half2 r = __hmax2(*reinterpret_cast<const __half2*>(&x), *reinterpret_cast<const __half2*>(&y));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Larger of the two halves of a packed pair of non-negative fp16 values, as fp32.
__device__ __forceinline__ float hpair_max(uint32_t x) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x));
  return fmaxf(f.x, f.y);
}

// Largest fp32 over the warp of non-negative values (their bit patterns order
// like the values).
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}

// Codes of the fp16 pair w, each in the low byte of its fp32 lane: n = x*127
// exactly (one mixed-precision FMA per value, fp16 operands, fp32 result),
// q = fl(n*ra), r = fma(q, -a, n), q' = fma(r, ra, q) (the FMA-corrected
// quotient of quant_common.cuh, the same operations in the same order), then
// the 1.5*2^23 rounding. ra2 = (ra, ra), na2 = (-a, -a), magic2 = (1.5*2^23) x 2,
// h127 = 127.0 in binary16.
__device__ __forceinline__ uint64_t code_pair_h(uint32_t w, uint64_t ra2, uint64_t na2,
                                                uint64_t magic2, uint16_t h127) {
  uint64_t s;
  asm("{\n\t"
      ".reg .b16 l, h;\n\t"
      ".reg .f32 n0, n1;\n\t"
      ".reg .b64 n, q, r;\n\t"
      "mov.b32 {l, h}, %1;\n\t"
      "fma.rn.f32.f16 n0, l, %5, %6;\n\t"
      "fma.rn.f32.f16 n1, h, %5, %6;\n\t"
      "mov.b64 n, {n0, n1};\n\t"
      "mul.rn.f32x2 q, n, %2;\n\t"
      "fma.rn.f32x2 r, q, %3, n;\n\t"
      "fma.rn.f32x2 q, r, %2, q;\n\t"
      "add.rn.f32x2 %0, q, %4;\n\t"
      "}"
      : "=l"(s)
      : "r"(w), "l"(ra2), "l"(na2), "l"(magic2), "h"(h127), "f"(-0.0f));
  return s;
}

// Eight INT8 codes of the vector u (codes8 of quant_common.cuh, n formed by the
// mixed-precision FMA).
__device__ __forceinline__ uint2 codes8_h(const uint4& u, uint64_t ra2, uint64_t na2,
                                          uint64_t magic2, uint16_t h127) {
  const uint64_t s0 = code_pair_h(u.x, ra2, na2, magic2, h127);
  const uint64_t s1 = code_pair_h(u.y, ra2, na2, magic2, h127);
  const uint64_t s2 = code_pair_h(u.z, ra2, na2, magic2, h127);
  const uint64_t s3 = code_pair_h(u.w, ra2, na2, magic2, h127);
  const uint32_t w0 = __byte_perm(__byte_perm(static_cast<uint32_t>(s0), static_cast<uint32_t>(s0 >> 32), 0x0040),
                                  __byte_perm(static_cast<uint32_t>(s1), static_cast<uint32_t>(s1 >> 32), 0x0040),
                                  0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(static_cast<uint32_t>(s2), static_cast<uint32_t>(s2 >> 32), 0x0040),
                                  __byte_perm(static_cast<uint32_t>(s3), static_cast<uint32_t>(s3 >> 32), 0x0040),
                                  0x5410);
  return make_uint2(w0, w1);
}

// Shared-memory layout (16-byte aligned pieces):
//   rows   [NW] slots        one slot per warp for its piece of a row (pv
//                            vectors); after the stream the outlier list [K] u16
//   lbits  [words] u32       the CTA's own column flags
//   gbits  [words] u32       the batch bitmap, after the grid barrier
//   gred   [kMaxGroups][2][kMaxWarps] f32  per-warp row maxima of each group,
//                            alternating between consecutive rows
//   m1     [kRowBlock] f32   row maxima m1 of the first rows of the block
//   mo     [kRowBlock] u32   fix-up maxima mO (fp32 bit patterns) of a round
//   misc   [4] i32           list count, redo count
//   redo   [kMaxRedo] i32    rows to code again
//   bar    [kMaxWarps] u64   one mbarrier per slot
struct StreamSmem {
  size_t rows, lbits, gbits, gred, m1, mo, misc, redo, bar, total;
};

__host__ __device__ inline size_t up16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

__host__ __device__ inline StreamSmem stream_smem_layout(int K, size_t slot_bytes) {
  StreamSmem L;
  const size_t words = static_cast<size_t>((K + 31) / 32);
  const size_t list_bytes = static_cast<size_t>(K) * 2;
  size_t off = 0;
  L.rows = off;   off = up16(off + (slot_bytes > list_bytes ? slot_bytes : list_bytes));
  L.lbits = off;  off = up16(off + words * 4);
  L.gbits = off;  off = up16(off + words * 4);
  L.gred = off;   off = up16(off + kMaxGroups * 2 * kMaxWarps * 4);
  L.m1 = off;     off = up16(off + kRowBlock * 4);
  L.mo = off;     off = up16(off + kRowBlock * 4);
  L.misc = off;   off = up16(off + 16);
  L.redo = off;   off = up16(off + kMaxRedo * 4);
  L.bar = off;    off = up16(off + kMaxWarps * 8);
  L.total = off;
  return L;
}

}  // namespace

template <int VPL, bool FULL, bool GIVEN>
__global__ void __launch_bounds__(32 * kMaxWarps, 1)
    stream_quantize_kernel(FusedArgs a, uint32_t th2bits, int GW) {
  extern __shared__ __align__(128) uint8_t ssm[];
  const int K = a.K;
  const int NW = static_cast<int>(blockDim.x) >> 5;
  const int NG = NW / GW;
  const int words = (K + 31) >> 5;
  const int nv = K >> 3;
  const int pv = (nv + GW - 1) / GW;   // vectors of a row per warp of a group
  const StreamSmem L = stream_smem_layout(K, static_cast<size_t>(NW) * pv * 16);
  uint16_t* s_idx = reinterpret_cast<uint16_t*>(ssm + L.rows);   // valid after the stream
  uint32_t* s_lbits = reinterpret_cast<uint32_t*>(ssm + L.lbits);
  uint32_t* s_gbits = reinterpret_cast<uint32_t*>(ssm + L.gbits);
  float* s_gred = reinterpret_cast<float*>(ssm + L.gred);
  float* s_m1 = reinterpret_cast<float*>(ssm + L.m1);
  uint32_t* s_mo = reinterpret_cast<uint32_t*>(ssm + L.mo);
  int32_t* s_misc = reinterpret_cast<int32_t*>(ssm + L.misc);
  int32_t* s_redo = reinterpret_cast<int32_t*>(ssm + L.redo);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(ssm + L.bar);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const __half2 th2 = *reinterpret_cast<const __half2*>(&th2bits);

  const int rows_per = (a.M + gridDim.x - 1) / gridDim.x;
  const int r0 = min(a.M, static_cast<int>(blockIdx.x) * rows_per);
  const int R = min(a.M, r0 + rows_per) - r0;
  const int nper = (a.N + gridDim.x - 1) / gridDim.x;
  const int wn0 = min(a.N, static_cast<int>(blockIdx.x) * nper);
  const int wn1 = min(a.N, wn0 + nper);

  // The GEMM that follows may launch now; it waits for this grid's completion
  // before reading anything written here.
  griddep_launch_dependents();
  // Given-set mode (token-sharded batches, top-k): the outlier set is the OR of
  // the given bitmaps and final; the threshold plays no part.
  constexpr bool given = GIVEN;
  for (int w = tid; w < words; w += blockDim.x) {
    uint32_t b = 0u;
    if (given)
      for (int r = 0; r < a.given_n; ++r) b |= __ldg(a.given + static_cast<size_t>(r) * words + w);
    s_lbits[w] = b;
  }
  for (int r = tid; r < kRowBlock; r += blockDim.x) s_mo[r] = 0u;
  if (tid == 0) {
    for (int s = 0; s < NW; ++s) mbar_init(&s_bar[s], 1);
    fence_mbarrier_init();
    s_misc[1] = 0;
  }
  __syncthreads();

  // ------------------------------------------------------------ stream
  const int g = warp / GW;            // group
  const int gw = warp - g * GW;       // warp within the group
  const int v0 = gw * pv;             // first vector of this warp's piece of a row
  const int npv = FULL ? VPL * 32 : max(0, min(pv, nv - v0));
  const uint32_t piece_bytes = static_cast<uint32_t>(npv) * 16u;
  const int nrows = R > g ? (R - g + NG - 1) / NG : 0;   // rows of this group: g, g + NG, ...
  const uint4* slot = reinterpret_cast<const uint4*>(ssm + L.rows + static_cast<size_t>(warp) * pv * 16);
  uint64_t* bar = &s_bar[warp];
  const __half* xpiece = a.X + static_cast<size_t>(r0 + g) * K + static_cast<size_t>(v0) * 8;
  const size_t row_step = static_cast<size_t>(NG) * K;   // elements from one row of the group to its next
  auto issue = [&](int i) {   // lane 0: this warp's piece of the group's i-th row
    // Earlier generic-proxy reads of the slot before the async-proxy write.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, piece_bytes);
    bulk_load(const_cast<uint4*>(slot), xpiece + static_cast<size_t>(i) * row_step, piece_bytes, bar);
  };
  if (lane == 0 && npv > 0 && nrows > 0) issue(0);
  // Loop-invariant operands of the code arithmetic.
  const uint64_t magic2 = f2pack(kMagic, kMagic);
  const uint16_t h127 = 0x57F0u;   // 127.0 in binary16
  // Given-set mode: the set bits of the thread's vectors (the same columns on
  // every row), four 8-bit masks per word.
  uint32_t gmask[(VPL + 3) / 4];
#pragma unroll
  for (int j = 0; j < (VPL + 3) / 4; ++j) gmask[j] = 0u;
  if (given) {
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const int v = v0 + c * 32 + lane;
      const uint32_t m8 = (FULL || c * 32 + lane < npv) ? (s_lbits[v >> 2] >> (8 * (v & 3))) & 0xFFu : 0u;
      gmask[c >> 2] |= m8 << (8 * (c & 3));
    }
  }
  auto gm8 = [&](int c) { return (gmask[c >> 2] >> (8 * (c & 3))) & 0xFFu; };
  bool ok = true;
  uint2* dst = reinterpret_cast<uint2*>(a.Xq + static_cast<size_t>(r0 + g) * K) + v0 + lane;
  const size_t dst_step = row_step / 8;                    // uint2 per group row step
  for (int i = 0; i < nrows; ++i, dst += dst_step) {
    uint4 u[VPL];
    if (npv > 0) {
      if (ok && !mbar_wait(bar, static_cast<uint32_t>(i & 1))) {
        ok = false;
        if (lane == 0) atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
      }
#pragma unroll
      for (int c = 0; c < VPL; ++c)
        u[c] = (FULL || c * 32 + lane < npv) ? slot[c * 32 + lane] : make_uint4(0u, 0u, 0u, 0u);
      // The piece is in registers: the slot takes the group's next row now,
      // while this one is coded.
      __syncwarp();
      if (lane == 0 && i + 1 < nrows) issue(i + 1);
    } else {
#pragma unroll
      for (int c = 0; c < VPL; ++c) u[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    // Pass 1: maximum |x| of each vector and of the lane. Only a lane whose
    // maximum exceeds the threshold (rare) takes the per-entry flags of its
    // vectors that exceed it and the maximum over its unflagged entries.
    uint32_t vm[VPL];
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      uint32_t ax = u[c].x & 0x7FFF7FFFu, ay = u[c].y & 0x7FFF7FFFu;
      uint32_t az = u[c].z & 0x7FFF7FFFu, aw = u[c].w & 0x7FFF7FFFu;
      if (given) {
        const uint32_t m8 = gm8(c);
        if (m8 != 0u) {   // given outlier columns are left out of the maximum
          ax &= keep_half2(m8, 0);
          ay &= keep_half2(m8, 1);
          az &= keep_half2(m8, 2);
          aw &= keep_half2(m8, 3);
        }
      }
      vm[c] = hmax2_bits(hmax2_bits(ax, ay), hmax2_bits(az, aw));
    }
    uint32_t rm = vm[0];
#pragma unroll
    for (int c = 1; c < VPL; ++c) rm = hmax2_bits(rm, vm[c]);
    if (!given && __hgt2_mask(*reinterpret_cast<const __half2*>(&rm), th2) != 0u) {
      rm = 0u;
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        if (__hgt2_mask(*reinterpret_cast<const __half2*>(&vm[c]), th2) == 0u) {
          rm = hmax2_bits(rm, vm[c]);
          continue;
        }
        const uint32_t wd[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
        uint32_t f8 = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t ab = wd[k] & 0x7FFF7FFFu;
          const uint32_t fl = __hgt2_mask(*reinterpret_cast<const __half2*>(&ab), th2);
          rm = hmax2_bits(rm, ab & ~fl);
          f8 |= ((fl & 1u) << (2 * k)) | (((fl >> 16) & 1u) << (2 * k + 1));
        }
        const int v = v0 + c * 32 + lane;
        if (FULL || c * 32 + lane < npv) atomicOr(&s_lbits[v >> 2], f8 << (8 * (v & 3)));
      }
    }
    float m1 = warp_max_nonneg(hpair_max(rm));
    if (GW > 1) {
      float* red = s_gred + (g * 2 + (i & 1)) * kMaxWarps;
      if (lane == 0) red[gw] = m1;
      named_bar_sync(1u + static_cast<uint32_t>(g), GW * 32);
      m1 = warp_max_nonneg(red[lane < GW ? lane : 0]);
    }
    const float ra = quant_rcp(m1);
    const uint64_t ra2 = f2pack(ra, ra), na2 = f2pack(-m1, -m1);
    // Pass 2: the codes with m1 (entries the row flags itself get codes that
    // the fix-up overwrites with 0).
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      if (FULL || c * 32 + lane < npv) {
        uint2 q = codes8_h(u[c], ra2, na2, magic2, h127);
        if (given) {   // codes at the given outlier columns are 0
          const uint32_t m8 = gm8(c);
          if (m8 != 0u) {
            q.x &= keep_bytes(m8 & 0xFu);
            q.y &= keep_bytes(m8 >> 4);
          }
        }
        dst[c * 32] = q;
      }
    }
    if (gw == 0 && lane == 0) {
      const int row = g + i * NG;
      a.x_scale[r0 + row] = m1;
      if (row < kRowBlock) s_m1[row] = m1;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------ list, arrival
  // Ascending list of a bitmap (one warp; lane l scans a contiguous run of
  // words) into s_idx, its length into s_misc[0].
  auto build_list = [&](const uint32_t* bits) {
    const int lper = (words + 31) >> 5;
    const int lw0 = min(words, lane * lper), lw1 = min(words, lw0 + lper);
    int cnt = 0;
    for (int w = lw0; w < lw1; ++w) cnt += __popc(bits[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
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

  // One W_O item: 8 consecutive panel columns of one weight row n of the CTA's
  // range, read from the rows idx[p] of Wt ([K][N]); consecutive items are
  // consecutive n, so each of the 8 loads is coalesced across a warp (the
  // caller stores the 16 bytes).
  auto gather_item = [&](int it, int count, int chunks, int& n, int& ch) {
    (void)chunks;
    const int nr = wn1 - wn0;
    ch = it / nr;
    n = wn0 + (it - ch * nr);
    const __half* wcol = a.W + n;
    uint4 o;
    __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int p = ch * 8 + i;
      h[i] = (p < count) ? __ldg(wcol + static_cast<size_t>(s_idx[p]) * a.N) : __float2half_rn(0.0f);
    }
    return o;
  };
  auto store_item = [&](int n, int ch, const uint4& o) {
    reinterpret_cast<uint4*>(a.W_O + static_cast<size_t>(n) * a.ld)[ch] = o;
  };

  // Fix-up with the list in s_idx, by threads [0, nw*32): every (row, listed
  // column) pair of the CTA's rows in parallel (code zeroed, entry into X_O,
  // zero padding to 16 columns; with `check` the row's largest listed |x| <=
  // threshold into s_mo, and the rows with mO >= m1 > 0 noted for a second
  // coding), and the CTA's rows of W_O, whose first two items' loads are issued
  // before the fix-up so that the latencies overlap.
  auto fix_and_gather = [&](int count, bool check, int nw) {
    if (count == 0) return;
    const int nt = nw * 32;
    const int pw = (count + 15) & ~15;
    const int chunks = pw >> 3;
    const int items = (wn1 - wn0) * chunks;
    int n0 = -1, c0 = 0, n1 = -1, c1 = 0;
    uint4 g0 = make_uint4(0u, 0u, 0u, 0u), g1 = g0;
    if (tid < items) g0 = gather_item(tid, count, chunks, n0, c0);
    if (tid + nt < items) g1 = gather_item(tid + nt, count, chunks, n1, c1);
    for (int rb = 0; rb < R; rb += kRowBlock) {
      const int nrb = min(kRowBlock, R - rb);
      for (int e = tid; e < nrb * pw; e += nt) {
        const int rl = e / pw;
        const int p = e - rl * pw;
        const size_t rr = static_cast<size_t>(r0 + rb + rl);
        __half h = __float2half_rn(0.0f);
        if (p < count) {
          const int col = s_idx[p];
          h = a.X[rr * K + col];
          a.Xq[rr * K + col] = 0;
          const float f = fabsf(__half2float(h));
          if (check && f <= a.threshold) atomicMax(&s_mo[rl], __float_as_uint(f));
        }
        a.X_O[rr * a.ld + p] = h;
      }
      if (check) {
        named_bar_sync(kFixBar, nt);
        for (int r = tid; r < nrb; r += nt) {
          const int row = rb + r;
          const float m1 = row < kRowBlock ? s_m1[row] : a.x_scale[r0 + row];
          const float mo = __uint_as_float(s_mo[r]);
          s_mo[r] = 0u;
          if (m1 > 0.0f && mo >= m1) {
            const int i = atomicAdd(&s_misc[1], 1);
            if (i < kMaxRedo) s_redo[i] = row;
          }
        }
        named_bar_sync(kFixBar, nt);
      }
    }
    if (n0 >= 0) store_item(n0, c0, g0);
    if (n1 >= 0) store_item(n1, c1, g1);
    for (int it = tid + 2 * nt; it < items; it += nt) {
      int n, ch;
      const uint4 o = gather_item(it, count, chunks, n, ch);
      store_item(n, ch, o);
    }
  };

  // Codes of rows again, read from X (L2), with the columns of `mbits` masked
  // out; one warp per row, all warps.
  auto recode = [&](const uint32_t* mbits, int nrows, const int32_t* rows) {
    for (int i = warp; i < nrows; i += NW) {
      const int row = rows ? rows[i] : i;
      const uint4* xs = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(r0 + row) * K);
      uint32_t hm = 0u;
      for (int v = lane; v < nv; v += 32) {
        const uint4 u = __ldg(xs + v);
        const uint32_t m8 = (mbits[v >> 2] >> (8 * (v & 3))) & 0xFFu;
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) hm = hmax2_bits(hm, wd[k] & 0x7FFF7FFFu & keep_half2(m8, k));
      }
      const float m1 = warp_max_nonneg(hpair_max(hm));
      const float ra = quant_rcp(m1);
      uint2* dst = reinterpret_cast<uint2*>(a.Xq + static_cast<size_t>(r0 + row) * K);
      for (int v = lane; v < nv; v += 32) {
        const uint32_t m8 = (mbits[v >> 2] >> (8 * (v & 3))) & 0xFFu;
        uint2 q = codes8(__ldg(xs + v), m1, ra);
        q.x &= keep_bytes(m8 & 0xFu);
        q.y &= keep_bytes(m8 >> 4);
        dst[v] = q;
      }
      if (lane == 0) a.x_scale[r0 + row] = m1;
    }
  };

  if (given) {
    // The set is final: the list, the bitmap (CTA 0) and the panels; no check.
    if (warp == 0) build_list(s_lbits);
    if (blockIdx.x == 0)
      for (int w = tid; w < words; w += blockDim.x) a.bitmap[w] = s_lbits[w];
    __syncthreads();
    fix_and_gather(s_misc[0], false, NW);
    __syncthreads();
    if (blockIdx.x == 0) {
      const int count = s_misc[0];
      for (int p = tid; p < count; p += blockDim.x) a.col_idx[p] = s_idx[p];
      if (tid == 0) *a.n_outliers = count;
    }
    return;
  }
  const int ctl = NW - 1;                  // control warp: batch bitmap and arrival
  const int nwork = NW > 1 ? NW - 1 : 1;   // warps of the fix-up
  if (warp == 0) build_list(s_lbits);
  if (warp == ctl)
    for (int w = lane; w < words; w += 32) {
      const uint32_t b = s_lbits[w];
      if (b != 0u) atomicOr(a.bitmap + w, b);
    }
  __syncthreads();
  if (warp == ctl) {
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(a.sync_ctr, 1);   // arrival at the grid barrier
    }
    __syncwarp();
  }

  // ------------------------------------------------------------ fix-up
  if (warp < nwork) fix_and_gather(s_misc[0], true, nwork);
  __syncthreads();
  const int nredo = s_misc[1];
  if (nredo > kMaxRedo)
    recode(s_lbits, R, nullptr);
  else if (nredo > 0)
    recode(s_lbits, nredo, s_redo);

  // ------------------------------------------------------------ check
  if (tid == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (load_acquire(a.sync_ctr) < static_cast<int>(gridDim.x)) {
      __nanosleep(64);
      if (globaltimer_ns() - t0 > kGridWaitNs) {
        atomicCAS(a.status, 0, -5 /* I8MM_ERR_TIMEOUT */);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  int extra = 0;
  for (int w = tid; w < words; w += blockDim.x) {
    const uint32_t g = __ldcg(a.bitmap + w);
    s_gbits[w] = g;
    extra |= (g & ~s_lbits[w]) != 0u;
  }
  extra = __syncthreads_or(extra);
  if (extra) {
    // The batch has an outlier column this CTA's rows missed: everything of
    // the CTA again with the batch's set.
    recode(s_gbits, R, nullptr);
    __syncthreads();
    if (warp == 0) build_list(s_gbits);
    __syncthreads();
    fix_and_gather(s_misc[0], false, NW);
    __syncthreads();
  }
  if (blockIdx.x == 0) {
    const int count = s_misc[0];
    for (int p = tid; p < count; p += blockDim.x) a.col_idx[p] = s_idx[p];
    if (tid == 0) *a.n_outliers = count;
  }
}

namespace {

// Bit pattern of the largest fp16 value not above t (t >= 0; +inf for t = inf):
// for every fp16 value h, h > t in fp32 exactly when h > that value in fp16.
uint16_t half_floor_bits(float t) {
  if (std::isinf(t)) return 0x7C00u;
  auto val = [](uint16_t b) {
    __half_raw r;
    r.x = b;
    return __half2float(__half(r));
  };
  if (val(0x7BFFu) <= t) return 0x7BFFu;
  uint16_t lo = 0, hi = 0x7BFFu;   // val(lo) <= t < val(hi)
  while (hi - lo > 1) {
    const uint16_t mid = static_cast<uint16_t>((lo + hi) / 2);
    if (val(mid) <= t)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

// Co-resident CTAs of the kernel on the current device for a launch shape,
// looked up once per shape (the attribute call and the occupancy query cost
// microseconds per call). 0 with *err set on failure.
int coresident_ctas(const void* fn, int dev, int nw, size_t smem, cudaError_t* err) {
  struct Entry {
    const void* fn;
    int dev, nw;
    size_t smem;
    int ctas;
  };
  static Entry cache[64];
  static int cached = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < cached; ++i)
      if (cache[i].fn == fn && cache[i].dev == dev && cache[i].nw == nw && cache[i].smem == smem)
        return cache[i].ctas;
  }
  // The attribute is raised to the device's opt-in maximum, never lowered, so
  // that a cached shape with more shared memory stays launchable.
  int optin = 0, per_sm = 0, sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e == cudaSuccess && static_cast<size_t>(optin) < smem) e = cudaErrorInvalidConfiguration;
  if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 32 * nw, smem);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess && per_sm < 1) e = cudaErrorInvalidConfiguration;
  if (e != cudaSuccess) {
    *err = e;
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cached < 64) cache[cached++] = Entry{fn, dev, nw, smem, per_sm * sms};
  return per_sm * sms;
}

}  // namespace

// Absmax codes, with detection or with a given outlier set (not the zero-point codes).
cudaError_t launch_detect_quantize_stream(const FusedArgs& a, cudaStream_t s) {
  // 16 warps in groups of GW warps per row, GW the smallest power of two that
  // leaves each warp at most 256 vectors (8 per lane, held in registers) of a
  // row; VPL = vectors per lane, a power of two; one slot per warp for its
  // piece of a row.
  const int nv = a.K / 8;
  int GW = 1;
  while ((nv + GW - 1) / GW > 256 && GW < kMaxWarps) GW *= 2;
  const int pv = (nv + GW - 1) / GW;
  int VPL = 1;
  while (VPL * 32 < pv) VPL *= 2;
  // Every warp's piece full (no bounds checks in the stream) for the usual K.
  const bool full = nv == GW * VPL * 32;
  const bool given = a.given != nullptr;
  const void* fn = nullptr;
#define I8MM_STREAM_FN(V)                                                                      \
  (full ? (given ? reinterpret_cast<const void*>(stream_quantize_kernel<V, true, true>)          \
                 : reinterpret_cast<const void*>(stream_quantize_kernel<V, true, false>))       \
        : (given ? reinterpret_cast<const void*>(stream_quantize_kernel<V, false, true>)        \
                 : reinterpret_cast<const void*>(stream_quantize_kernel<V, false, false>)))
  switch (VPL) {
    case 1: fn = I8MM_STREAM_FN(1); break;
    case 2: fn = I8MM_STREAM_FN(2); break;
    case 4: fn = I8MM_STREAM_FN(4); break;
    case 8: fn = I8MM_STREAM_FN(8); break;
    default: fn = I8MM_STREAM_FN(16); break;
  }
#undef I8MM_STREAM_FN
  const int NW = kMaxWarps;
  const size_t smem = stream_smem_layout(a.K, static_cast<size_t>(NW) * pv * 16).total;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int ctas = coresident_ctas(fn, dev, NW, smem, &e);
  if (ctas == 0) return e;
  // Enough CTAs to keep every SM streaming, but not more than can be co-resident.
  const int want = max((a.M + 1) / 2, (a.N + 15) / 16);
  const int grid = max(1, min(ctas, want));
  const uint32_t th = half_floor_bits(a.threshold);
  uint32_t th2 = th | (th << 16);
  int gw = GW;
  FusedArgs args = a;
  void* params[] = {&args, &th2, &gw};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(32 * NW), params, smem, s);
}

}  // namespace i8mm

// Importance on the 5th-generation tensor cores (bf16 inputs, fp32 accumulate).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp_j = (1/L_q) sum_q softmax_j(q.k_j / sqrt(d)) over
// the clean candidate keys.
//
// The L_q x L_k probability matrix is never stored.  Two passes recompute the
// logits with tcgen05.mma:
//   pass 1 (rows)     CTA = 256 queries of one head; streams every 256-key
//                     tile; D = Q K^T in TMEM; the epilogue thread that owns a
//                     query row keeps a (reference, sum) pair in log2 units
//                     and the CTA writes nl_q = -log2 sum_j 2^(c s_qj),
//                     c = scale*log2(e) (padded query rows: -inf).
//   pass 2 (columns)  CTA = 256 keys of one head (128 for the CTAs that make
//                     up a last, partial wave: measured 0.7-2 % faster than
//                     a last wave of 256-key CTAs); streams every 256-query tile;
//                     D = K Q^T + nl/c in TMEM (keys on the TMEM lanes), so
//                     each epilogue thread owns one key and sums 2^(c D)
//                     over all queries in registers: no atomics, no partial
//                     buffers, deterministic.  The query's nl_q/c enters the
//                     accumulator through one extra K=16 MMA step per tile:
//                     a block of ones on the key side against, per query,
//                     nl_q/(2c) split into three bf16 terms and stored twice
//                     (exact to ~2^-24 relative), written by pass 1 (or the
//                     merge) and brought in by TMA with the query tile.  The
//                     epilogue then needs no per-column shared-memory loads
//                     (measured 2.8 % faster for both passes than adding nl_q
//                     in the epilogue).
//
// Work per score is one tensor-core MAC row (256 flops at d=128) and one
// exponential.  The SM's special-function unit retires ~16 exponentials per
// clock against ~32 scores per clock of dense bf16 MMA, so the epilogue, not
// the MMA, sets the pace.  The design therefore
//   - issues M=128, N=256, K=16 MMAs: at N=128 the single-CTA MMA is bound by
//     reading its operands from shared memory (measured ~1.0 PFLOP/s with the
//     epilogue and TMA removed); N=256 reuses each A fragment for twice the
//     columns;
//   - holds two 128-row A tiles per CTA, each with its own 256-column TMEM
//     accumulator, and feeds every streamed B tile to both (ping-pong): the
//     eight epilogue warps of one A tile drain its accumulator (two
//     warpgroups, 128 columns each) while the MMA for the other tile runs,
//     and an accumulator is handed back to the MMA as soon as each of its
//     warps has loaded its slice (measured 1-3 % faster than one A tile with
//     two accumulators, and each B tile crosses from L2 once per 256 rows);
//   - uses packed f32x2 FMA/ADD for the scale-and-shift and the running sums;
//   - evaluates part of the exponentials on the FMA pipes (ex2_poly2, a
//     degree-3 polynomial of our own: 3 in 16 in the row pass, 3 in 8 in the
//     column pass) and the rest on the special-function unit (sweeps of the
//     mix and the degree on B200 put the optimum there; the packed f16x2 and
//     bf16x2 forms of ex2 retire no more exponentials per clock than the
//     float32 one, 16 per SM);
//   - in pass 1 shifts by a lagged reference instead of the exact running max:
//     the reference only moves (with an exact rescale) when a chunk's sum
//     exceeds 2^32, so the per-element max disappears from the common path;
//     the chunks of a slice fold their overflow tests into one flag, read once
//     before the accumulator is released, and the rare overflowing slice is
//     redone from TMEM with the exact per-chunk test (a branch per chunk kept
//     the next chunk's work from overlapping: 3 % of both passes);
//   - in pass 1 splits the key range in 2-4 parts when that fills the last
//     wave of CTAs better; a small kernel merges the partial (reference, sum)
//     pairs.
//
// Roles (640 threads): warp 0 lane 0 issues TMA loads (3D tensor maps over
// [H][L][d], 128-byte swizzle, zero fill past L, no multicast; pass 2 also the
// [H][Lq_pad][16] extra rows, 32-byte swizzle), warp 1 lane 0
// issues the MMAs (M=128, N=256, K=16 steps), warp 2 owns the TMEM allocation
// (all 512 columns), warps 4-11 drain A tile 0 and warps 12-19 A tile 1 (warp w
// reads TMEM lanes 32(w%4)..+31).  A two-stage shared-memory ring of 64 KB operand
// tiles decouples TMA from the MMAs.  Every mbarrier wait is bounded; on timeout the kernel
// records an error word in the workspace and winds down (no trap, no endless
// spin).
#include <cuda.h>

#include "fc_common.cuh"
#include "fc_kernels.h"
#include "tc_ptx.cuh"

namespace fc {

namespace {
constexpr int kBM = 128;      // rows of the resident A tile (MMA M, TMEM lanes)
constexpr int kBN = 256;      // rows of each streamed B tile (MMA N, TMEM columns)
constexpr int kStages = 2;    // shared-memory ring depth (64 KB B tiles)
constexpr int kNA = 2;        // A tiles per CTA, one TMEM accumulator of kBN columns each
// Which of the 16 pairs of a 32-column chunk take the FMA-pipe exponential,
// per pass (bit p: pair p), and the degree of its polynomial.  Measured on
// B200 (both passes; one layer of 24 heads at L_k = 16384, 12 heads at
// 131072, 40 heads at 32760): degree 3 with 3/16 of the row pass's and 3/8 of
// the column pass's exponentials on the FMA pipes was the steadiest and,
// under the power cap of the long heads, the fastest (5.90 ms against
// 6.03-6.19 for degree 5 with 1/4 in both); masks whose register schedule
// spills (5 or 8 of 16 pairs in some placements) run 2-3x slower.
#ifndef FC_IMP_EMU_MASK1
#define FC_IMP_EMU_MASK1 0x0222  // pairs 1, 5, 9 of 16: 3/16 of the exponentials
#endif
#ifndef FC_IMP_EMU_MASK2
#define FC_IMP_EMU_MASK2 0x4A4A  // pairs 1, 3, 6, 9, 11, 14: 3/8
#endif
#ifndef FC_IMP_POLY_DEG
#define FC_IMP_POLY_DEG 3  // relative error below 7.6e-5 per exponential
#endif
constexpr int kWG = 2;        // epilogue warpgroups per A tile; each owns kBN/kWG columns
constexpr int kEpiWarps = kNA * kWG * 4;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr int kCh = 32;       // TMEM columns per tcgen05.ld chunk
constexpr int kSlice = kBN / kWG;  // columns of a tile that one warpgroup drains
static_assert(kSlice % kCh == 0, "each warpgroup drains whole chunks");
constexpr int kHalfA = kBM * 64 * 2;  // one 128-row x 64-element bf16 swizzled block (16 KB)
constexpr int kHalfB = kBN * 64 * 2;  // one 256-row x 64-element bf16 swizzled block (32 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kErrOffset = 0;      // error word in the workspace
constexpr size_t kLseOffset = 256;    // nl extra rows [H][Lq_pad][16] bf16, then split partials
constexpr int kMaxSplit = 4;          // pass 1 may split the key range in up to 4 parts
constexpr float kRescaleAt = 4294967296.0f;  // 2^32

template <int kPass>
__device__ __forceinline__ constexpr bool emulated_pair(int p) {
  return (((kPass == 1 ? FC_IMP_EMU_MASK1 : FC_IMP_EMU_MASK2) >> p) & 1) != 0;
}

template <int D>
constexpr int a_bytes() {
  return (D / 64) * kHalfA;
}
template <int D>
constexpr int b_bytes() {
  return (D / 64) * kHalfB;
}
constexpr int kXRow = 32;                // bytes of one extra K block row (16 bf16)
constexpr int kXBytes = kBN * kXRow;     // pass 2: the query tile's extra block, per stage
constexpr int kOnesBytes = kBM * kXRow;  // pass 2: the key tile's extra block (all ones)
template <int D>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)kNA * a_bytes<D>() + (size_t)kStages * b_bytes<D>() +
         (size_t)kStages * kXBytes + kOnesBytes + 256 + (size_t)kNA * kWG * 2 * kBM * sizeof(float);
}

// Row of the extra K block of pass 2 for one query: x = nl / (2 c) split into
// three bf16 terms (a + b + c = x to ~2^-24 relative), stored twice, so that
// against a block of ones the MMA adds 2(a + b + c) = nl / c to every logit of
// the query.  Padded queries get a large negative value (their terms vanish).
__device__ __forceinline__ void write_nlx(uint4* dst, float nl, float c2) {
  uint32_t w0 = 0xF149u, w1 = 0u;  // bf16 -1e30
  if (nl != -INFINITY) {
    const float x = __fdiv_rn(nl, 2.0f * c2);
    const __nv_bfloat16 a = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(a);
    const __nv_bfloat16 b = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(b);
    const __nv_bfloat16 c = __float2bfloat16_rn(r2);
    w0 = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
    w1 = (uint32_t)__bfloat16_as_ushort(c);
  }
  const uint4 w = make_uint4(w0, w1, 0u, 0u);
  dst[0] = w;
  dst[1] = w;
}

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t a_full;
  uint64_t acc_full[kNA];
  uint64_t acc_empty[kNA];
  uint32_t tmem_slot;
};

__device__ __forceinline__ void epilogue_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");  // the epilogue warps only
}

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}

template <int kPass>
__device__ __forceinline__ float2 exp2_pair(int p, float2 x) {
  if (emulated_pair<kPass>(p)) return tc::ex2_poly2<kPass == 1, FC_IMP_POLY_DEG>(x);
  return make_float2(tc::ex2(x.x), tc::ex2(x.y));
}

// Sum of 2^(c*s - ref) over one chunk; mixes MUFU and FMA-pipe exponentials.
__device__ __forceinline__ float chunk_sum_shifted(const uint32_t (&r)[kCh], float c, float ref) {
  const float2 cc = make_float2(c, c), sh = make_float2(-ref, -ref);
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < kCh / 2; ++p) {
    const float2 e = exp2_pair<1>(p, tc::ffma2(f2(r[2 * p], r[2 * p + 1]), cc, sh));
    if (p & 1)
      a1 = tc::fadd2(a1, e);
    else
      a0 = tc::fadd2(a0, e);
  }
  const float2 a = tc::fadd2(a0, a1);
  return a.x + a.y;
}

__device__ __forceinline__ float chunk_max(const uint32_t (&r)[kCh]) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kCh; j += 4) {
    m0 = tc::fmax3(m0, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
    m1 = tc::fmax3(m1, __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
  }
  return fmaxf(m0, m1);
}

// Pass 1 on one chunk: mask keys past L_k, then fold the chunk into the row's
// (reference, sum) pair.  The reference lags the running max: it only moves
// when the chunk's sum passes 2^32, and then exactly (rescale, recompute).
__device__ __forceinline__ void row_chunk(uint32_t (&r)[kCh], int valid, float c2, float& ref,
                                          float& l) {
  if (valid < kCh) {
#pragma unroll
    for (int j = 0; j < kCh; ++j)
      if (j >= valid) r[j] = 0xff800000u;  // -inf
  }
  if (ref == -INFINITY) ref = chunk_max(r) * c2;  // first values this group sees
  if (ref == -INFINITY) return;                   // every key here was padding
  float cs = chunk_sum_shifted(r, c2, ref);
  if (!(cs <= kRescaleAt)) {
    const float rnew = fmaxf(ref, chunk_max(r) * c2);
    l *= tc::ex2(ref - rnew);
    ref = rnew;
    cs = chunk_sum_shifted(r, c2, ref);
  }
  l += cs;
}

// Pass 1, the rare path: redo the first n chunks of a slice from TMEM with
// the exact per-chunk check (out of line, so its registers do not weigh on
// the common path).  Called by all 32 lanes of a warp together (tcgen05.ld
// and its wait are warp-collective).
__device__ __noinline__ void redo_chunks(uint32_t addr, int n, float c2, float& ref, float& l) {
  for (int c = 0; c < n; ++c) {
    uint32_t r[kCh];
    tc::tmem_ld32(addr + c * kCh, r);
    tc::tmem_ld_wait(r);
    row_chunk(r, kCh, c2, ref, l);
  }
}

// Pass 2 on one chunk: acc += 2^(c*(s + nl_q/c)) over the chunk's 32 queries
// (the MMA already added nl_q/c to every logit).
__device__ __forceinline__ void col_chunk(const uint32_t (&r)[kCh], float c2, float2& acc) {
  const float2 cc = make_float2(c2, c2), z = make_float2(0.f, 0.f);
  float2 a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < kCh / 2; ++p) {
    const float2 e = exp2_pair<2>(p, tc::ffma2(f2(r[2 * p], r[2 * p + 1]), cc, z));
    if (p & 1)
      a1 = tc::fadd2(a1, e);
    else
      acc = tc::fadd2(acc, e);
  }
  acc = tc::fadd2(acc, a1);
}

// CTA = two A tiles (256 rows) of one head; every streamed B tile feeds two
// MMAs, one per A tile, each into its own 256-column accumulator.  The eight
// epilogue warps of A tile j drain accumulator j while the MMA for the other
// tile runs (ping-pong).
// kPass 1: A = Q tiles, B = K tiles of one key split, epilogue = row log-sum-exp.
// kPass 2: A = K tiles, B = Q tiles (+ the extra K step), epilogue = column
// sums of 2^(c (s + nl/c)).
template <int D, int kPass>
__global__ void __launch_bounds__(kThreads, 1)
    imp_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                  const __grid_constant__ CUtensorMap mapX,
                  int Lq, int Lk, int lq_pad, int nsplit, float c2, uint4* __restrict__ nlx,
                  float2* __restrict__ part, float* __restrict__ imp, int* __restrict__ err,
                  int tph, int npair) {
  constexpr int KB = D / 64;
  constexpr int TA = a_bytes<D>();
  constexpr int TB = b_bytes<D>();
  constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kBM, kBN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sA = base;                        // [kNA] A tiles
  uint8_t* sB = base + kNA * TA;             // [kStages] B tiles
  uint8_t* sX = sB + kStages * TB;           // pass 2: [kStages][kBN][32 B]
  uint8_t* sOnes = sX + kStages * kXBytes;   // pass 2: [kBM][32 B] of bf16 ones
  Bars* bars = reinterpret_cast<Bars*>(sOnes + kOnesBytes);
  float* sM = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // merge buffer

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Pass 1: grid (query-tile pairs x splits, heads).  Pass 2: a flat grid
  // over every head's key tiles (tph per head, even): npair CTAs of two
  // tiles, then one CTA per remaining tile, so that the last, partial wave
  // is made of half-length CTAs.
  const int split = kPass == 1 ? blockIdx.x % nsplit : 0;
  int h, a0, na;
  if (kPass == 1) {
    h = blockIdx.y;
    a0 = (blockIdx.x / nsplit) * (kNA * kBM);
    na = kNA;
  } else {
    const int x = blockIdx.x;
    const int gt = x < npair ? 2 * x : 2 * npair + (x - npair);
    h = gt / tph;
    a0 = (gt % tph) * kBM;
    na = x < npair ? 2 : 1;
  }
  int t_begin = 0, nB;
  if (kPass == 1) {
    const int nkt = (Lk + kBN - 1) / kBN;
    const int per = (nkt + nsplit - 1) / nsplit;
    t_begin = split * per;
    nB = min(nkt, t_begin + per) - t_begin;
  } else {
    nB = lq_pad / kBN;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    tc::mbar_init(&bars->a_full, 1);
    for (int j = 0; j < kNA; ++j) {
      tc::mbar_init(&bars->acc_full[j], 1);
      tc::mbar_init(&bars->acc_empty[j], 4 * kWG);  // every warp of tile j reads its slice
    }
    tc::fence_barrier_init();
  }
  if (warp == 2) tc::tmem_alloc(&bars->tmem_slot, kNA * kBN);
  if (kPass == 2 && threadIdx.x >= 128 && threadIdx.x < 128 + kOnesBytes / 16) {
    reinterpret_cast<uint4*>(sOnes)[threadIdx.x - 128] =
        make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the MMA
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      tc::mbar_expect_tx(&bars->a_full, na * TA);
      for (int j = 0; j < na; ++j)
        for (int kb = 0; kb < KB; ++kb)
          tc::tma_load_3d(sA + j * TA + kb * kHalfA, &mapA, &bars->a_full, kb * 64,
                          a0 + j * kBM, h);
      // Pass 2 may start while the row pass (or the merge) finishes: only the
      // normaliser rows depend on it, so wait for it before the first stage.
      if (kPass == 2) grid_dep_wait();
      for (int t = 0; t < nB; ++t) {
        const int s = t % kStages, u = t / kStages;
        if (!tc::mbar_wait(&bars->empty[s], (u & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc::mbar_expect_tx(&bars->full[s], TB + (kPass == 2 ? kXBytes : 0));
        const int row_b = (t_begin + t) * kBN;
        for (int kb = 0; kb < KB; ++kb)
          tc::tma_load_3d(sB + s * TB + kb * kHalfB, &mapB, &bars->full[s], kb * 64, row_b, h);
        if (kPass == 2) tc::tma_load_3d(sX + s * kXBytes, &mapX, &bars->full[s], 0, row_b, h);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      ok = tc::mbar_wait(&bars->a_full, 0);
      for (int t = 0; ok && t < nB; ++t) {
        const int s = t % kStages, u = t / kStages;
        if (!tc::mbar_wait(&bars->full[s], u & 1)) {
          ok = false;
          break;
        }
        const uint32_t b_addr = tc::smem_u32(sB + s * TB);
        for (int j = 0; j < na; ++j) {
          if (!tc::mbar_wait(&bars->acc_empty[j], (t & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a_addr = tc::smem_u32(sA + j * TA);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ks = (kk & 3) * 32;  // 16 bf16 = 32 bytes per K step
            tc::mma_bf16(tmem + j * kBN, tc::desc_k_sw128(a_addr + (kk >> 2) * kHalfA + ks),
                         tc::desc_k_sw128(b_addr + (kk >> 2) * kHalfB + ks), kIdesc,
                         kk > 0 ? 1u : 0u);
          }
          if (kPass == 2)  // + nl_q / c on every logit of query q
            tc::mma_bf16(tmem + j * kBN, tc::desc_k_sw32(tc::smem_u32(sOnes)),
                         tc::desc_k_sw32(tc::smem_u32(sX + s * kXBytes)), kIdesc, 1u);
          tc::mma_commit(&bars->acc_full[j]);  // accumulator j ready
        }
        tc::mma_commit(&bars->empty[s]);  // operand stage reusable once both MMAs read it
      }
    }
  } else if (warp >= 4) {  // ---- epilogue: 4 kWG warpgroups per A tile, each on its column slice
    const int e = warp - 4;
    const int j = e / (4 * kWG);       // A tile (and accumulator) of this warp
    const int g = (e / 4) % kWG;       // column slice within the tile
    const int sub = warp & 3;          // TMEM lane quarter
    const int rloc = sub * 32 + lane;  // this thread's row of A tile j
    const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16) + j * kBN + g * kSlice;
    float ref = -INFINITY, l = 0.0f;     // pass 1: reference and sum (log2 units)
    float2 acc = make_float2(0.f, 0.f);  // pass 2: column sum
    for (int t = 0; t < (j < na ? nB : 0); ++t) {
      // the warp leaves together (the TMEM loads below are warp-collective)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->acc_full[j], t & 1))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const int valid = Lk - (t_begin + t) * kBN - g * kSlice;  // pass 1: keys left
      constexpr int kNch = kSlice / kCh;
      if (kPass == 1 && valid >= kSlice) {
        // A full slice: the chunks' overflow checks are folded into one flag,
        // so no chunk but the last ends in a branch.  If a chunk before the
        // last overflowed (rare), the slice is redone from TMEM, chunk by
        // chunk with the exact check, before the accumulator is released.
        const float l0 = l, ref0 = ref;
        bool bad = false;
#pragma unroll
        for (int c = 0; c < kNch; ++c) {
          uint32_t ra[kCh];
          // tcgen05.ld is warp-collective: the whole warp redoes the slice if
          // any of its rows overflowed (the others recompute the same sums).
          if (c + 1 == kNch && __any_sync(0xffffffffu, bad)) {
            l = l0;
            ref = ref0;
            redo_chunks(lane_addr, kNch - 1, c2, ref, l);
          }
          tc::tmem_ld32(lane_addr + c * kCh, ra);
          tc::tmem_ld_wait(ra);
          if (c + 1 == kNch) {  // the slice is in registers: free the accumulator
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->acc_empty[j]);
          }
          if (c == 0 && ref == -INFINITY) ref = chunk_max(ra) * c2;
          if (c + 1 < kNch) {
            const float cs = chunk_sum_shifted(ra, c2, ref);
            bad |= !(cs <= kRescaleAt);
            l += cs;
          } else {
            row_chunk(ra, kCh, c2, ref, l);
          }
        }
        continue;
      }
#pragma unroll
      for (int c = 0; c < kNch; ++c) {
        uint32_t ra[kCh];
        tc::tmem_ld32(lane_addr + c * kCh, ra);
        tc::tmem_ld_wait(ra);
        if (c + 1 == kSlice / kCh) {  // the slice is in registers: free the accumulator
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->acc_empty[j]);
        }
        if (kPass == 1)
          row_chunk(ra, valid - c * kCh, c2, ref, l);
        else
          col_chunk(ra, c2, acc);
      }
    }
    // Merge the slices' partial results for each row (every warp reaches
    // this barrier, also after a timeout).
    float* mj = sM + (size_t)j * kWG * 2 * kBM;
    if (g > 0) {
      mj[(2 * g) * kBM + rloc] = kPass == 1 ? ref : acc.x + acc.y;
      mj[(2 * g + 1) * kBM + rloc] = l;
    }
    epilogue_sync();
    if (g == 0 && ok && j < na) {
      const int row = a0 + j * kBM + rloc;
      if (kPass == 1) {
        float M = ref;
#pragma unroll
        for (int q = 1; q < kWG; ++q) M = fmaxf(M, mj[(2 * q) * kBM + rloc]);
        float L = (ref == -INFINITY) ? 0.0f : l * tc::ex2(ref - M);
#pragma unroll
        for (int q = 1; q < kWG; ++q) {
          const float rq = mj[(2 * q) * kBM + rloc];
          if (rq != -INFINITY) L += mj[(2 * q + 1) * kBM + rloc] * tc::ex2(rq - M);
        }
        if (nsplit == 1)
          write_nlx(nlx + ((size_t)h * lq_pad + row) * 2, row < Lq ? -(M + __log2f(L)) : -INFINITY,
                    c2);
        else
          part[((size_t)split * gridDim.y + h) * lq_pad + row] = make_float2(M, L);
      } else {
        float sum = acc.x + acc.y;
#pragma unroll
        for (int q = 1; q < kWG; ++q) sum += mj[(2 * q) * kBM + rloc];
        if (row < Lk) imp[(size_t)h * Lk + row] = sum / (float)Lq;
      }
    }
  }
  if (!ok) atomicExch(err, 1);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 2) tc::tmem_dealloc(tmem, kNA * kBN);
}

// Combine the key-split partial (reference, sum) pairs of every query row.
__global__ void nl_merge_kernel(const float2* __restrict__ part, int nsplit, int H, int Lq,
                                int lq_pad, float c2, uint4* __restrict__ nlx) {
  grid_dep_wait();  // the row pass's partials
  grid_dep_launch();
  const int64_t n = (int64_t)H * lq_pad;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int row = (int)(i % lq_pad);
    float M = -INFINITY;
    for (int q = 0; q < nsplit; ++q) M = fmaxf(M, part[q * n + i].x);
    float L = 0.0f;
    for (int q = 0; q < nsplit; ++q) {
      const float2 p = part[q * n + i];
      if (p.x != -INFINITY) L += p.y * tc::ex2(p.x - M);
    }
    write_nlx(nlx + i * 2, row < Lq ? -(M + __log2f(L)) : -INFINITY, c2);
  }
}

// Key splits for pass 1: the fewest (<= kMaxSplit) whose grid wastes at most
// 10 % of the last wave, keeping >= 4 key tiles (1024 keys) per split.
int choose_split(int units, int nkt) {
  const int sms = sm_count();
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= kMaxSplit; ++s) {
    if (s > 1 && nkt / s < 4) break;
    const double n = (double)units * s;
    const double eff = n / (ceil_div((int64_t)n, sms) * (double)sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
    if (eff >= 0.90) break;
  }
  return best;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [H][L][d] bf16, box = 64 elements (128 B, the swizzle span) x `rows` x 1 head.
// Tensor map over [H][L][d] bf16 whose heads are `ld` rows apart (ld >= L);
// rows past L read as zero.
bool make_map(CUtensorMap* map, const void* ptr, int H, int L, int d, int rows, int ld) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)ld * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [H][lq_pad][16] bf16 extra K blocks, box = 16 elements (32 B, the swizzle
// span) x kBN queries x 1 head.
bool make_map_x(CUtensorMap* map, const void* ptr, int H, int lq_pad) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {16, (cuuint64_t)lq_pad, (cuuint64_t)H};
  const cuuint64_t strides[2] = {(cuuint64_t)kXRow, (cuuint64_t)lq_pad * kXRow};
  const cuuint32_t box[3] = {16, (cuuint32_t)kBN, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t run(const void* q, const void* k, int H, int Lq, int Lk, int ldk, float scale,
                float* imp, void* ws, cudaStream_t s) {
  // A operands are 128-row tiles, B operands 256-row tiles.
  CUtensorMap mqA, mqB, mkA, mkB;
  if (!make_map(&mqA, q, H, Lq, D, kBM, Lq) || !make_map(&mqB, q, H, Lq, D, kBN, Lq) ||
      !make_map(&mkA, k, H, Lk, D, kBM, ldk) || !make_map(&mkB, k, H, Lk, D, kBN, ldk))
    return cudaErrorInvalidValue;
  int* err = reinterpret_cast<int*>(static_cast<char*>(ws) + kErrOffset);
  const int lq_pad = (int)ceil_div(Lq, kBN) * kBN;
  uint4* nlx = reinterpret_cast<uint4*>(static_cast<char*>(ws) + kLseOffset);
  float2* part = reinterpret_cast<float2*>(
      static_cast<char*>(ws) + kLseOffset + align_up((size_t)H * lq_pad * kXRow, 256));
  CUtensorMap mx;
  if (!make_map_x(&mx, nlx, H, lq_pad)) return cudaErrorInvalidValue;
  const float c2 = scale * kLog2e;
  const size_t smem = smem_bytes<D>();
  cudaError_t e;
  e = cudaFuncSetAttribute(imp_tc_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(imp_tc_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  const int nq = lq_pad / (kNA * kBM);
  const int nkt = (int)ceil_div(Lk, kBN);
  const int nsplit = choose_split(nq * H, nkt);
  imp_tc_kernel<D, 1><<<dim3(nq * nsplit, H), kThreads, smem, s>>>(
      mqA, mkB, mx, Lq, Lk, lq_pad, nsplit, c2, nlx, part, imp, err, 0, 0);
  add_launches(nsplit > 1 ? 3 : 2);
  // The merge and the column pass are launched as programmatic dependents of
  // the kernel before them and wait for it (griddepcontrol.wait) only where
  // they read what it wrote.  The passes themselves do not trigger their
  // dependents early: column-pass CTAs waiting on idle SMs during the row
  // pass's tail starved the redundancy kernel running beside the importance
  // (measured: 27 us more per bench step).
  cudaLaunchAttribute pdl[1] = {pdl_attribute()};
  if (nsplit > 1) {
    const int64_t n = (int64_t)H * lq_pad;
    const int64_t blocks = ceil_div(n, 256);
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3((unsigned)(blocks < 4096 ? blocks : 4096));
    mc.blockDim = dim3(256);
    mc.stream = s;
    mc.attrs = pdl;
    mc.numAttrs = 1;
    e = cudaLaunchKernelEx(&mc, nl_merge_kernel, (const float2*)part, nsplit, H, Lq, lq_pad, c2,
                           nlx);
    if (e != cudaSuccess) return e;
  }
  // pass 2: whole waves of two-tile CTAs; a remainder of at most one wave's
  // worth of tiles goes to one-tile CTAs (half as long), else to pairs too
  const int tph = (int)ceil_div(Lk, 2 * kBM) * 2;
  const int64_t tiles = (int64_t)tph * H;
  const int64_t wave2 = 2 * (int64_t)sm_count();
  int64_t rem = tiles % wave2;
  if (rem > wave2 / 2) rem = 0;
  const int64_t npair = (tiles - rem) / 2;
  cudaLaunchConfig_t pc = {};
  pc.gridDim = dim3((unsigned)(npair + rem), 1);
  pc.blockDim = dim3(kThreads);
  pc.dynamicSmemBytes = smem;
  pc.stream = s;
  pc.attrs = pdl;
  pc.numAttrs = 1;
  e = cudaLaunchKernelEx(&pc, imp_tc_kernel<D, 2>, mkA, mqB, mx, Lq, Lk, lq_pad, 1, c2, nlx, part,
                         imp, err, tph, (int)npair);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Self-test of the two exponentials (MUFU and FMA-pipe) on given inputs.
__global__ void exp2_selftest_kernel(const float* x, float* y_mufu, float* y_poly, int n) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 v = make_float2(x[i], x[i + 1]);
    y_mufu[i] = tc::ex2(v.x);
    y_mufu[i + 1] = tc::ex2(v.y);
    const float2 p = tc::ex2_poly2<false, FC_IMP_POLY_DEG>(v);
    y_poly[i] = p.x;
    y_poly[i + 1] = p.y;
  }
}
// Self-test of the bounded wait: every thread waits on an mbarrier that
// nothing arrives on, gives up after `limit` clocks and records it.
__global__ void wait_selftest_kernel(long long limit, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait(&bar, 0, limit);
  if (!ok && threadIdx.x == 0) atomicAdd(err, 1);
  __syncthreads();
}
}  // namespace

cudaError_t launch_wait_selftest(long long limit_cycles, int* err, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit_cycles, err);
  add_launches(1);
  return cudaGetLastError();
}

size_t importance_ws_bytes(int H, int Lq) {
  const size_t rows = (size_t)H * ceil_div(Lq, kBN) * kBN;
  return kLseOffset + align_up(rows * kXRow, 256) + kMaxSplit * rows * sizeof(float2);
}

bool importance_tc_supported(int d) { return d == 64 || d == 128; }

cudaError_t launch_importance_tc(const void* q, const void* k, int H, int Lq, int Lk, int d,
                                 float scale, float* imp, void* ws, cudaStream_t s, int ldk) {
  if (ldk <= 0) ldk = Lk;
  return d == 128 ? run<128>(q, k, H, Lq, Lk, ldk, scale, imp, ws, s)
                  : run<64>(q, k, H, Lq, Lk, ldk, scale, imp, ws, s);
}

cudaError_t launch_exp2_selftest(const float* x, float* y_mufu, float* y_poly, int n,
                                 cudaStream_t s) {
  const int pairs = n / 2;
  if (pairs > 0) {
    exp2_selftest_kernel<<<(unsigned)ceil_div(pairs, 256), 256, 0, s>>>(x, y_mufu, y_poly, n);
    add_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace fc

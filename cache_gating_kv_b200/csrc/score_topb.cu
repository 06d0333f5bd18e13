// Joint score and per-head top-B selection.
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp~ is the 1D max-pooled importance;
// Score_j = lambda*Imp~_j - (1-lambda)*Red_j; each head keeps its top-B tokens.
//
//   score kernel   grid (L_k/1024, H): pooled importance from a shared-memory
//                  tile with halo, the float32 score, and an order-preserving
//                  uint32 key (larger score -> larger key; -0 folded into +0)
//   select kernel  one 1024-thread block per head: a 4-pass MSB radix select
//                  (8-bit digits, per-warp histograms with match_any
//                  aggregation) finds the B-th largest key T and how many
//                  copies of T to keep; then one ordered compaction pass writes
//                  every kept index, ascending, using warp ballots for the
//                  in-warp ranks and a block scan over warps.  Ties at T keep
//                  the lowest indices.
// Keys are staged in shared memory when a head's keys fit, otherwise they are
// re-read from global memory (L2-resident) on every pass.
#include <cooperative_groups.h>

#include "fc_common.cuh"
#include "fc_kernels.h"

namespace cg = cooperative_groups;

namespace fc {

namespace {
constexpr int kScoreTile = 1024;
constexpr int kScoreThreads = 256;
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxPool = 255;
constexpr int kHistBytes = kSelWarps * 256 * 4;
constexpr int kSelSmemLimit = 220 * 1024;

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;  // -0 ties with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kScoreThreads)
    score_kernel(const float* __restrict__ imp, const float* __restrict__ red, int Lk, int r,
                 float lam, float one_minus_lam, float* __restrict__ score,
                 uint32_t* __restrict__ keys) {
  __shared__ float tile[kScoreTile + 2 * kMaxPool];
  const int h = blockIdx.y;
  const int j0 = blockIdx.x * kScoreTile;
  const float* ih = imp + (size_t)h * Lk;
  const int n = kScoreTile + 2 * r;
  for (int t = threadIdx.x; t < n; t += kScoreThreads) {
    const int j = j0 - r + t;
    tile[t] = (j >= 0 && j < Lk) ? ih[j] : -INFINITY;  // out-of-range taps ignored
  }
  __syncthreads();
  for (int t = threadIdx.x; t < kScoreTile; t += kScoreThreads) {
    const int j = j0 + t;
    if (j >= Lk) break;
    float p = tile[t];
    for (int o = 1; o <= 2 * r; ++o) p = fmaxf(p, tile[t + o]);
    const float a = __fmul_rn(lam, p);
    const float b = __fmul_rn(one_minus_lam, red[(size_t)h * Lk + j]);
    const float sc = __fsub_rn(a, b);
    if (score) score[(size_t)h * Lk + j] = sc;
    keys[(size_t)h * Lk + j] = order_key(sc);
  }
}

template <bool kStaged>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const uint32_t* __restrict__ keys, int Lk, int B, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned* hist = reinterpret_cast<unsigned*>(smem);  // [kSelWarps][256]
  uint32_t* skeys = reinterpret_cast<uint32_t*>(smem + kHistBytes);
  __shared__ unsigned s_total[256];
  __shared__ uint32_t s_prefix, s_pmask;
  __shared__ int s_remaining;
  __shared__ int s_gt[kSelWarps], s_tie[kSelWarps];

  const int h = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t* kh = keys + (size_t)h * Lk;
  if (kStaged) {
    for (int j = tid; j < Lk; j += kSelThreads) skeys[j] = kh[j];
  }
  auto key_at = [&](int j) -> uint32_t { return kStaged ? skeys[j] : __ldcg(kh + j); };
  if (tid == 0) {
    s_prefix = 0u;
    s_pmask = 0u;
    s_remaining = B;
  }

  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kSelWarps * 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, pmask = s_pmask;
    unsigned* wh = hist + warp * 256;
    for (int j0 = warp * 32; j0 < Lk; j0 += kSelThreads) {
      const int j = j0 + lane;
      uint32_t key = 0u;
      bool in = false;
      if (j < Lk) {
        key = key_at(j);
        in = (key & pmask) == prefix;
      }
      const unsigned vm = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned digit = (key >> shift) & 0xffu;
        const unsigned peers = __match_any_sync(vm, digit);
        if ((unsigned)lane == (unsigned)(__ffs(peers) - 1)) atomicAdd(&wh[digit], __popc(peers));
      }
    }
    __syncthreads();
    if (tid < 256) {
      unsigned t = 0u;
#pragma unroll 8
      for (int w = 0; w < kSelWarps; ++w) t += hist[w * 256 + tid];
      s_total[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l owns bins 255-8l .. 248-8l (lane 0 the largest digits).
      const int top = 255 - 8 * lane;
      unsigned mine = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) mine += s_total[top - i];
      unsigned cum = mine;  // inclusive scan from lane 0
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
      }
      const unsigned need = (unsigned)s_remaining;
      const unsigned hit = __ballot_sync(0xffffffffu, cum >= need);
      const int L = __ffs(hit) - 1;  // exists: the prefix holds >= need keys
      if (lane == L) {
        unsigned before = cum - mine;
        int digit = top;
        for (int i = 0; i < 8; ++i) {
          const unsigned c = s_total[top - i];
          if (before + c >= need) {
            digit = top - i;
            break;
          }
          before += c;
        }
        s_remaining = (int)(need - before);
        s_prefix = s_prefix | ((uint32_t)digit << shift);
        s_pmask = s_pmask | (0xffu << shift);
      }
    }
    __syncthreads();
  }

  // T = the B-th largest key; keep every key > T and the first `need` keys == T.
  const uint32_t T = s_prefix;
  const int need = s_remaining;
  const int seg = (int)ceil_div(ceil_div(Lk, kSelWarps), 32) * 32;
  const int w_lo = min(Lk, warp * seg), w_hi = min(Lk, w_lo + seg);
  int gt = 0, tie = 0;
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < w_hi ? key_at(j) : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, j < w_hi && key > T));
    tie += __popc(__ballot_sync(0xffffffffu, j < w_hi && key == T));
  }
  if (lane == 0) {
    s_gt[warp] = gt;
    s_tie[warp] = tie;
  }
  __syncthreads();
  int gt_base = 0, tie_base = 0;
  for (int w = 0; w < warp; ++w) {
    gt_base += s_gt[w];
    tie_base += s_tie[w];
  }
  int out = gt_base + min(need, tie_base);  // kept indices before this warp
  int tie_run = tie_base;
  const unsigned lt = (1u << lane) - 1u;
  int32_t* oh = idx + (size_t)h * B;
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < w_hi ? key_at(j) : 0u;
    const bool is_gt = j < w_hi && key > T;
    const bool is_tie = j < w_hi && key == T;
    const unsigned tb = __ballot_sync(0xffffffffu, is_tie);
    const bool sel = is_gt || (is_tie && tie_run + __popc(tb & lt) < need);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = out + __popc(sb & lt);
    if (sel && pos < B) oh[pos] = j;  // pos < B always holds; the check keeps writes in bounds
    out += __popc(sb);
    tie_run += __popc(tb);
  }
}

// ---------------------------------------------------------------------------
// Fused score + top-B for one head per thread-block cluster (the common case).
// Each CTA of the cluster owns a contiguous slice of the head's tokens: it
// scores its slice (pooled importance from a shared-memory tile with halo)
// straight into shared-memory keys, every radix pass sums the CTAs' 256-bin
// histograms through distributed shared memory (every CTA derives the same
// digit), and the final ordered compaction offsets each CTA by the kept
// counts of the CTAs before it.  Cluster barriers are hardware barriers.
//
// Two shapes.  8-CTA clusters (L_k <= 32768): 512-thread CTAs, a histogram
// per warp, the slice's pooling tile and its keys in separate buffers.
// 16-CTA clusters: 256 threads, one histogram, and the keys written over the
// pooling tile (each key over the tile position of its own first tap, a
// chunk of 2048 keys at a time once the chunk's taps have been read), so that
// a CTA needs about 37 KB of shared memory at L_k = 131072 and six fit on an
// SM: 40 heads' 640 CTAs then run in one wave.  (With separate 1024-key
// pooling sub-tiles, 44 KB and five per SM, the GPU held 38 such clusters at
// once and the last two heads ran in a second wave: 124 us per call against
// 49 us for four heads.)
// ---------------------------------------------------------------------------
constexpr int kCsMaxSlice = 12288;  // keys per CTA held in shared memory
constexpr int kCsMaxCluster = 16;   // CTAs per cluster (one head)
constexpr int kCsCandCap = 384;     // in-place shape: room for the last passes' candidates

// kThreads: CTA size; kHists: histogram copies (one per warp, or fewer shared
// by several warps); kInPlace: the keys overwrite the pooling tile (and the
// last passes' candidates get a small buffer of their own after it).
// Resident CTAs per SM each shape is compiled for (registers capped to fit):
// three 512-thread CTAs keep 40 heads' 320 CTAs of the 8-CTA shape in one
// wave (at 59 registers two fit, and the call took 46 instead of 34 us); six
// 256-thread CTAs the 16-CTA shape's 640.
template <int kThreads>
constexpr int cs_min_blocks() {
  return kThreads == 512 ? 3 : 6;
}

template <int kThreads, int kHists, bool kInPlace>
__global__ void __launch_bounds__(kThreads, cs_min_blocks<kThreads>())
    score_select_cluster_kernel(const float* __restrict__ imp, const float* __restrict__ red,
                                int Lk, int r, float lam, float one_minus_lam, int B,
                                float* __restrict__ score, int32_t* __restrict__ idx) {
  static_assert(kThreads >= 256, "one thread per histogram bin");
  constexpr int kWarps = kThreads / 32;
  static_assert(kWarps % kHists == 0, "warps share histograms evenly");
  grid_dep_wait();  // the kernel before this one (importance) has finished
  grid_dep_launch();
  cg::cluster_group cluster = cg::this_cluster();
  const int nrank = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per = (int)ceil_div(Lk, nrank);
  const int lo = min(Lk, rank * per), hi = min(Lk, lo + per);
  const int n = hi - lo;

  // Separate buffers: keys [per], then the pooling tile [per + 2r].  In place:
  // the pooling tile [per + 2r] whose first n positions end up holding the
  // keys, then the candidate buffer [kCsCandCap].
  extern __shared__ __align__(16) unsigned char csm[];
  uint32_t* skeys = reinterpret_cast<uint32_t*>(csm);
  float* tile = reinterpret_cast<float*>(kInPlace ? csm : csm + (size_t)per * 4);
  __shared__ unsigned whist[kHists][256];
  __shared__ unsigned hist[2][256];  // this CTA's histogram, double-buffered by pass
  // the cluster's totals of a pass: written after the pass's histograms have
  // been folded into hist[] and read before they are cleared for the next
  unsigned* s_total = &whist[0][0];
  __shared__ uint32_t s_prefix, s_pmask;
  __shared__ int s_remaining;
  __shared__ int s_cnt[2];   // this CTA's (greater, tie) counts (read by the cluster)
  __shared__ int s_wgt[kWarps], s_wtie[kWarps];
  __shared__ int s_ncand;
  unsigned* myhist = whist[warp % kHists];

  // The first radix pass's histogram (top 8 bits) is built while the keys
  // are formed.
  for (int i = tid; i < kHists * 256; i += kThreads) (&whist[0][0])[i] = 0u;

  // ---- scores of the slice -> order-preserving keys ------------------------
  // Imp and Red were just written by the kernels before: each thread issues
  // kLd loads before it uses the first, so their L2 latencies overlap.
  constexpr int kLd = 8;
  const float* ih = imp + (size_t)h * Lk;
  const float* rh = red + (size_t)h * Lk;
  const int nt = n + 2 * r;
  for (int t0 = tid; t0 < nt; t0 += kThreads * kLd) {
    float v[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int t = t0 + u * kThreads, j = lo - r + t;
      v[u] = (t < nt && j >= 0 && j < Lk) ? ih[j] : -INFINITY;  // out-of-range taps ignored
    }
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int t = t0 + u * kThreads;
      if (t < nt) tile[t] = v[u];
    }
  }
  __syncthreads();
  // Block-uniform loop over chunks of kThreads * kLd keys (every lane takes
  // part in the histogram's votes, and the in-place shape's barrier is
  // reached by every thread).  Key t reads taps t .. t + 2r of the tile.
  for (int c0 = 0; c0 < n; c0 += kThreads * kLd) {
    const int t0 = c0 + warp * 32 + lane;
    float rv[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int t = t0 + u * kThreads;
      rv[u] = t < n ? rh[lo + t] : 0.0f;
    }
    uint32_t kk[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int t = t0 + u * kThreads;
      uint32_t key = 0u;
      if (t < n) {
        float pm = tile[t];
        for (int o = 1; o <= 2 * r; ++o) pm = fmaxf(pm, tile[t + o]);
        const float sc = __fsub_rn(__fmul_rn(lam, pm), __fmul_rn(one_minus_lam, rv[u]));
        if (score) score[(size_t)h * Lk + lo + t] = sc;
        key = order_key(sc);
        if (!kInPlace) skeys[t] = key;
      }
      kk[u] = key;
      const unsigned vm = __ballot_sync(0xffffffffu, t < n);
      if (t < n) {
        const unsigned digit = key >> 24;
        const unsigned peers = __match_any_sync(vm, digit);
        if ((unsigned)lane == (unsigned)(__ffs(peers) - 1)) atomicAdd(&myhist[digit], __popc(peers));
      }
    }
    if (kInPlace) {
      // Every tap of this chunk has been read; its keys go over its first
      // positions.  The next chunk reads taps from position c0 + kThreads*kLd
      // on, which no key of this chunk overwrites.
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        const int t = t0 + u * kThreads;
        if (t < n) skeys[t] = kk[u];
      }
    }
  }
  if (tid == 0) {
    s_prefix = 0u;
    s_pmask = 0u;
    s_remaining = B;
  }
  __syncthreads();

  // ---- 4 radix passes over the cluster's keys ----------------------------------
  // Pass 0's histogram is already built.  Once two passes have fixed the top
  // 16 bits of the threshold, the keys that still match them (a small part of
  // the slice) are gathered into `cand` (the pooling tile's space, free by
  // then) and the last two passes count only those; if more match than the
  // space holds, the last passes scan the whole slice instead.
  uint32_t* cand = kInPlace ? skeys + (per + 2 * r) : reinterpret_cast<uint32_t*>(tile);
  const int cand_cap = kInPlace ? kCsCandCap : per + 2 * r;
  const uint32_t* src = skeys;
  int nsrc = n;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t prefix = s_prefix, pmask = s_pmask;
    if (pass == 2) {
      if (tid == 0) s_ncand = 0;
      __syncthreads();
      const unsigned lt = (1u << lane) - 1u;
      for (int j0 = warp * 32; j0 < n; j0 += kThreads) {
        const int j = j0 + lane;
        const uint32_t key = j < n ? skeys[j] : 0u;
        const bool in = j < n && (key & pmask) == prefix;
        const unsigned b = __ballot_sync(0xffffffffu, in);
        int off = 0;
        if (lane == 0 && b) off = atomicAdd(&s_ncand, __popc(b));
        off = __shfl_sync(0xffffffffu, off, 0);
        const int pos = off + __popc(b & lt);
        if (in && pos < cand_cap) cand[pos] = key;
      }
      __syncthreads();
      if (s_ncand <= cand_cap) {
        src = cand;
        nsrc = s_ncand;
      }
    }
    if (pass > 0) {
      for (int i = tid; i < kHists * 256; i += kThreads) (&whist[0][0])[i] = 0u;
      __syncthreads();
      for (int j0 = warp * 32; j0 < nsrc; j0 += kThreads) {
        const int j = j0 + lane;
        uint32_t key = 0u;
        bool in = false;
        if (j < nsrc) {
          key = src[j];
          in = (key & pmask) == prefix;
        }
        const unsigned vm = __ballot_sync(0xffffffffu, in);
        if (in) {
          const unsigned digit = (key >> shift) & 0xffu;
          const unsigned peers = __match_any_sync(vm, digit);
          if ((unsigned)lane == (unsigned)(__ffs(peers) - 1)) atomicAdd(&myhist[digit], __popc(peers));
        }
      }
      __syncthreads();
    }
    if (tid < 256) {  // one thread per bin
      unsigned t = 0u;
#pragma unroll
      for (int w = 0; w < kHists; ++w) t += whist[w][tid];
      hist[pass & 1][tid] = t;
    }
    cluster.sync();
    if (tid < 256) {
      // every CTA's count of this bin, all loads in flight before the sum
      unsigned c[kCsMaxCluster];
#pragma unroll
      for (int q = 0; q < kCsMaxCluster; ++q)
        c[q] = q < nrank ? *cluster.map_shared_rank(&hist[pass & 1][tid], q) : 0u;
      unsigned t = 0u;
#pragma unroll
      for (int q = 0; q < kCsMaxCluster; ++q) t += c[q];
      s_total[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l owns bins 255-8l .. 248-8l (lane 0 the largest digits).
      const int top = 255 - 8 * lane;
      unsigned mine = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) mine += s_total[top - i];
      unsigned cum = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
      }
      const unsigned need = (unsigned)s_remaining;
      const unsigned hit = __ballot_sync(0xffffffffu, cum >= need);
      const int L = __ffs(hit) - 1;  // exists: the prefix holds >= need keys
      if (lane == L) {
        unsigned before = cum - mine;
        int digit = top;
        for (int i = 0; i < 8; ++i) {
          const unsigned c = s_total[top - i];
          if (before + c >= need) {
            digit = top - i;
            break;
          }
          before += c;
        }
        s_remaining = (int)(need - before);
        s_prefix = s_prefix | ((uint32_t)digit << shift);
        s_pmask = s_pmask | (0xffu << shift);
      }
    }
    __syncthreads();
  }

  // ---- ordered compaction: keep every key > T and the first `need` keys == T ----
  const uint32_t T = s_prefix;
  const int need = s_remaining;
  const int seg = (int)ceil_div(ceil_div(n, kWarps), 32) * 32;
  const int w_lo = min(n, warp * seg), w_hi = min(n, w_lo + seg);
  int gt = 0, tie = 0;
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < w_hi ? skeys[j] : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, j < w_hi && key > T));
    tie += __popc(__ballot_sync(0xffffffffu, j < w_hi && key == T));
  }
  if (lane == 0) {
    s_wgt[warp] = gt;
    s_wtie[warp] = tie;
  }
  __syncthreads();
  if (tid == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < kWarps; ++w) {
      a += s_wgt[w];
      b += s_wtie[w];
    }
    s_cnt[0] = a;
    s_cnt[1] = b;
  }
  cluster.sync();
  // Counts of the CTAs before this one (their tokens come first), all loads
  // in flight before the sums.
  int gt_base = 0, tie_base = 0;
  {
    int cg_[kCsMaxCluster], ct_[kCsMaxCluster];
#pragma unroll
    for (int q = 0; q < kCsMaxCluster; ++q) {
      cg_[q] = q < rank ? *cluster.map_shared_rank(&s_cnt[0], q) : 0;
      ct_[q] = q < rank ? *cluster.map_shared_rank(&s_cnt[1], q) : 0;
    }
#pragma unroll
    for (int q = 0; q < kCsMaxCluster; ++q) {
      gt_base += cg_[q];
      tie_base += ct_[q];
    }
  }
  for (int w = 0; w < warp; ++w) {
    gt_base += s_wgt[w];
    tie_base += s_wtie[w];
  }
  int out = gt_base + min(need, tie_base);
  int tie_run = tie_base;
  const unsigned lt = (1u << lane) - 1u;
  int32_t* oh = idx + (size_t)h * B;
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < w_hi ? skeys[j] : 0u;
    const bool is_gt = j < w_hi && key > T;
    const bool is_tie = j < w_hi && key == T;
    const unsigned tb = __ballot_sync(0xffffffffu, is_tie);
    const bool sel = is_gt || (is_tie && tie_run + __popc(tb & lt) < need);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = out + __popc(sb & lt);
    if (sel && pos < B) oh[pos] = lo + j;  // pos < B always holds; the check keeps writes in bounds
    out += __popc(sb);
    tie_run += __popc(tb);
  }
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

__global__ void fill_all_kernel(int32_t* idx, int Lk, int B, int H) {
  const int64_t n = (int64_t)H * B;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i % B);
    idx[i] = r < Lk ? r : -1;
  }
}
}  // namespace

size_t score_topb_ws_bytes(int H, int Lk) { return align_up((size_t)H * Lk * 4, 256); }

cudaError_t launch_score_topb(const float* imp, const float* red, int H, int Lk, int pool,
                              float lambda, int B, float* score, int32_t* idx, void* ws,
                              cudaStream_t s) {
  uint32_t* keys = static_cast<uint32_t*>(ws);
  const float one_minus = 1.0f - lambda;  // float32, as the score's definition
  const int r = pool / 2;
  if (B < Lk && Lk <= 16 * kCsMaxSlice) {
    // One cluster per head: 8 CTAs of 512 threads, or 16 (non-portable) of
    // 256 threads with sub-tiled pooling for long histories.
    const bool large = Lk > 8 * 4096;
    const int csize = large ? 16 : 8;
    const int threads = large ? 256 : 512;
    const int per = (int)ceil_div(Lk, csize);
    const size_t smem = large ? (size_t)(per + 2 * r + kCsCandCap) * 4
                              : (size_t)per * 4 + (size_t)(per + 2 * r) * 4;
    auto kern = large ? score_select_cluster_kernel<256, 1, true>
                      : score_select_cluster_kernel<512, 16, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    if (csize > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      // all of the SM's shared memory, so that six ~37 KB CTAs fit on an SM
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)csize, (unsigned)H, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attribute();  // scheduled while the importance finishes
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, imp, red, Lk, r, lambda, one_minus, B, score, idx);
    if (e != cudaSuccess) return e;
    add_launches(1);
    return cudaSuccess;
  }
  dim3 g1((unsigned)ceil_div(Lk, kScoreTile), H);
  score_kernel<<<g1, kScoreThreads, 0, s>>>(imp, red, Lk, r, lambda, one_minus, score, keys);
  add_launches(2);  // the score kernel and one selection (or keep-all) kernel
  if (B >= Lk) {
    const int64_t nfb = ceil_div((int64_t)H * B, 256);
    fill_all_kernel<<<(unsigned)(nfb < 1024 ? nfb : 1024), 256, 0, s>>>(
        idx, Lk, B, H);
    return cudaGetLastError();
  }
  const size_t staged = (size_t)kHistBytes + (size_t)Lk * 4;
  if (staged <= (size_t)kSelSmemLimit) {
    const cudaError_t e = cudaFuncSetAttribute(
        select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)staged);
    if (e != cudaSuccess) return e;
    select_kernel<true><<<H, kSelThreads, staged, s>>>(keys, Lk, B, idx);
  } else {
    const cudaError_t e = cudaFuncSetAttribute(
        select_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHistBytes);
    if (e != cudaSuccess) return e;
    select_kernel<false><<<H, kSelThreads, kHistBytes, s>>>(keys, Lk, B, idx);
  }
  return cudaGetLastError();
}

}  // namespace fc

// Redundancy of every clean key, per head, as an HBM stream over K.
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Red_j = softmax_j((1/L_k) sum_i S_ij), S the cosine
// similarity of l2-normalised keys with its diagonal set to zero.
//
// The L_k x L_k matrix is never formed.  With s = sum_i khat_i,
//   sum_{i != j} khat_i . khat_j = khat_j . s - ||khat_j||^2      (exact)
// so the logits r_j need one reduction over K and one dot pass.  r_j lies in
// [-1, 1], hence exp(r_j) cannot overflow and the softmax needs no max.
//
// Three phases per head, each over fixed slices of its keys (one CTA per
// slice; 512 or 1024 keys, by the head's size), so a head's result does not
// depend on how many heads a call has:
//   1. sum:       the slice's sum of khat, converted to 2^-32 fixed point and
//                 added to the head's 64-bit integer accumulators (integer
//                 addition is exact, so s is the same whatever order the
//                 slices finish in);
//   2. logits:    every row's r_j and e_j = exp(r_j) (written to red), and the
//                 slice's sum of e_j added the same way;
//   3. normalise: red_j *= 1 / sum_j e_j.
// Phase 2 reads K a second time.  The heads go in groups whose keys take at
// most 48 MB (80 MB for heads of 8 MB and more), and launch g runs phase 1 of
// group g, phase 2 of group g-1 and phase 3 of group g-2, so that one group's
// sum streams from HBM while the previous group's logits run.  (The groups
// were sized for the re-read to come from L2; measured on B200 it does not:
// the re-read found 2 % of its lines in L2, and a 48 MB buffer read twice in
// a row alone found 60 %, so the L2 keeps much less than its 126 MB of one
// stream.  K is read twice from HBM; what the pipeline gains is overlap.)  The
// launches are programmatic dependents of each other: the sum CTAs of launch
// g start as the SMs of launch g-1 free up; the logit and normalise CTAs wait
// (griddepcontrol.wait) for launch g-1 to complete.  No CTA spins on another.
#include <algorithm>

#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

namespace {
constexpr int kRedThreads = 256;
constexpr int kRedWarps = kRedThreads / 32;
// Keys per CTA and the keys' bytes per head group.  Both depend on the head's
// size only (its L_k, d and dtype), never on H, so a head's result does not
// depend on the call.  Measured on B200 (bf16, d=128): heads of 4 MB (L_k =
// 16384) ran best with 512-key slices in 48 MB groups (47 us for 24 heads
// against 55-72 with 1024/2048-key slices or 80 MB groups); heads of 8 MB
// and more with 1024-key slices in 80 MB groups (121 us for 40 heads of 32760
// keys against 129; 414 us for 40 heads of 131072 against 471).
constexpr int kSliceSmall = 512, kSliceLarge = 1024;
constexpr size_t kGroupSmall = 48ull << 20, kGroupLarge = 80ull << 20;
constexpr size_t kLargeHead = 8ull << 20;  // per-head key bytes from which the large shape is used
constexpr double kFix = 4294967296.0;       // 2^32: scale of the fixed-point accumulators
constexpr int kMaxLk = 1 << 26;             // keeps every accumulator below 2^63

// Each lane holds two 16-byte vectors (32 contiguous bytes) of a row.
template <typename T, int D>
struct RowLayout {
  static constexpr int VPL = 2;                     // vectors per lane
  static constexpr int EPL = VPL * Vec16<T>::N;     // elements per lane
  static constexpr int LPR = D / EPL;               // lanes per row
  static constexpr int RPW = 32 / LPR;              // rows per warp step
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row layout");
};

// 1/max(||k||, 1e-12) from ||k||^2 on the special-function unit.
__device__ __forceinline__ float inv_norm(float n2) {
  return n2 > 1e-24f ? rsqrtf(n2) : 1e12f;
}
__device__ __forceinline__ float exp_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
  return y;
}

// Sum over the LPR lanes that hold one row (xor offsets below LPR stay inside
// the row's lane group).
template <int LPR>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16-byte read-only load that does not allocate in L1, with an L2 cache policy
// (evict_last for the first read of a key, evict_first for its last read:
// measured 2-5 % faster than no hint at every size).
__device__ __forceinline__ uint4 ld_nc_v4_pol(const void* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ uint64_t l2_policy(bool keep) {
  uint64_t pol;
  if (keep)
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

template <typename T, int D, int U>
__device__ __forceinline__ void load_rows(const T* kh, int r0, int hi, int sub, int cl,
                                          uint4 (&u)[U][2], uint64_t pol) {
  using L = RowLayout<T, D>;
#pragma unroll
  for (int i = 0; i < U; ++i) {
    const int r = r0 + i * L::RPW + sub;
    const T* p = kh + (size_t)r * D + cl * L::EPL;
    u[i][0] = r < hi ? ld_nc_v4_pol(p, pol) : make_uint4(0u, 0u, 0u, 0u);
    u[i][1] = r < hi ? ld_nc_v4_pol(p + Vec16<T>::N, pol) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T, int D>
__device__ __forceinline__ void unpack(const uint4 (&u)[2], float* e) {
  Vec16<T>::to_float(u[0], e);
  Vec16<T>::to_float(u[1], e + Vec16<T>::N);
}

__device__ __forceinline__ long long to_fix(double v) { return __double2ll_rn(v * kFix); }
__device__ __forceinline__ double from_fix(long long v) { return (double)v * (1.0 / kFix); }

// The phases of one launch, by CTA index: first n1*S CTAs sum heads
// [h1, h1+n1), then n2*S CTAs form the logits of heads [h2, h2+n2), then n3*S
// CTAs normalise heads [h3, h3+n3).
struct Roles {
  int h1, n1, h2, n2, h3, n3;
};

// Workspace: per head D fixed-point sums of khat, then per head the
// fixed-point sum of e_j; zeroed at the start of every call.
template <int D>
__device__ __forceinline__ long long* s_fix(long long* ws, int h) {
  return ws + (size_t)h * (D + 1);
}

template <typename T, int D, int U>
__global__ void __launch_bounds__(kRedThreads)
    red_phase_kernel(const T* __restrict__ k, int Lk, int ldk, int rows, int S, Roles ro,
                     long long* __restrict__ acc, float* __restrict__ red) {
  // The next launch may start on the SMs this one frees; its phase-2 and
  // phase-3 CTAs still wait for this whole launch.
  grid_dep_launch();
  using L = RowLayout<T, D>;
  constexpr int kRowsPerIter = kRedWarps * L::RPW * U;
  const int b = blockIdx.x;
  int phase, h, sl;
  if (b < ro.n1 * S) {
    phase = 1;
    h = ro.h1 + b / S;
    sl = b % S;
  } else if (b < (ro.n1 + ro.n2) * S) {
    const int c = b - ro.n1 * S;
    phase = 2;
    h = ro.h2 + c / S;
    sl = c % S;
  } else {
    const int c = b - (ro.n1 + ro.n2) * S;
    phase = 3;
    h = ro.h3 + c / S;
    sl = c % S;
  }
  const int lo = sl * rows, hi = min(Lk, lo + rows);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / L::LPR, cl = lane % L::LPR;
  const T* kh = k + (size_t)h * ldk * D;
  long long* sh = s_fix<D>(acc, h);  // [D] sums of khat, then [1] sum of e
  float* rh = red + (size_t)h * Lk;

  __shared__ float s_acc[kRedWarps][D];
  __shared__ float s_vec[D];
  __shared__ double s_esum[kRedWarps];

  if (phase == 1) {  // ---- sum of the slice's normalised rows ----------------
    const uint64_t pol = l2_policy(true);
    float a[L::EPL];
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) a[i] = 0.0f;
    for (int r0 = lo + warp * L::RPW * U; r0 < hi; r0 += kRowsPerIter) {
      uint4 raw[U][2];
      load_rows<T, D, U>(kh, r0, hi, sub, cl, raw, pol);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float e[L::EPL];
        unpack<T, D>(raw[u], e);
        float n2 = 0.0f;
#pragma unroll
        for (int i = 0; i < L::EPL; ++i) n2 = fmaf(e[i], e[i], n2);
        n2 = row_sum<L::LPR>(n2);
        const float inv = inv_norm(n2);  // a zero key (or a row past hi) adds zero
#pragma unroll
        for (int i = 0; i < L::EPL; ++i) a[i] = fmaf(e[i], inv, a[i]);
      }
    }
#pragma unroll
    for (int o = L::LPR; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[i], o);
    if (sub == 0) {
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) s_acc[warp][cl * L::EPL + i] = a[i];
    }
    __syncthreads();
    for (int c = tid; c < D; c += kRedThreads) {
      float t = 0.0f;
#pragma unroll
      for (int w = 0; w < kRedWarps; ++w) t += s_acc[w][c];
      atomicAdd(reinterpret_cast<unsigned long long*>(sh + c), (unsigned long long)to_fix(t));
    }
    return;
  }

  grid_dep_wait();  // the sums (phase 2) or the e_j (phase 3) of the launch before
  if (phase == 2) {  // ---- logits r_j and e_j = exp(r_j) ---------------------
    for (int c = tid; c < D; c += kRedThreads) s_vec[c] = (float)from_fix(__ldcg(sh + c));
    __syncthreads();
    float sv[L::EPL];
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) sv[i] = s_vec[cl * L::EPL + i];
    const float inv_lk = 1.0f / (float)Lk;
    const uint64_t pol = l2_policy(false);
    double esum = 0.0;
    for (int r0 = lo + warp * L::RPW * U; r0 < hi; r0 += kRowsPerIter) {
      uint4 raw[U][2];
      load_rows<T, D, U>(kh, r0, hi, sub, cl, raw, pol);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float e[L::EPL];
        unpack<T, D>(raw[u], e);
        float n2 = 0.0f, dot = 0.0f;
#pragma unroll
        for (int i = 0; i < L::EPL; ++i) {
          n2 = fmaf(e[i], e[i], n2);
          dot = fmaf(e[i], sv[i], dot);
        }
        n2 = row_sum<L::LPR>(n2);
        dot = row_sum<L::LPR>(dot);
        const float inv = inv_norm(n2);
        // r_j = (khat_j . s - ||khat_j||^2) / L_k
        const float rj = (dot * inv - n2 * inv * inv) * inv_lk;
        const float ej = exp_fast(rj);
        const int r = r0 + u * L::RPW + sub;
        if (r < hi && cl == 0) {
          rh[r] = ej;
          esum += (double)ej;
        }
      }
    }
    esum = warp_sum(esum);
    if (lane == 0) s_esum[warp] = esum;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
#pragma unroll
      for (int w = 0; w < kRedWarps; ++w) t += s_esum[w];
      atomicAdd(reinterpret_cast<unsigned long long*>(sh + D), (unsigned long long)to_fix(t));
    }
    return;
  }

  // ---- phase 3: normalise the slice ---------------------------------------------
  const float inv = (float)(1.0 / from_fix(__ldcg(sh + D)));
  for (int r = lo + tid; r < hi; r += kRedThreads) rh[r] = rh[r] * inv;
}

template <typename T, int D>
cudaError_t run(const T* k, int H, int Lk, int ldk, float* red, void* ws, cudaStream_t s) {
  constexpr int U = 4;  // rows in flight per lane (two 16-byte loads each)
  auto kern = red_phase_kernel<T, D, U>;
  const size_t head_bytes = (size_t)Lk * D * sizeof(T);
  const bool large = head_bytes >= kLargeHead;
  const int rows = large ? kSliceLarge : kSliceSmall;
  const size_t group_bytes = large ? kGroupLarge : kGroupSmall;
  const int S = (int)ceil_div(Lk, rows);
  const int G = (int)std::max<size_t>(1, std::min<size_t>(H, group_bytes / head_bytes));
  const int nG = (int)ceil_div(H, G);
  long long* acc = static_cast<long long*>(ws);
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)H * (D + 1) * sizeof(long long), s);
  if (e != cudaSuccess) return e;
  add_launches(1);
  cudaLaunchAttribute pdl[1] = {pdl_attribute()};
  auto heads = [&](int g, int& h0, int& n) {
    if (g < 0 || g >= nG) {
      h0 = 0;
      n = 0;
      return;
    }
    h0 = g * G;
    n = std::min(G, H - h0);
  };
  for (int g = 0; g < nG + 2; ++g) {
    Roles ro;
    heads(g, ro.h1, ro.n1);
    heads(g - 1, ro.h2, ro.n2);
    heads(g - 2, ro.h3, ro.n3);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((ro.n1 + ro.n2 + ro.n3) * S));
    cfg.blockDim = dim3(kRedThreads);
    cfg.stream = s;
    // The first launch follows the memset (and whatever wrote K) in plain
    // stream order; the later ones are programmatic dependents.
    cfg.attrs = g > 0 ? pdl : nullptr;
    cfg.numAttrs = g > 0 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, k, Lk, ldk, rows, S, ro, acc, red);
    if (e != cudaSuccess) return e;
    add_launches(1);
  }
  return cudaSuccess;
}
}  // namespace

size_t redundancy_ws_bytes(int H, int Lk, int d) {
  (void)Lk;
  return align_up((size_t)H * (d + 1) * sizeof(long long), 256);
}

int redundancy_max_lk() { return kMaxLk; }

cudaError_t launch_redundancy(const void* k, bool bf16, int H, int Lk, int d, float* red,
                              void* ws, cudaStream_t s, int ldk) {
  if (ldk <= 0) ldk = Lk;
  if (Lk > kMaxLk) return cudaErrorInvalidValue;
  if (bf16) {
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    return d == 128 ? run<__nv_bfloat16, 128>(kb, H, Lk, ldk, red, ws, s)
                    : run<__nv_bfloat16, 64>(kb, H, Lk, ldk, red, ws, s);
  }
  const float* kf = static_cast<const float*>(k);
  return d == 128 ? run<float, 128>(kf, H, Lk, ldk, red, ws, s)
                  : run<float, 64>(kf, H, Lk, ldk, red, ws, s);
}

}  // namespace fc

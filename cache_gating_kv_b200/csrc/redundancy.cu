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
// One kernel, one thread-block cluster per head (8 or 16 CTAs, each owning a
// contiguous slice of the head's rows):
//   1. every CTA sums khat over its rows; the partial d-vectors are exchanged
//      through distributed shared memory and every CTA adds them in rank order
//      (identical s everywhere, deterministic);
//   2. every CTA re-reads its rows backwards (the last ones read are still in
//      L2), forms r_j and
//      e_j = exp(r_j), writes e_j, and the per-CTA sums of e_j are exchanged
//      the same way;
//   3. every CTA scales its rows by 1/sum_j e_j.
// The cluster barriers are hardware barriers (no spin loops).  Each lane
// holds two 16-byte vectors of a row (16 bf16 or 8 fp32 elements), so a row's
// reductions take log2(d*elem/32) shuffles; the per-row scalars use the
// special-function unit (rsqrt, ex2: ~2^-22 relative error); every lane keeps
// two or four rows' loads in flight.
#include <cooperative_groups.h>

#include "fc_common.cuh"
#include "fc_kernels.h"

namespace cg = cooperative_groups;

namespace fc {

namespace {
constexpr int kRedThreads = 256;
constexpr int kRedWarps = kRedThreads / 32;

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

template <typename T, int D, int U>
__device__ __forceinline__ void load_rows(const T* kh, int r0, int hi, int sub, int cl,
                                          uint4 (&u)[U][2]) {
  using L = RowLayout<T, D>;
#pragma unroll
  for (int i = 0; i < U; ++i) {
    const int r = r0 + i * L::RPW + sub;
    const T* p = kh + (size_t)r * D + cl * L::EPL;
    u[i][0] = r < hi ? ld_nc_v4(p) : make_uint4(0u, 0u, 0u, 0u);
    u[i][1] = r < hi ? ld_nc_v4(p + Vec16<T>::N) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T, int D>
__device__ __forceinline__ void unpack(const uint4 (&u)[2], float* e) {
  Vec16<T>::to_float(u[0], e);
  Vec16<T>::to_float(u[1], e + Vec16<T>::N);
}

// U: rows in flight per lane (two 16-byte loads each).
template <typename T, int D, int U>
__global__ void __launch_bounds__(kRedThreads)
    red_cluster_kernel(const T* __restrict__ k, int Lk, int ldk, int h0, float* __restrict__ red) {
  using L = RowLayout<T, D>;
  cg::cluster_group cluster = cg::this_cluster();
  const int nrank = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int h = h0 + blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / L::LPR, cl = lane % L::LPR;
  const int per = (int)ceil_div(Lk, nrank);
  const int lo = min(Lk, rank * per), hi = min(Lk, lo + per);
  const T* kh = k + (size_t)h * ldk * D;
  constexpr int kRowsPerIter = kRedWarps * L::RPW * U;

  __shared__ float s_acc[kRedWarps][D];
  __shared__ float s_part[D];  // this CTA's sum of khat (read by the whole cluster)
  __shared__ float s_vec[D];   // the head's s
  __shared__ double s_esum[kRedWarps];
  __shared__ double s_epart;   // this CTA's sum of e (read by the whole cluster)
  __shared__ float s_inv;

  // ---- 1. sum of the normalised rows --------------------------------------
  float acc[L::EPL];
#pragma unroll
  for (int i = 0; i < L::EPL; ++i) acc[i] = 0.0f;
  for (int r0 = lo + warp * L::RPW * U; r0 < hi; r0 += kRowsPerIter) {
    uint4 raw[U][2];
    load_rows<T, D, U>(kh, r0, hi, sub, cl, raw);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float e[L::EPL];
      unpack<T, D>(raw[u], e);
      float n2 = 0.0f;
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) n2 = fmaf(e[i], e[i], n2);
      n2 = row_sum<L::LPR>(n2);
      const float inv = inv_norm(n2);  // a zero key stays zero
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) acc[i] = fmaf(e[i], inv, acc[i]);
    }
  }
#pragma unroll
  for (int o = L::LPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (sub == 0) {
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) s_acc[warp][cl * L::EPL + i] = acc[i];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kRedThreads) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kRedWarps; ++w) t += s_acc[w][c];
    s_part[c] = t;
  }
  cluster.sync();
  for (int c = threadIdx.x; c < D; c += kRedThreads) {
    double t = 0.0;
    for (int q = 0; q < nrank; ++q) t += (double)*cluster.map_shared_rank(&s_part[c], q);
    s_vec[c] = (float)t;
  }
  __syncthreads();

  // ---- 2. logits r_j and e_j = exp(r_j) -------------------------------------
  float sv[L::EPL];
#pragma unroll
  for (int i = 0; i < L::EPL; ++i) sv[i] = s_vec[cl * L::EPL + i];
  const float inv_lk = 1.0f / (float)Lk;
  float* rh = red + (size_t)h * Lk;
  double esum = 0.0;
  // Backwards over the slice: the rows read last by step 1 come first, while
  // they are still in L2.
  const int n_iter = (int)ceil_div(hi - lo, kRowsPerIter);
  for (int it = n_iter - 1; it >= 0; --it) {
    const int r0 = lo + it * kRowsPerIter + warp * L::RPW * U;
    uint4 raw[U][2];
    load_rows<T, D, U>(kh, r0, hi, sub, cl, raw);
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
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kRedWarps; ++w) t += s_esum[w];
    s_epart = t;
  }
  cluster.sync();
  if (threadIdx.x == 0) {
    double z = 0.0;
    for (int q = 0; q < nrank; ++q) z += *cluster.map_shared_rank(&s_epart, q);
    s_inv = (float)(1.0 / z);
  }
  cluster.sync();  // no CTA leaves while another may still read its shared memory

  // ---- 3. normalise this CTA's rows ----------------------------------------------
  const float inv = s_inv;
  for (int r = lo + threadIdx.x; r < hi; r += kRedThreads) rh[r] = rh[r] * inv;
}

template <typename T, int D>
cudaError_t run(const T* k, int H, int Lk, int ldk, float* red, cudaStream_t s) {
  // 16 CTAs per head when the slices stay long enough, else the portable 8.
  const int csize = (Lk >= 16 * 64) ? 16 : 8;
  // Long heads keep four rows per lane in flight (two measured 17 % slower at
  // L_k = 131072); short ones two (four measured 17 % slower at 16384).
  auto kern = Lk >= 65536 ? red_cluster_kernel<T, D, 4> : red_cluster_kernel<T, D, 2>;
  if (csize > 8) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)csize, (unsigned)H, 1);
  cfg.blockDim = dim3(kRedThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, k, Lk, ldk, 0, red);
  if (e != cudaSuccess) return e;
  add_launches(1);
  return cudaSuccess;
}
}  // namespace

size_t redundancy_ws_bytes(int H, int d) {
  (void)H;
  (void)d;
  return 256;  // the fused kernel keeps its partial sums in (distributed) shared memory
}

cudaError_t launch_redundancy(const void* k, bool bf16, int H, int Lk, int d, float* red,
                              void* ws, cudaStream_t s, int ldk) {
  (void)ws;
  if (ldk <= 0) ldk = Lk;
  if (bf16) {
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    return d == 128 ? run<__nv_bfloat16, 128>(kb, H, Lk, ldk, red, s)
                    : run<__nv_bfloat16, 64>(kb, H, Lk, ldk, red, s);
  }
  const float* kf = static_cast<const float*>(k);
  return d == 128 ? run<float, 128>(kf, H, Lk, ldk, red, s) : run<float, 64>(kf, H, Lk, ldk, red, s);
}

}  // namespace fc

// Importance on CUDA cores (float32 inputs, or bf16 inputs without the
// tensor-core path).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp_j = (1/L_q) sum_q softmax_j(q.k_j / sqrt(d)), the
// attention of the denoising queries over the clean keys averaged over the
// queries.
//
// Two passes, both tiled 64 x 64 with a 4 x 4 register tile per thread:
//   pass 1  one thread-block cluster of C1 CTAs per (query tile, head): CTA r
//           streams the r-th share of the key tiles and keeps a running
//           (max, sum) per row in the log2 domain; CTA 0 merges the C1 pairs
//           of each row over distributed shared memory, in rank order, and
//           stores lse2_q = log2 sum_j 2^(c*s_qj) with c = scale*log2(e)
//   pass 2  one cluster of C2 CTAs per (key tile, head): CTA r streams the
//           r-th share of the query tiles and accumulates 2^(c*s_qj - lse2_q)
//           per key; CTA 0 adds the C2 partial sums in rank order and divides
//           by L_q.  No atomics: each cluster owns its rows or keys.
// C1 and C2 (at most 8) spread small problems over the SMs (the 2-head
// parity case has 8 query tiles and 32 key tiles in all); they depend only on
// the problem's size, so the result is the same on every run.  float32
// accumulation throughout; exp2f / log2f are the accurate library functions
// (this path carries the float32 tolerance).
#include <cooperative_groups.h>

#include <algorithm>

#include "fc_common.cuh"
#include "fc_kernels.h"

namespace cg = cooperative_groups;

namespace fc {

namespace {
constexpr int kT = 64;
constexpr int kPad = 68;  // padded row of the transposed tiles (keeps float4 alignment)
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

// dst[c][r] = src[row0 + r][c] for r < 64 (zero beyond `valid` rows).
template <typename T, int D>
__device__ __forceinline__ void load_tile_t(float* __restrict__ dst, const T* __restrict__ src,
                                            int valid) {
  constexpr int EPL = Vec16<T>::N;
  constexpr int VPR = D / EPL;  // 16-byte vectors per row
  for (int i = threadIdx.x; i < kT * VPR; i += kThreads) {
    const int r = i % kT, cv = i / kT;
    float e[EPL];
    if (r < valid) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + (size_t)r * D + cv * EPL);
      Vec16<T>::to_float(u, e);
    } else {
#pragma unroll
      for (int x = 0; x < EPL; ++x) e[x] = 0.0f;
    }
#pragma unroll
    for (int x = 0; x < EPL; ++x) dst[(cv * EPL + x) * kPad + r] = e[x];
  }
}

template <int D>
__device__ __forceinline__ void tile_dot(const float* __restrict__ As, const float* __restrict__ Bs,
                                         int ty, int tx, float (&acc)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
#pragma unroll 8
  for (int kk = 0; kk < D; ++kk) {
    const float4 a = *reinterpret_cast<const float4*>(As + kk * kPad + ty * 4);
    const float4 b = *reinterpret_cast<const float4*>(Bs + kk * kPad + tx * 4);
    const float av[4] = {a.x, a.y, a.z, a.w};
    const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// (max, sum) of two partial log2-domain sums merged; -inf max means empty.
__device__ __forceinline__ void merge_ml(float& m, float& l, float mo, float lo) {
  const float mn = fmaxf(m, mo);
  if (mn != -INFINITY) {
    const float a = (m == -INFINITY) ? 0.0f : l * exp2f(m - mn);
    const float b = (mo == -INFINITY) ? 0.0f : lo * exp2f(mo - mn);
    l = a + b;
    m = mn;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    imp_lse_simt(const T* __restrict__ q, const T* __restrict__ k, int Lq, int Lk, int ldk,
                 float c2,
                 float* __restrict__ lse2) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = sm + D * kPad;
  __shared__ float2 s_ml[kT];  // this CTA's (max, sum) per row of the query tile
  cg::cluster_group cluster = cg::this_cluster();
  const int nr = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const int h = blockIdx.y, q0 = (blockIdx.x / nr) * kT;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int nkt = (int)ceil_div(Lk, kT), per = (int)ceil_div(nkt, nr);
  const int kt0 = rank * per, kt1 = min(nkt, kt0 + per);
  load_tile_t<T, D>(Qs, q + ((size_t)h * Lq + q0) * D, min(kT, Lq - q0));
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
  }
  for (int k0 = kt0 * kT; k0 < kt1 * kT; k0 += kT) {
    __syncthreads();
    load_tile_t<T, D>(Ks, k + ((size_t)h * ldk + k0) * D, min(kT, Lk - k0));
    __syncthreads();
    float acc[4][4];
    tile_dot<D>(Qs, Ks, ty, tx, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[4];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        t[j] = (k0 + tx * 4 + j < Lk) ? acc[i][j] * c2 : -INFINITY;
        mx = fmaxf(mx, t[j]);
      }
      if (mx > m[i]) {
        if (m[i] != -INFINITY) l[i] *= exp2f(m[i] - mx);
        m[i] = mx;
      }
      if (m[i] != -INFINITY) {
#pragma unroll
        for (int j = 0; j < 4; ++j) l[i] += exp2f(t[j] - m[i]);
      }
    }
  }
  // Merge the 16 column slices of each row (lanes tx = 0..15 of a half-warp).
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[i], o);
      const float lo = __shfl_xor_sync(0xffffffffu, l[i], o);
      merge_ml(m[i], l[i], mo, lo);
    }
    if (tx == 0) s_ml[ty * 4 + i] = make_float2(m[i], l[i]);
  }
  cluster.sync();
  // CTA 0 merges the cluster's key shares of each row, in rank order.
  if (rank == 0 && threadIdx.x < kT) {
    float2 ml = s_ml[threadIdx.x];
    for (int r = 1; r < nr; ++r) {
      const float2 o = *cluster.map_shared_rank(&s_ml[threadIdx.x], r);
      merge_ml(ml.x, ml.y, o.x, o.y);
    }
    const int row = q0 + threadIdx.x;
    if (row < Lq) lse2[(size_t)h * Lq + row] = ml.x + log2f(ml.y);
  }
  cluster.sync();  // no CTA leaves while CTA 0 may still read its shared memory
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    imp_col_simt(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse2,
                 int Lq, int Lk, int ldk, float c2, float* __restrict__ imp) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Qs = sm + D * kPad;
  float* sl = sm + 2 * D * kPad;  // [64] row normalisers of the query tile
  __shared__ float s_col[kT];     // this CTA's column sums of the key tile
  cg::cluster_group cluster = cg::this_cluster();
  const int nr = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const int h = blockIdx.y, k0 = (blockIdx.x / nr) * kT;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int nqt = (int)ceil_div(Lq, kT), per = (int)ceil_div(nqt, nr);
  const int qt0 = rank * per, qt1 = min(nqt, qt0 + per);
  load_tile_t<T, D>(Ks, k + ((size_t)h * ldk + k0) * D, min(kT, Lk - k0));
  float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int q0 = qt0 * kT; q0 < qt1 * kT; q0 += kT) {
    __syncthreads();
    load_tile_t<T, D>(Qs, q + ((size_t)h * Lq + q0) * D, min(kT, Lq - q0));
    if (threadIdx.x < kT) {
      const int row = q0 + threadIdx.x;
      sl[threadIdx.x] = row < Lq ? lse2[(size_t)h * Lq + row] : INFINITY;  // padded rows give 0
    }
    __syncthreads();
    float acc[4][4];
    tile_dot<D>(Qs, Ks, ty, tx, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float L = sl[ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) cs[j] += exp2f(acc[i][j] * c2 - L);
    }
  }
  __syncthreads();
  float* red = sm;  // reuse: [16][64]
#pragma unroll
  for (int j = 0; j < 4; ++j) red[ty * kT + tx * 4 + j] = cs[j];
  __syncthreads();
  if (threadIdx.x < kT) {
    float t = 0.0f;
#pragma unroll
    for (int y = 0; y < 16; ++y) t += red[y * kT + threadIdx.x];
    s_col[threadIdx.x] = t;
  }
  cluster.sync();
  // CTA 0 adds the cluster's query shares of each key, in rank order.
  if (rank == 0 && threadIdx.x < kT) {
    float t = s_col[threadIdx.x];
    for (int r = 1; r < nr; ++r) t += *cluster.map_shared_rank(&s_col[threadIdx.x], r);
    const int key = k0 + threadIdx.x;
    if (key < Lk) imp[(size_t)h * Lk + key] = t / (float)Lq;
  }
  cluster.sync();  // no CTA leaves while CTA 0 may still read its shared memory
}

// CTAs per cluster for `units` (tile, head) pairs each splittable into `tiles`
// shares: enough to give about two CTAs per SM, at most 8 (the portable
// cluster size) and at most one share per tile.
int cluster_split(int64_t units, int tiles) {
  const int64_t want = ceil_div(2 * (int64_t)sm_count(), units);
  return (int)std::max<int64_t>(1, std::min<int64_t>({want, (int64_t)tiles, 8}));
}

template <typename K, typename... Args>
cudaError_t launch_clustered(K kern, int nx, int H, int csize, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nx * csize), (unsigned)H, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename T, int D>
cudaError_t run(const T* q, const T* k, int H, int Lq, int Lk, int ldk, float scale, float* imp,
                float* lse2, cudaStream_t s) {
  const float c2 = scale * kLog2e;
  const size_t smem1 = (size_t)2 * D * kPad * sizeof(float);
  const size_t smem2 = smem1 + kT * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(imp_lse_simt<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(imp_col_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem2);
  if (e != cudaSuccess) return e;
  const int nqt = (int)ceil_div(Lq, kT), nkt = (int)ceil_div(Lk, kT);
  const int c1 = cluster_split((int64_t)nqt * H, nkt);
  const int cc2 = cluster_split((int64_t)nkt * H, nqt);
  e = launch_clustered(imp_lse_simt<T, D>, nqt, H, c1, smem1, s, q, k, Lq, Lk, ldk, c2, lse2);
  if (e != cudaSuccess) return e;
  e = launch_clustered(imp_col_simt<T, D>, nkt, H, cc2, smem2, s, q, k, (const float*)lse2, Lq,
                       Lk, ldk, c2, imp);
  if (e != cudaSuccess) return e;
  add_launches(2);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_importance_simt(const void* q, const void* k, bool bf16, int H, int Lq, int Lk,
                                   int d, float scale, float* imp, void* ws, cudaStream_t s,
                                   int ldk) {
  if (ldk <= 0) ldk = Lk;
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);  // after the error word
  if (bf16) {
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    return d == 128 ? run<__nv_bfloat16, 128>(qb, kb, H, Lq, Lk, ldk, scale, imp, lse2, s)
                    : run<__nv_bfloat16, 64>(qb, kb, H, Lq, Lk, ldk, scale, imp, lse2, s);
  }
  const auto* qf = static_cast<const float*>(q);
  const auto* kf = static_cast<const float*>(k);
  return d == 128 ? run<float, 128>(qf, kf, H, Lq, Lk, ldk, scale, imp, lse2, s)
                  : run<float, 64>(qf, kf, H, Lq, Lk, ldk, scale, imp, lse2, s);
}

}  // namespace fc

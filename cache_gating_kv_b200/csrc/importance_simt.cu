// Importance on CUDA cores (float32 inputs, or bf16 inputs without the
// tensor-core path).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp_j = (1/L_q) sum_q softmax_j(q.k_j / sqrt(d)), the
// attention of the denoising queries over the clean keys averaged over the
// queries.
//
// Two passes, both tiled 64 x 64 with a 4 x 4 register tile per thread:
//   pass 1  grid (L_q/64, H): for a query tile, stream every key tile and keep
//           a running (max, sum) per row in the log2 domain; store
//           lse2_q = log2 sum_j 2^(c*s_qj) with c = scale*log2(e)
//   pass 2  grid (L_k/64, H): for a key tile, stream every query tile and
//           accumulate 2^(c*s_qj - lse2_q) per key; fixed-order reduction at
//           the end, divided by L_q.  No atomics: each block owns its keys.
// float32 accumulation throughout; exp2f / log2f are the accurate library
// functions (this path carries the float32 tolerance).
#include "fc_common.cuh"
#include "fc_kernels.h"

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

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    imp_lse_simt(const T* __restrict__ q, const T* __restrict__ k, int Lq, int Lk, int ldk,
                 float c2,
                 float* __restrict__ lse2) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = sm + D * kPad;
  const int h = blockIdx.y, q0 = blockIdx.x * kT;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  load_tile_t<T, D>(Qs, q + ((size_t)h * Lq + q0) * D, min(kT, Lq - q0));
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
  }
  for (int k0 = 0; k0 < Lk; k0 += kT) {
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
      const float mn = fmaxf(m[i], mo);
      if (mn != -INFINITY) {
        const float a = (m[i] == -INFINITY) ? 0.0f : l[i] * exp2f(m[i] - mn);
        const float b = (mo == -INFINITY) ? 0.0f : lo * exp2f(mo - mn);
        l[i] = a + b;
        m[i] = mn;
      }
    }
    const int row = q0 + ty * 4 + i;
    if (tx == 0 && row < Lq) lse2[(size_t)h * Lq + row] = m[i] + log2f(l[i]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    imp_col_simt(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse2,
                 int Lq, int Lk, int ldk, float c2, float* __restrict__ imp) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Qs = sm + D * kPad;
  float* sl = sm + 2 * D * kPad;  // [64] row normalisers of the query tile
  const int h = blockIdx.y, k0 = blockIdx.x * kT;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  load_tile_t<T, D>(Ks, k + ((size_t)h * ldk + k0) * D, min(kT, Lk - k0));
  float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int q0 = 0; q0 < Lq; q0 += kT) {
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
    const int key = k0 + threadIdx.x;
    if (key < Lk) imp[(size_t)h * Lk + key] = t / (float)Lq;
  }
}

template <typename T, int D>
cudaError_t run(const T* q, const T* k, int H, int Lq, int Lk, int ldk, float scale, float* imp,
                float* lse2, cudaStream_t s) {
  const float c2 = scale * kLog2e;
  const size_t smem1 = (size_t)2 * D * kPad * sizeof(float);
  const size_t smem2 = smem1 + kT * sizeof(float);
  cudaFuncSetAttribute(imp_lse_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem1);
  cudaFuncSetAttribute(imp_col_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem2);
  imp_lse_simt<T, D><<<dim3((unsigned)ceil_div(Lq, kT), H), kThreads, smem1, s>>>(q, k, Lq, Lk,
                                                                                  ldk, c2, lse2);
  imp_col_simt<T, D><<<dim3((unsigned)ceil_div(Lk, kT), H), kThreads, smem2, s>>>(
      q, k, lse2, Lq, Lk, ldk, c2, imp);
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

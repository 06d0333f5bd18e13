// Redundancy of every clean key, per head, as an HBM stream over K.
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Red_j = softmax_j((1/L_k) sum_i S_ij), S the cosine
// similarity of l2-normalised keys with its diagonal set to zero.
//
// The L_k x L_k matrix is never formed.  With s = sum_i khat_i,
//   sum_{i != j} khat_i . khat_j = khat_j . s - ||khat_j||^2      (exact)
// so the logits r_j need one reduction pass over K and one dot pass.  r_j lies
// in [-1, 1], hence exp(r_j) cannot overflow and the softmax needs no max.
//
//   pass A  grid (blocks_per_head, H): normalise rows, per-block partial s
//   pass B  same grid: fixed-order sum of the partials -> s, then for every
//           row r_j and e_j = exp(r_j) (written to red), per-block partial sum
//   pass C  grid over H x L_k: fixed-order sum of the partials -> Z, red = e/Z
// Each 16-byte lane vector holds 8 bf16 or 4 fp32 elements; a row of d
// elements is spread over d*elem/16 lanes of a warp, so loads are coalesced
// 16-byte vectors and every reduction runs in a fixed order (deterministic).
#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

namespace {
constexpr int kRedThreads = 256;
constexpr int kRedWarps = kRedThreads / 32;
constexpr int kRedMaxBlocksPerHead = 512;

template <typename T, int D>
struct RowLayout {
  static constexpr int EPL = Vec16<T>::N;        // elements per lane
  static constexpr int LPR = D / EPL;            // lanes per row
  static constexpr int RPW = 32 / LPR;           // rows per warp step
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row layout");
};

// Sum over the LPR lanes that hold one row (xor offsets below LPR stay inside
// the row's lane group).
template <int LPR>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void block_rows(int Lk, int bph, int b, int& lo, int& hi) {
  const int per = (int)ceil_div(Lk, bph);
  lo = min(Lk, per * b);
  hi = min(Lk, lo + per);
}

// Pass A: partial_s[h][b][:] = sum over this block's rows of khat.
template <typename T, int D>
__global__ void __launch_bounds__(kRedThreads)
    red_sum_kernel(const T* __restrict__ k, int Lk, int bph, float* __restrict__ partial_s) {
  using L = RowLayout<T, D>;
  const int h = blockIdx.y, b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / L::LPR, cl = lane % L::LPR;
  int lo, hi;
  block_rows(Lk, bph, b, lo, hi);
  const T* kh = k + (size_t)h * Lk * D;

  float acc[L::EPL];
#pragma unroll
  for (int i = 0; i < L::EPL; ++i) acc[i] = 0.0f;
  for (int r0 = lo + warp * L::RPW; r0 < hi; r0 += kRedWarps * L::RPW) {
    const int r = r0 + sub;
    const bool valid = r < hi;
    float e[L::EPL];
    if (valid) {
      const uint4 u = ld_nc_v4(kh + (size_t)r * D + cl * L::EPL);
      Vec16<T>::to_float(u, e);
    } else {
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) e[i] = 0.0f;
    }
    float n2 = 0.0f;
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) n2 = fmaf(e[i], e[i], n2);
    n2 = row_sum<L::LPR>(n2);
    const float inv = 1.0f / fmaxf(sqrtf(n2), 1e-12f);  // a zero key stays zero
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) acc[i] = fmaf(e[i], inv, acc[i]);
  }
  // Reduce the rows of the warp: lanes with equal cl hold the same columns.
#pragma unroll
  for (int o = L::LPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  __shared__ float s_acc[kRedWarps][D];
  if (sub == 0) {
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) s_acc[warp][cl * L::EPL + i] = acc[i];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kRedThreads) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kRedWarps; ++w) t += s_acc[w][c];
    partial_s[((size_t)h * bph + b) * D + c] = t;
  }
}

// Pass B: s = fixed-order sum of the partials, then e_j = exp(r_j) for this
// block's rows; partial_e[h][b] = sum of this block's e_j.
template <typename T, int D>
__global__ void __launch_bounds__(kRedThreads)
    red_dot_kernel(const T* __restrict__ k, int Lk, int bph, const float* __restrict__ partial_s,
                   float* __restrict__ e_out, double* __restrict__ partial_e) {
  using L = RowLayout<T, D>;
  const int h = blockIdx.y, b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / L::LPR, cl = lane % L::LPR;
  __shared__ float s_vec[D];
  for (int c = threadIdx.x; c < D; c += kRedThreads) {
    double t = 0.0;
    for (int i = 0; i < bph; ++i) t += (double)partial_s[((size_t)h * bph + i) * D + c];
    s_vec[c] = (float)t;
  }
  __syncthreads();
  float sv[L::EPL];
#pragma unroll
  for (int i = 0; i < L::EPL; ++i) sv[i] = s_vec[cl * L::EPL + i];

  int lo, hi;
  block_rows(Lk, bph, b, lo, hi);
  const T* kh = k + (size_t)h * Lk * D;
  const float inv_lk = 1.0f / (float)Lk;
  double esum = 0.0;
  for (int r0 = lo + warp * L::RPW; r0 < hi; r0 += kRedWarps * L::RPW) {
    const int r = r0 + sub;
    const bool valid = r < hi;
    float e[L::EPL];
    if (valid) {
      const uint4 u = ld_nc_v4(kh + (size_t)r * D + cl * L::EPL);
      Vec16<T>::to_float(u, e);
    } else {
#pragma unroll
      for (int i = 0; i < L::EPL; ++i) e[i] = 0.0f;
    }
    float n2 = 0.0f, dot = 0.0f;
#pragma unroll
    for (int i = 0; i < L::EPL; ++i) {
      n2 = fmaf(e[i], e[i], n2);
      dot = fmaf(e[i], sv[i], dot);
    }
    n2 = row_sum<L::LPR>(n2);
    dot = row_sum<L::LPR>(dot);
    const float inv = 1.0f / fmaxf(sqrtf(n2), 1e-12f);
    // r_j = (khat_j . s - ||khat_j||^2) / L_k
    const float rj = (dot * inv - n2 * inv * inv) * inv_lk;
    const float ej = expf(rj);
    if (valid && cl == 0) {
      e_out[(size_t)h * Lk + r] = ej;
      esum += (double)ej;
    }
  }
  esum = warp_sum(esum);
  __shared__ double s_e[kRedWarps];
  if (lane == 0) s_e[warp] = esum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kRedWarps; ++w) t += s_e[w];
    partial_e[(size_t)h * bph + b] = t;
  }
}

// Pass C: red = e / sum_j e_j.
__global__ void __launch_bounds__(kRedThreads)
    red_norm_kernel(float* __restrict__ red, int Lk, int bph, const double* __restrict__ partial_e) {
  const int h = blockIdx.y;
  __shared__ float s_inv;
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < bph; ++i) t += partial_e[(size_t)h * bph + i];
    s_inv = (float)(1.0 / t);
  }
  __syncthreads();
  const float inv = s_inv;
  float* rh = red + (size_t)h * Lk;
  for (int j = blockIdx.x * kRedThreads + threadIdx.x; j < Lk; j += gridDim.x * kRedThreads)
    rh[j] = rh[j] * inv;
}

template <typename T, int D>
cudaError_t run(const T* k, int H, int Lk, float* red, char* ws, cudaStream_t s) {
  using L = RowLayout<T, D>;
  int bph = (int)ceil_div((int64_t)sm_count() * 4, H);
  const int min_rows = kRedWarps * L::RPW * 4;  // at least four warp steps per block
  bph = min(bph, (int)ceil_div(Lk, min_rows));
  bph = max(1, min(bph, kRedMaxBlocksPerHead));
  float* partial_s = reinterpret_cast<float*>(ws);
  double* partial_e = reinterpret_cast<double*>(
      ws + align_up((size_t)H * kRedMaxBlocksPerHead * D * sizeof(float), 256));
  dim3 grid(bph, H);
  red_sum_kernel<T, D><<<grid, kRedThreads, 0, s>>>(k, Lk, bph, partial_s);
  red_dot_kernel<T, D><<<grid, kRedThreads, 0, s>>>(k, Lk, bph, partial_s, red, partial_e);
  const int64_t nbc = ceil_div(Lk, kRedThreads);
  dim3 gridc((unsigned)(nbc < 64 ? nbc : 64), H);
  red_norm_kernel<<<gridc, kRedThreads, 0, s>>>(red, Lk, bph, partial_e);
  return cudaGetLastError();
}
}  // namespace

size_t redundancy_ws_bytes(int H, int d) {
  return align_up((size_t)H * kRedMaxBlocksPerHead * d * sizeof(float), 256) +
         (size_t)H * kRedMaxBlocksPerHead * sizeof(double);
}

cudaError_t launch_redundancy(const void* k, bool bf16, int H, int Lk, int d, float* red,
                              void* ws, cudaStream_t s) {
  char* w = static_cast<char*>(ws);
  if (bf16) {
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    return d == 128 ? run<__nv_bfloat16, 128>(kb, H, Lk, red, w, s)
                    : run<__nv_bfloat16, 64>(kb, H, Lk, red, w, s);
  }
  const float* kf = static_cast<const float*>(k);
  return d == 128 ? run<float, 128>(kf, H, Lk, red, w, s) : run<float, 64>(kf, H, Lk, red, w, s);
}

}  // namespace fc

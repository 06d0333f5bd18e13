// Consumer of the gate's recompute mask: gather the recompute chunks into a
// dense batch for the model forward, and scatter the fresh velocities back
// into the per-chunk velocity cache (reuse chunks keep their cached one).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// flowchart of 整体框架 and 关键设计 2: chunks whose accumulator crosses the
// threshold recompute their forward; the others reuse cached activations.
//
// Pure data movement, bound by HBM.  Each block finds the chunk of its slot
// itself (a warp ballot scan of the mask, n_chunks bytes), so gather and
// scatter are one launch each with no host round trip: the recompute count
// stays on the device.
#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

namespace {
constexpr int kMoveThreads = 256;
constexpr int kMoveVec = 4;  // float4 per thread per block tile
constexpr int64_t kMoveTile = (int64_t)kMoveThreads * kMoveVec * 4;  // floats per block

// The chunk index of dense slot `slot` (the slot-th set mask byte), or -1,
// and the number of set bytes.  Warp-wide; every lane gets the results.
__device__ __forceinline__ void slot_chunk(const uint8_t* __restrict__ mask, int n_c, int slot,
                                           int& src, int& total) {
  const int lane = threadIdx.x & 31;
  src = -1;
  total = 0;
  for (int base = 0; base < n_c; base += 32) {
    const int c = base + lane;
    const unsigned bits = __ballot_sync(0xffffffffu, c < n_c && mask[c] != 0);
    const int cnt = __popc(bits);
    if (src < 0 && slot >= total && slot < total + cnt) {
      unsigned b = bits;
      for (int k = 0; k < slot - total; ++k) b &= b - 1;  // drop the lower set bits
      src = base + __ffs(b) - 1;
    }
    total += cnt;
  }
}

__device__ __forceinline__ void copy_range(const float* __restrict__ src, float* __restrict__ dst,
                                           int64_t N, int64_t lo, int64_t hi) {
  const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
  if (vec) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* d4 = reinterpret_cast<float4*>(dst);
    const int64_t l4 = lo >> 2, h4 = hi >> 2;  // lo is a multiple of 4
    float4 buf[kMoveVec];
#pragma unroll
    for (int u = 0; u < kMoveVec; ++u) {
      const int64_t i = l4 + threadIdx.x + (int64_t)u * kMoveThreads;
      if (i < h4) buf[u] = __ldcs(s4 + i);
    }
#pragma unroll
    for (int u = 0; u < kMoveVec; ++u) {
      const int64_t i = l4 + threadIdx.x + (int64_t)u * kMoveThreads;
      if (i < h4) d4[i] = buf[u];
    }
    for (int64_t e = (h4 << 2) + threadIdx.x; e < hi; e += kMoveThreads) dst[e] = src[e];
  } else {
    for (int64_t e = lo + threadIdx.x; e < hi; e += kMoveThreads) dst[e] = src[e];
  }
}

__global__ void __launch_bounds__(kMoveThreads)
    gather_kernel(const float* __restrict__ x, const uint8_t* __restrict__ mask, int n_c,
                  int64_t N, float* __restrict__ dense, int32_t* __restrict__ ids,
                  int32_t* __restrict__ count) {
  __shared__ int s_src;
  const int slot = blockIdx.y;
  if (threadIdx.x < 32) {
    int src, total;
    slot_chunk(mask, n_c, slot, src, total);
    if (threadIdx.x == 0) {
      s_src = src;
      if (blockIdx.x == 0) {
        ids[slot] = src;
        if (slot == 0) *count = total;
      }
    }
  }
  __syncthreads();
  const int src = s_src;
  if (src < 0) return;  // no recompute chunk for this slot: the row is left as it was
  const int64_t lo = (int64_t)blockIdx.x * kMoveTile, hi = min(N, lo + kMoveTile);
  if (lo >= hi) return;
  copy_range(x + (size_t)src * N, dense + (size_t)slot * N, N, lo, hi);
}

__global__ void __launch_bounds__(kMoveThreads)
    scatter_kernel(const float* __restrict__ v_dense, const int32_t* __restrict__ ids,
                   const int32_t* __restrict__ count, int n_c, int64_t N,
                   float* __restrict__ v_cache) {
  const int slot = blockIdx.y;
  const int64_t lo = (int64_t)blockIdx.x * kMoveTile, hi = min(N, lo + kMoveTile);
  if (lo >= hi) return;
  const float* src = v_dense + (size_t)slot * N;
  const bool vec = (N & 3) == 0 && ((reinterpret_cast<uintptr_t>(v_dense) |
                                     reinterpret_cast<uintptr_t>(v_cache)) & 15) == 0;
  if (vec) {
    // Whole 16-byte rows: the source tile is loaded before count and ids are
    // read (the slot's source row is known), so those dependent loads do not
    // hold up the stream; nothing is written before the slot is known valid.
    const float4* s4 = reinterpret_cast<const float4*>(src);
    const int64_t l4 = lo >> 2, h4 = hi >> 2;
    float4 buf[kMoveVec];
#pragma unroll
    for (int u = 0; u < kMoveVec; ++u) {
      const int64_t i = l4 + threadIdx.x + (int64_t)u * kMoveThreads;
      if (i < h4) buf[u] = __ldcs(s4 + i);
    }
    if (slot >= *count) return;
    const int dst = ids[slot];
    if (dst < 0 || dst >= n_c) return;
    float4* d4 = reinterpret_cast<float4*>(v_cache + (size_t)dst * N);
#pragma unroll
    for (int u = 0; u < kMoveVec; ++u) {
      const int64_t i = l4 + threadIdx.x + (int64_t)u * kMoveThreads;
      if (i < h4) d4[i] = buf[u];
    }
    return;
  }
  if (slot >= *count) return;
  const int dst = ids[slot];
  if (dst < 0 || dst >= n_c) return;
  copy_range(src, v_cache + (size_t)dst * N, N, lo, hi);
}
}  // namespace

cudaError_t launch_gather_recompute(const float* x, const uint8_t* mask, int n_c, int64_t N,
                                    float* dense, int32_t* ids, int32_t* count, cudaStream_t s) {
  const int64_t bx = N > 0 ? ceil_div(N, kMoveTile) : 1;
  gather_kernel<<<dim3((unsigned)bx, (unsigned)n_c), kMoveThreads, 0, s>>>(x, mask, n_c, N, dense,
                                                                          ids, count);
  add_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_scatter_velocity(const float* v_dense, const int32_t* ids, const int32_t* count,
                                    int n_c, int64_t N, float* v_cache, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  scatter_kernel<<<dim3((unsigned)ceil_div(N, kMoveTile), (unsigned)n_c), kMoveThreads, 0, s>>>(
      v_dense, ids, count, n_c, N, v_cache);
  add_launches(1);
  return cudaGetLastError();
}

}  // namespace fc

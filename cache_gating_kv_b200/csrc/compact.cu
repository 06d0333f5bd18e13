// Compaction of the kept K/V rows into the fixed-budget buffer.
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: the fixed buffer B_total is split into the compressed
// clean region B_budget and the active region; the top-B tokens of every head
// are kept in B_budget.
//
// A pure HBM gather: k_out[h][r] = k[h][idx[h][r]] and the same for V, the
// input heads ldk rows apart (L_k, or B_budget + C for a cache buffer) and the
// output heads ldo rows apart (B for a dense [H][B][d] result, B_budget + C
// when the kept rows land in the clean region of a cache buffer).  A row
// of d elements is d*elem/16 lanes of 16-byte vectors; each thread gathers
// four rows before storing them so that enough loads are in flight; grid z
// selects K or V.
#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

namespace {
constexpr int kCompactThreads = 256;
constexpr int kCompactUnroll = 4;

template <int LPR>
__global__ void __launch_bounds__(kCompactThreads)
    compact_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, int Lk, int ldk, int B,
                   int ldo, const int32_t* __restrict__ idx, uint4* __restrict__ ko,
                   uint4* __restrict__ vo) {
  grid_dep_wait();  // idx (and anything the kernel before touched) is ready
  grid_dep_launch();
  constexpr int RPW = 32 / LPR;
  constexpr int kRowsPerStep = (kCompactThreads / 32) * RPW;
  constexpr int kRowsPerBlock = kRowsPerStep * kCompactUnroll;
  const int h = blockIdx.y;
  const uint4* src = (blockIdx.z == 0 ? k : v) + (size_t)h * ldk * LPR;
  uint4* dst = (blockIdx.z == 0 ? ko : vo) + (size_t)h * ldo * LPR;
  const int32_t* ih = idx + (size_t)h * B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, cl = lane % LPR;
  const int r0 = blockIdx.x * kRowsPerBlock + warp * RPW + sub;
  uint4 buf[kCompactUnroll];
#pragma unroll
  for (int u = 0; u < kCompactUnroll; ++u) {
    const int r = r0 + u * kRowsPerStep;
    buf[u] = make_uint4(0u, 0u, 0u, 0u);
    if (r < B) {
      const int j = __ldg(ih + r);
      if (j >= 0 && j < Lk) buf[u] = __ldcs(src + (size_t)j * LPR + cl);
    }
  }
#pragma unroll
  for (int u = 0; u < kCompactUnroll; ++u) {
    const int r = r0 + u * kRowsPerStep;
    if (r < B) dst[(size_t)r * LPR + cl] = buf[u];
  }
}

template <int LPR>
cudaError_t run(const void* k, const void* v, int H, int Lk, int ldk, const int32_t* idx, int B,
                int ldo, void* ko, void* vo, cudaStream_t s) {
  constexpr int kRowsPerBlock = (kCompactThreads / 32) * (32 / LPR) * kCompactUnroll;
  dim3 grid((unsigned)ceil_div(B, kRowsPerBlock), H, 2);
  // a programmatic dependent: scheduled while the selection finishes
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kCompactThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, compact_kernel<LPR>, static_cast<const uint4*>(k), static_cast<const uint4*>(v), Lk,
      ldk, B, ldo, idx, static_cast<uint4*>(ko), static_cast<uint4*>(vo));
  if (e != cudaSuccess) return e;
  add_launches(1);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_compact(const void* k, const void* v, int elem_bytes, int H, int Lk, int d,
                           const int32_t* idx, int B, int ldo, void* k_out, void* v_out,
                           cudaStream_t s, int ldk) {
  if (ldk <= 0) ldk = Lk;
  const int row_bytes = d * elem_bytes;
  switch (row_bytes / 16) {
    case 8: return run<8>(k, v, H, Lk, ldk, idx, B, ldo, k_out, v_out, s);
    case 16: return run<16>(k, v, H, Lk, ldk, idx, B, ldo, k_out, v_out, s);
    case 32: return run<32>(k, v, H, Lk, ldk, idx, B, ldo, k_out, v_out, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc

// Importance on the 5th-generation tensor cores (bf16 inputs, fp32 accumulate).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp_j = (1/L_q) sum_q softmax_j(q.k_j / sqrt(d)) over
// the clean candidate keys.
//
// The L_q x L_k probability matrix is never stored.  Two passes recompute the
// logits with tcgen05.mma:
//   pass 1 (rows)     CTA = 128 queries of one head; streams every 128-key
//                     tile; D = Q K^T in TMEM; each of 128 epilogue threads
//                     owns one query row and keeps a running (max, sum) in the
//                     log2 domain -> lse2_q = log2 sum_j 2^(c s_qj),
//                     c = scale*log2(e).  Padded query rows get +inf.
//   pass 2 (columns)  CTA = 128 keys of one head; streams every 128-query tile;
//                     D = K Q^T in TMEM (keys on the TMEM lanes), so each
//                     epilogue thread owns one key and sums 2^(c s - lse2_q)
//                     over all queries in registers: no atomics, no partial
//                     buffers, deterministic.
// Roles (256 threads): warp 0 lane 0 issues TMA loads (3D tensor maps over
// [H][L][d], 128-byte swizzle, zero fill past L), warp 1 lane 0 issues the
// MMAs (M=128, N=128, K=16 steps), warp 2 owns the TMEM allocation (two
// 128-column fp32 accumulators: the MMA of tile t+1 overlaps the epilogue of
// tile t), warps 4-7 are the epilogue (warp w reads TMEM lanes 32(w%4)..+31).
// A 4-stage shared-memory ring of operand tiles decouples TMA from the MMAs.
// Every mbarrier wait is bounded; on timeout the kernel records an error word
// in the workspace and winds down (no trap, no endless spin).
#include <cuda.h>

#include "fc_common.cuh"
#include "fc_kernels.h"
#include "tc_ptx.cuh"

namespace fc {

namespace {
constexpr int kBM = 128;      // rows of the resident A tile (TMEM lanes)
constexpr int kBN = 128;      // rows of each streamed B tile (MMA N, TMEM columns)
constexpr int kStages = 4;    // shared-memory ring depth
constexpr int kThreads = 256;
constexpr int kHalf = kBM * 64 * 2;  // one 128 x 64 bf16 swizzled block (16 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kErrOffset = 0;      // error word in the workspace
constexpr size_t kLseOffset = 256;    // lse2 [H][Lq_pad] follows

template <int D>
constexpr int tile_bytes() {
  return (D / 64) * kHalf;
}
template <int D>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)(1 + kStages) * tile_bytes<D>() + 256 + kStages * kBN * sizeof(float);
}

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t a_full;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_slot;
};

// kPass 1: A = Q tile, B = K tiles, epilogue = row log-sum-exp.
// kPass 2: A = K tile, B = Q tiles, epilogue = column sums of 2^(c s - lse2).
template <int D, int kPass>
__global__ void __launch_bounds__(kThreads, 1)
    imp_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                  int Lq, int Lk, int lq_pad, float c2, float* __restrict__ lse2,
                  float* __restrict__ imp, int* __restrict__ err) {
  constexpr int KB = D / 64;
  constexpr int TB = tile_bytes<D>();
  constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kBM, kBN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + TB;
  Bars* bars = reinterpret_cast<Bars*>(sB + kStages * TB);
  float* sL = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // [kStages][kBN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int a0 = blockIdx.x * kBM;  // first row of the A tile
  const int nB = kPass == 1 ? (Lk + kBN - 1) / kBN : lq_pad / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      // pass 2: a stage also carries the query tile's lse2 values, so it is
      // released by the MMA commit and by each of the 4 epilogue warps
      tc::mbar_init(&bars->empty[s], kPass == 2 ? 5 : 1);
    }
    tc::mbar_init(&bars->a_full, 1);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars->acc_full[b], 1);
      tc::mbar_init(&bars->acc_empty[b], 4);
    }
    tc::fence_barrier_init();
  }
  if (warp == 2) tc::tmem_alloc(&bars->tmem_slot, 2 * kBN);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      tc::mbar_expect_tx(&bars->a_full, TB);
      for (int kb = 0; kb < KB; ++kb) tc::tma_load_3d(sA + kb * kHalf, &mapA, &bars->a_full, kb * 64, a0, h);
      for (int t = 0; t < nB; ++t) {
        const int s = t % kStages, u = t / kStages;
        if (!tc::mbar_wait(&bars->empty[s], (u & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc::mbar_expect_tx(&bars->full[s], TB + (kPass == 2 ? kBN * 4 : 0));
        for (int kb = 0; kb < KB; ++kb)
          tc::tma_load_3d(sB + s * TB + kb * kHalf, &mapB, &bars->full[s], kb * 64, t * kBN, h);
        if (kPass == 2)
          tc::bulk_load(sL + s * kBN, lse2 + (size_t)h * lq_pad + t * kBN, kBN * 4, &bars->full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      ok = tc::mbar_wait(&bars->a_full, 0);
      const uint32_t a_addr = tc::smem_u32(sA);
      for (int t = 0; ok && t < nB; ++t) {
        const int s = t % kStages, u = t / kStages, b = t & 1, v = t >> 1;
        if (!tc::mbar_wait(&bars->acc_empty[b], (v & 1) ^ 1) ||
            !tc::mbar_wait(&bars->full[s], u & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t b_addr = tc::smem_u32(sB + s * TB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;  // 16 bf16 = 32 bytes per step
          tc::mma_bf16(tmem + b * kBN, tc::desc_k_sw128(a_addr + off),
                       tc::desc_k_sw128(b_addr + off), kIdesc, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->empty[s]);     // operand stage reusable once read
        tc::mma_commit(&bars->acc_full[b]);  // accumulator b ready
      }
    }
  } else if (warp >= 4) {  // ---- epilogue warpgroup
    const int sub = warp & 3;
    const int row = a0 + sub * 32 + lane;  // this thread's A row (query or key)
    const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
    float m = -INFINITY, l = 0.0f;  // pass 1 state
    float acc0 = 0.0f, acc1 = 0.0f;  // pass 2 state (two chains)
    for (int t = 0; t < nB; ++t) {
      const int b = t & 1, v = t >> 1, s = t % kStages, u = t / kStages;
      if (!tc::mbar_wait(&bars->acc_full[b], v & 1) ||
          (kPass == 2 && !tc::mbar_wait(&bars->full[s], u & 1))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(lane_addr + b * kBN + c * 32, r[c]);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->acc_empty[b]);  // values are in registers now

      if (kPass == 1) {
        const int valid = Lk - t * kBN;  // >= kBN except on the last tile
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j < valid) tmax = fmaxf(tmax, __uint_as_float(r[c][j]));
        const float mnew = fmaxf(m, tmax * c2);
        if (mnew > m) {
          if (m != -INFINITY) l *= tc::ex2(m - mnew);
          m = mnew;
        }
        const float nm = -m;
        float l0 = 0.0f, l1 = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            if (c * 32 + j < valid) l0 += tc::ex2(fmaf(__uint_as_float(r[c][j]), c2, nm));
            if (c * 32 + j + 1 < valid) l1 += tc::ex2(fmaf(__uint_as_float(r[c][j + 1]), c2, nm));
          }
        l += l0 + l1;
      } else {
        const float4* L4 = reinterpret_cast<const float4*>(sL + s * kBN);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 L = L4[(c * 32 + j) >> 2];
            acc0 += tc::ex2(fmaf(__uint_as_float(r[c][j]), c2, -L.x));
            acc1 += tc::ex2(fmaf(__uint_as_float(r[c][j + 1]), c2, -L.y));
            acc0 += tc::ex2(fmaf(__uint_as_float(r[c][j + 2]), c2, -L.z));
            acc1 += tc::ex2(fmaf(__uint_as_float(r[c][j + 3]), c2, -L.w));
          }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->empty[s]);  // done with this stage's lse2
      }
    }
    if (ok) {
      if (kPass == 1) {
        if (row < lq_pad)
          lse2[(size_t)h * lq_pad + row] = row < Lq ? m + __log2f(l) : INFINITY;
      } else {
        if (row < Lk) imp[(size_t)h * Lk + row] = (acc0 + acc1) / (float)Lq;
      }
    }
  }
  if (!ok) atomicExch(err, 1);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 2) tc::tmem_dealloc(tmem, 2 * kBN);
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

// [H][L][d] bf16, box = 64 elements (128 B, the swizzle span) x 128 rows x 1 head.
bool make_map(CUtensorMap* map, const void* ptr, int H, int L, int d) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t run(const void* q, const void* k, int H, int Lq, int Lk, float scale, float* imp,
                void* ws, cudaStream_t s) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, q, H, Lq, D) || !make_map(&mk, k, H, Lk, D)) return cudaErrorInvalidValue;
  int* err = reinterpret_cast<int*>(static_cast<char*>(ws) + kErrOffset);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + kLseOffset);
  const int lq_pad = (int)ceil_div(Lq, kBM) * kBM;
  const float c2 = scale * kLog2e;
  const size_t smem = smem_bytes<D>();
  cudaError_t e;
  e = cudaFuncSetAttribute(imp_tc_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(imp_tc_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  imp_tc_kernel<D, 1><<<dim3(lq_pad / kBM, H), kThreads, smem, s>>>(mq, mk, Lq, Lk, lq_pad, c2,
                                                                     lse2, imp, err);
  imp_tc_kernel<D, 2><<<dim3((unsigned)ceil_div(Lk, kBM), H), kThreads, smem, s>>>(
      mk, mq, Lq, Lk, lq_pad, c2, lse2, imp, err);
  return cudaGetLastError();
}
}  // namespace

size_t importance_ws_bytes(int H, int Lq) {
  return kLseOffset + align_up((size_t)H * ceil_div(Lq, kBM) * kBM * sizeof(float), 256);
}

bool importance_tc_supported(int d) { return d == 64 || d == 128; }

cudaError_t launch_importance_tc(const void* q, const void* k, int H, int Lq, int Lk, int d,
                                 float scale, float* imp, void* ws, cudaStream_t s) {
  return d == 128 ? run<128>(q, k, H, Lq, Lk, scale, imp, ws, s)
                  : run<64>(q, k, H, Lq, Lk, scale, imp, ws, s);
}

}  // namespace fc

// Importance on the 5th-generation tensor cores (bf16 inputs, fp32 accumulate).
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 3: Imp_j = (1/L_q) sum_q softmax_j(q.k_j / sqrt(d)) over
// the clean candidate keys.
//
// The L_q x L_k probability matrix is never stored.  Two passes recompute the
// logits with tcgen05.mma:
//   pass 1 (rows)     CTA = 128 queries of one head; streams every 128-key
//                     tile; D = Q K^T in TMEM; the epilogue thread that owns a
//                     query row keeps a (reference, sum) pair in log2 units
//                     and the CTA writes nl_q = -log2 sum_j 2^(c s_qj),
//                     c = scale*log2(e) (padded query rows: -inf).
//   pass 2 (columns)  CTA = 128 keys of one head; streams every 128-query tile;
//                     D = K Q^T in TMEM (keys on the TMEM lanes), so each
//                     epilogue thread owns one key and sums 2^(c s + nl_q)
//                     over all queries in registers: no atomics, no partial
//                     buffers, deterministic.
//
// Work per score is one tensor-core MAC row (256 flops at d=128) and one
// exponential.  The SM's special-function unit retires 16 exponentials per
// clock against ~32 scores per clock of dense bf16 MMA, so the epilogue, not
// the MMA, sets the pace.  The design therefore
//   - runs two epilogue warpgroups in ping-pong over four 128-column TMEM
//     accumulators (the tensor core fills tile t+2 while tiles t and t+1 are
//     being drained);
//   - uses packed f32x2 FMA/ADD for the scale-and-shift and the running sums;
//   - evaluates 3 of every 8 exponentials on the FMA pipes (ex2_poly2, a
//     polynomial of our own) and the rest on the special-function unit;
//   - in pass 1 shifts by a lagged reference instead of the exact running max:
//     the reference only moves (with an exact rescale) when a half tile's sum
//     exceeds 2^32, so the per-element max disappears from the common path.
//
// Roles (384 threads): warp 0 lane 0 issues TMA loads (3D tensor maps over
// [H][L][d], 128-byte swizzle, zero fill past L, no multicast), warp 1 lane 0
// issues the MMAs (M=128, N=128, K=16 steps), warp 2 owns the TMEM allocation
// (all 512 columns), warps 4-7 and 8-11 are the two epilogue warpgroups (warp
// w reads TMEM lanes 32(w%4)..+31).  A shared-memory ring of operand tiles
// decouples TMA from the MMAs.  Every mbarrier wait is bounded; on timeout the
// kernel records an error word in the workspace and winds down (no trap, no
// endless spin).
#include <cuda.h>

#include "fc_common.cuh"
#include "fc_kernels.h"
#include "tc_ptx.cuh"

namespace fc {

namespace {
constexpr int kBM = 128;      // rows of the resident A tile (TMEM lanes)
constexpr int kBN = 128;      // rows of each streamed B tile (MMA N, TMEM columns)
constexpr int kStages = 4;    // shared-memory ring depth
constexpr int kAcc = 4;       // TMEM accumulators of kBN columns
constexpr int kThreads = 384;
constexpr int kHalf = kBM * 64 * 2;  // one 128 x 64 bf16 swizzled block (16 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kErrOffset = 0;      // error word in the workspace
constexpr size_t kLseOffset = 256;    // nl [H][Lq_pad] follows
constexpr float kRescaleAt = 4294967296.0f;  // 2^32

// Which pairs of a 64-column half go to the FMA pipes: 3 of every 8 values.
__device__ __forceinline__ constexpr bool emulated_pair(int p) {
  return (p & 3) == 1 || (p & 7) == 6;
}

template <int D>
constexpr int tile_bytes() {
  return (D / 64) * kHalf;
}
template <int D>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)(1 + kStages) * tile_bytes<D>() + 256 + kStages * kBN * sizeof(float) +
         2 * kBM * sizeof(float);
}

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t a_full;
  uint64_t acc_full[kAcc];
  uint64_t acc_empty[kAcc];
  uint32_t tmem_slot;
};

__device__ __forceinline__ void epilogue_sync() {
  asm volatile("bar.sync 1, 256;" ::: "memory");  // the 8 epilogue warps only
}

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}

// Sum of 2^(c*s - ref) over 64 values; mixes MUFU and FMA-pipe exponentials.
template <bool kClampHigh>
__device__ __forceinline__ float half_sum_shifted(const uint32_t (&r)[64], float c, float ref) {
  const float2 cc = make_float2(c, c), sh = make_float2(-ref, -ref);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float2 x = tc::ffma2(f2(r[2 * p], r[2 * p + 1]), cc, sh);
    float2 e;
    if (emulated_pair(p)) {
      e = tc::ex2_poly2<kClampHigh>(x);
    } else {
      e.x = tc::ex2(x.x);
      e.y = tc::ex2(x.y);
    }
    if (p & 1)
      acc1 = tc::fadd2(acc1, e);
    else
      acc0 = tc::fadd2(acc0, e);
  }
  const float2 a = tc::fadd2(acc0, acc1);
  return a.x + a.y;
}

__device__ __forceinline__ float half_max(const uint32_t (&r)[64]) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 64; j += 4) {
    m0 = tc::fmax3(m0, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
    m1 = tc::fmax3(m1, __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
  }
  return fmaxf(m0, m1);
}

// kPass 1: A = Q tile, B = K tiles, epilogue = row log-sum-exp.
// kPass 2: A = K tile, B = Q tiles, epilogue = column sums of 2^(c s + nl).
template <int D, int kPass>
__global__ void __launch_bounds__(kThreads, 1)
    imp_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                  int Lq, int Lk, int lq_pad, float c2, float* __restrict__ nl,
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
  float* sM = sL + kStages * kBN;  // [2][kBM] merge buffer of the two warpgroups

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int a0 = blockIdx.x * kBM;  // first row of the A tile
  const int nB = kPass == 1 ? (Lk + kBN - 1) / kBN : lq_pad / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      // pass 2: a stage also carries the query tile's nl values, so it is
      // released by the MMA commit and by the 4 warps of the consuming group
      tc::mbar_init(&bars->empty[s], kPass == 2 ? 5 : 1);
    }
    tc::mbar_init(&bars->a_full, 1);
    for (int b = 0; b < kAcc; ++b) {
      tc::mbar_init(&bars->acc_full[b], 1);
      tc::mbar_init(&bars->acc_empty[b], 4);
    }
    tc::fence_barrier_init();
  }
  if (warp == 2) tc::tmem_alloc(&bars->tmem_slot, kAcc * kBN);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      tc::mbar_expect_tx(&bars->a_full, TB);
      for (int kb = 0; kb < KB; ++kb)
        tc::tma_load_3d(sA + kb * kHalf, &mapA, &bars->a_full, kb * 64, a0, h);
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
          tc::bulk_load(sL + s * kBN, nl + (size_t)h * lq_pad + t * kBN, kBN * 4, &bars->full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      ok = tc::mbar_wait(&bars->a_full, 0);
      const uint32_t a_addr = tc::smem_u32(sA);
      for (int t = 0; ok && t < nB; ++t) {
        const int s = t % kStages, u = t / kStages, b = t % kAcc, v = t / kAcc;
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
  } else if (warp >= 4) {  // ---- two epilogue warpgroups, tiles alternate between them
    const int g = (warp - 4) >> 2;   // warpgroup 0 takes even tiles, 1 odd tiles
    const int sub = warp & 3;        // TMEM lane quarter
    const int rloc = sub * 32 + lane;  // this thread's row of the A tile
    const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
    float ref = -INFINITY, l = 0.0f;  // pass 1: running reference and sum (log2 units)
    float2 acc = make_float2(0.f, 0.f);  // pass 2: column sum (two chains)
    for (int t = g; t < nB; t += 2) {
      const int b = t % kAcc, v = t / kAcc, s = t % kStages, u = t / kStages;
      if (!tc::mbar_wait(&bars->acc_full[b], v & 1) ||
          (kPass == 2 && !tc::mbar_wait(&bars->full[s], u & 1))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t r[64];
        tc::tmem_ld32(lane_addr + b * kBN + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(r));
        tc::tmem_ld32(lane_addr + b * kBN + hf * 64 + 32,
                      *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tc::tmem_ld_wait();
        if (hf == 1) {
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->acc_empty[b]);  // values are in registers
        }
        if (kPass == 1) {
          const int valid = Lk - t * kBN - hf * 64;  // >= 64 except near the end
          if (valid < 64) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j >= valid) r[j] = 0xff800000u;  // -inf: a key past L_k
          }
          if (ref == -INFINITY) ref = half_max(r) * c2;  // first values this group sees
          if (ref != -INFINITY) {
            float hs = half_sum_shifted<true>(r, c2, ref);
            if (!(hs <= kRescaleAt)) {  // much larger logits arrived: move the reference
              const float rnew = fmaxf(ref, half_max(r) * c2);
              l *= tc::ex2(ref - rnew);
              ref = rnew;
              hs = half_sum_shifted<true>(r, c2, ref);
            }
            l += hs;
          }
        } else {
          const float2* L2 = reinterpret_cast<const float2*>(sL + s * kBN + hf * 64);
          const float2 cc = make_float2(c2, c2);
          float2 acc1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int p = 0; p < 32; ++p) {
            const float2 x = tc::ffma2(f2(r[2 * p], r[2 * p + 1]), cc, L2[p]);
            float2 e;
            if (emulated_pair(p)) {
              e = tc::ex2_poly2<false>(x);
            } else {
              e.x = tc::ex2(x.x);
              e.y = tc::ex2(x.y);
            }
            if (p & 1)
              acc1 = tc::fadd2(acc1, e);
            else
              acc = tc::fadd2(acc, e);
          }
          acc = tc::fadd2(acc, acc1);
        }
      }
      if (kPass == 2) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->empty[s]);  // done with this stage's nl values
      }
    }
    // Merge the two warpgroups' partial results for each row (both groups
    // always reach this barrier, also after a timeout).
    if (kPass == 1) {
      if (g == 1) {
        sM[rloc] = ref;      // group 1's reference
        sM[kBM + rloc] = l;  // group 1's sum
      }
      epilogue_sync();
      if (g == 0 && ok) {
        const float r1 = sM[rloc], l1 = sM[kBM + rloc];
        const float M = fmaxf(ref, r1);
        float L = 0.0f;
        if (ref != -INFINITY) L += l * tc::ex2(ref - M);
        if (r1 != -INFINITY) L += l1 * tc::ex2(r1 - M);
        const int row = a0 + rloc;
        nl[(size_t)h * lq_pad + row] = row < Lq ? -(M + __log2f(L)) : -INFINITY;
      }
    } else {
      if (g == 1) sM[rloc] = acc.x + acc.y;
      epilogue_sync();
      if (g == 0 && ok) {
        const int row = a0 + rloc;
        if (row < Lk) imp[(size_t)h * Lk + row] = ((acc.x + acc.y) + sM[rloc]) / (float)Lq;
      }
    }
  }
  if (!ok) atomicExch(err, 1);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 2) tc::tmem_dealloc(tmem, kAcc * kBN);
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
  float* nl = reinterpret_cast<float*>(static_cast<char*>(ws) + kLseOffset);
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
                                                                     nl, imp, err);
  imp_tc_kernel<D, 2><<<dim3((unsigned)ceil_div(Lk, kBM), H), kThreads, smem, s>>>(
      mk, mq, Lq, Lk, lq_pad, c2, nl, imp, err);
  return cudaGetLastError();
}

// Self-test of the two exponentials (MUFU and FMA-pipe) on given inputs.
__global__ void exp2_selftest_kernel(const float* x, float* y_mufu, float* y_poly, int n) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 v = make_float2(x[i], x[i + 1]);
    y_mufu[i] = tc::ex2(v.x);
    y_mufu[i + 1] = tc::ex2(v.y);
    const float2 p = tc::ex2_poly2<false>(v);
    y_poly[i] = p.x;
    y_poly[i + 1] = p.y;
  }
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

cudaError_t launch_exp2_selftest(const float* x, float* y_mufu, float* y_poly, int n,
                                 cudaStream_t s) {
  const int pairs = n / 2;
  if (pairs > 0)
    exp2_selftest_kernel<<<(unsigned)ceil_div(pairs, 256), 256, 0, s>>>(x, y_mufu, y_poly, n);
  return cudaGetLastError();
}

}  // namespace fc

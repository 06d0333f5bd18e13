// Thin inline-PTX wrappers for the sm_100a features the tensor-core kernels
// use: mbarriers (with bounded waits), TMA tensor loads, TMEM allocation,
// tcgen05.mma / commit / ld, and the shared-memory matrix descriptor.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace fc {
namespace tc {

// A bounded wait gives up after this many SM clocks (~2 s at 1.9 GHz).
constexpr long long kWaitCycles = 4000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Wait for the phase of parity `parity` to complete; false if it did not
// within `limit` SM clocks (the caller records the error and winds down).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}

// ---- TMA --------------------------------------------------------------------
// 3D tiled load (no multicast) completing on `bar` with the byte count.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// ---- TMEM -------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- tcgen05.mma --------------------------------------------------------------
// Shared-memory matrix descriptor of a K-major operand stored with the 128-byte
// swizzle: rows of 128 bytes, groups of 8 rows 1024 bytes apart (SBO), the
// leading offset unused (encoded 16 bytes), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// The same for the 32-byte swizzle: rows of 32 bytes (16 bf16, one K step),
// groups of 8 rows 256 bytes apart, layout type 6.
__device__ __forceinline__ uint64_t desc_k_sw32(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(256 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)6 << 61;
  return d;
}
// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 TMEM lanes x 32 consecutive 32-bit columns: thread t of the warp gets
// lane (lane field of taddr) + t.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
      " [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// The same wait, with the registers of the last tcgen05.ld passed through it
// so the compiler cannot schedule any use of them before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
        "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
        "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
        "+r"(r[31])
      :
      : "memory");
}

// ---- arithmetic -----------------------------------------------------------------
// 2^x on the special-function unit (MUFU.EX2, ~2 ulp; flushes subnormals).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed float32 pairs (sm_100 f32x2 arithmetic: two lanes per instruction).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)),
        "l"(reinterpret_cast<const uint64_t&>(c)));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair, on the FMA pipes instead of the special-function unit, so
// that part of a tile's exponentials can run beside the MUFU ones.  Method:
// Cody-Waite style range reduction x = n + f with n = round(x) (the
// 1.5*2^23 rounding constant) and f in [-1/2, 1/2], a polynomial for 2^f whose
// coefficients we fitted (iteratively reweighted least squares for relative
// error on Chebyshev nodes; cache_gating_kv_b200/csrc/gen_exp2_poly.py), then
// n is added to the exponent field.  kDeg = 5: max relative error 2.4e-7;
// kDeg = 4: 2.7e-6; kDeg = 3: 7.6e-5 (for x >= -125).  Inputs below -125
// (including -inf) are clamped there, giving about 2^-125 instead of 0.  With
// kClampHigh, inputs above 64 are clamped to 64 (callers that must see
// overflow as a large value); without it the caller guarantees x <= 126.
template <bool kClampHigh, int kDeg>
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  static_assert(kDeg >= 3 && kDeg <= 5, "fitted degrees: 3, 4, 5");
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  if (kClampHigh) {
    x.x = fminf(x.x, 64.0f);
    x.y = fminf(x.y, 64.0f);
  }
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 j = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = fadd2(x, make_float2(-j.x, -j.y));
  float2 p;
  if constexpr (kDeg == 5) {
    p = make_float2(1.3278164e-03f, 1.3278164e-03f);
    p = ffma2(p, f, make_float2(9.6755559e-03f, 9.6755559e-03f));
    p = ffma2(p, f, make_float2(5.5507079e-02f, 5.5507079e-02f));
    p = ffma2(p, f, make_float2(2.4022119e-01f, 2.4022119e-01f));
    p = ffma2(p, f, make_float2(6.9314694e-01f, 6.9314694e-01f));
    p = ffma2(p, f, make_float2(1.0000001e+00f, 1.0000001e+00f));
  } else if constexpr (kDeg == 4) {
    p = make_float2(9.5718065e-03f, 9.5718065e-03f);
    p = ffma2(p, f, make_float2(5.5918004e-02f, 5.5918004e-02f));
    p = ffma2(p, f, make_float2(2.4024703e-01f, 2.4024703e-01f));
    p = ffma2(p, f, make_float2(6.9312179e-01f, 6.9312179e-01f));
    p = ffma2(p, f, make_float2(9.9999928e-01f, 9.9999928e-01f));
  } else {
    p = make_float2(5.5186376e-02f, 5.5186376e-02f);
    p = ffma2(p, f, make_float2(2.4261236e-01f, 2.4261236e-01f));
    p = ffma2(p, f, make_float2(6.9325829e-01f, 6.9325829e-01f));
    p = ffma2(p, f, make_float2(9.9992794e-01f, 9.9992794e-01f));
  }
  // the low bits of t hold n (two's complement); n << 23 lands in the exponent
  const uint32_t ex = (__float_as_uint(t.x) << 23) + __float_as_uint(p.x);
  const uint32_t ey = (__float_as_uint(t.y) << 23) + __float_as_uint(p.y);
  return make_float2(__uint_as_float(ex), __uint_as_float(ey));
}

}  // namespace tc
}  // namespace fc

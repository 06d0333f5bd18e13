// Chunkwise cache gate: fused Euler update, per-chunk relative-L1 reduction
// and the accumulator recurrence, in one memory-bound pass.
//
// Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
// 方法详解 / 关键设计 1 (L1_rel = ||v*dt||_1 / ||X_t||_1, the update form of the
// relative L1 distance between X_{t-1} and X_t) and 关键设计 2 (per-chunk
// accumulator f: forced recompute for the first m steps, recompute and reset
// when f + L1_rel > eps, otherwise accumulate and reuse).
//
// Design (B200): the pass moves 12 bytes per element (read X, read v, write
// X), so it is bound by HBM.  The grid is n_chunks x blocks_per_chunk with the
// total sized to fill all SMs (four resident blocks per SM); every thread
// streams 16-byte vectors with read-once cache hints, unrolled so that each
// thread keeps eight loads in flight, and the first of them go out before the
// chunk's step counter and dt are read.  (Staging the stream through shared
// memory with 1-D TMA bulk copies, one CTA per SM, measured 14% slower at 4
// chunks and 6% slower at 16 on B200.)  The four magnitudes of a vector are
// added in float32, the rest in float64, so the float32 L1_rel is within
// 2^-23 relative of the exact quotient.  Each block stores its partial
// pair; the last block of a chunk to finish (an integer completion counter,
// no spinning, no float atomics) sums the partials in a fixed order and runs
// the recurrence, so the result is deterministic and one launch does it all.
#include <cuda.h>

#include <mutex>

#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

namespace {
constexpr int kGateThreads = 256;
// 16-byte vectors of x (and of v) in flight per thread, and the resident
// blocks per SM the grid is sized for.  Measured on B200 against 8 vectors
// with 2 blocks per SM and 6 with 2: equal at 4 chunks of 777,600, 12 % faster
// at 8 chunks of 499,200 for 8 with 2, 7-14 % slower at 16 chunks.
constexpr int kGateUnroll = 4;
constexpr int kGateBlocksPerSm = 4;
constexpr int kGateMaxBlocksPerChunk = 1024;

template <bool kHist>
__device__ __forceinline__ void gate_finalize(int c, int st, int m, float eps, double num,
                                              double den, float* f, float* l1, uint8_t* mask) {
  float r;
  if (den > 0.0)
    r = (float)(num / den);
  else
    r = (num > 0.0) ? __int_as_float(0x7f800000) : 0.0f;
  l1[c] = r;
  const float reset = kHist ? r : 0.0f;
  if (st < m) {  // forced recompute during the first m steps of the chunk
    mask[c] = 1;
    f[c] = reset;
  } else {
    const float acc = __fadd_rn(f[c], r);
    if (acc > eps) {  // recompute and reset
      mask[c] = 1;
      f[c] = reset;
    } else {  // reuse, accumulate
      mask[c] = 0;
      f[c] = acc;
    }
  }
}

// FlowCache: p = v*dt (rounded once), X <- X + p (rounded once).
// History gate: p = h_t - h_{t+1} (rounded once), h_{t+1} <- h_t.
// |p| and |X before the step| of the four lanes of a vector are summed
// pairwise in float32 (two roundings: relative error below 2^-23, as all
// terms are non-negative), then widened and added to the float64 sums; the
// per-element float64 conversions measured on the conversion unit otherwise.
template <bool kHist>
__device__ __forceinline__ void gate_vec(float4& x, const float4& v, float h, double& num,
                                         double& den) {
  const float p0 = kHist ? __fsub_rn(v.x, x.x) : __fmul_rn(v.x, h);
  const float p1 = kHist ? __fsub_rn(v.y, x.y) : __fmul_rn(v.y, h);
  const float p2 = kHist ? __fsub_rn(v.z, x.z) : __fmul_rn(v.z, h);
  const float p3 = kHist ? __fsub_rn(v.w, x.w) : __fmul_rn(v.w, h);
  num += (double)__fadd_rn(__fadd_rn(fabsf(p0), fabsf(p1)), __fadd_rn(fabsf(p2), fabsf(p3)));
  den += (double)__fadd_rn(__fadd_rn(fabsf(x.x), fabsf(x.y)), __fadd_rn(fabsf(x.z), fabsf(x.w)));
  x.x = kHist ? v.x : __fadd_rn(x.x, p0);
  x.y = kHist ? v.y : __fadd_rn(x.y, p1);
  x.z = kHist ? v.z : __fadd_rn(x.z, p2);
  x.w = kHist ? v.w : __fadd_rn(x.w, p3);
}

// One element (the unaligned head and tail of a chunk), summed in float64.
template <bool kHist>
__device__ __forceinline__ void gate_elem(float& x, float vv, float h, double& num, double& den) {
  const float p = kHist ? __fsub_rn(vv, x) : __fmul_rn(vv, h);
  num += (double)fabsf(p);
  den += (double)fabsf(x);
  x = kHist ? vv : __fadd_rn(x, p);
}

template <bool kHist>
__global__ void __launch_bounds__(kGateThreads, kGateBlocksPerSm)
    gate_kernel(float* __restrict__ x, const float* __restrict__ v, int64_t N,
                const float* __restrict__ dt, const int32_t* __restrict__ step, int m, float eps,
                float* __restrict__ f, float* __restrict__ l1, uint8_t* __restrict__ mask,
                unsigned* __restrict__ counters, double2* __restrict__ partials, int bpc) {
  const int c = blockIdx.y;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t off = (int64_t)c * N;
  float* xc = x + off;
  const float* vc = v + off;

  // x and v are 16-byte aligned, so the chunk's misalignment is off mod 4.
  const int64_t mis = off & 3;
  int64_t head = mis ? 4 - mis : 0;
  if (head > N) head = N;
  const int64_t nvec = (N - head) >> 2;
  const int64_t tail0 = head + (nvec << 2);

  const int64_t per = ceil_div(nvec, bpc);
  const int64_t lo = min(nvec, per * b);
  const int64_t hi = min(nvec, lo + per);
  float4* x4 = reinterpret_cast<float4*>(xc + head);
  const float4* v4 = reinterpret_cast<const float4*>(vc + head);
  constexpr int64_t kStride = (int64_t)kGateThreads * kGateUnroll;

  // The first loads go out before the chunk's step and dt are read, so the
  // stream does not wait behind those two dependent loads; nothing is written
  // before the step is known.
  float4 xa[kGateUnroll], va[kGateUnroll];
  int64_t base = lo + tid;
#pragma unroll
  for (int u = 0; u < kGateUnroll; ++u) {
    const int64_t i = base + (int64_t)u * kGateThreads;
    if (i < hi) {
      xa[u] = __ldcs(x4 + i);
      va[u] = __ldcs(v4 + i);
    }
  }
  const int st = step[c];
  const float h = kHist ? 0.0f : dt[c];
  if (st < 0) {  // inactive chunk: nothing touched
    if (b == 0 && tid == 0) {
      l1[c] = 0.0f;
      mask[c] = 0;
    }
    return;
  }

  double num = 0.0, den = 0.0;
  for (; base < hi; base += kStride) {
#pragma unroll
    for (int u = 0; u < kGateUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kGateThreads;
      if (i < hi) {
        gate_vec<kHist>(xa[u], va[u], h, num, den);
        __stcs(x4 + i, xa[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kGateUnroll; ++u) {
      const int64_t i = base + kStride + (int64_t)u * kGateThreads;
      if (i < hi) {
        xa[u] = __ldcs(x4 + i);
        va[u] = __ldcs(v4 + i);
      }
    }
  }
  // Unaligned head (< 4 elements) and tail (< 4 elements): block 0.
  if (b == 0) {
    int64_t e = -1;
    if (tid < head)
      e = tid;
    else if (tid >= 4 && tid - 4 < N - tail0)
      e = tail0 + (tid - 4);
    if (e >= 0) {
      float xv = xc[e];
      gate_elem<kHist>(xv, vc[e], h, num, den);
      xc[e] = xv;
    }
  }

  // Block reduction in a fixed order.
  __shared__ double s_num[kGateThreads / 32], s_den[kGateThreads / 32];
  __shared__ int s_last;
  num = warp_sum(num);
  den = warp_sum(den);
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
    s_num[warp] = num;
    s_den[warp] = den;
  }
  __syncthreads();
  if (tid == 0) {
    double a = 0.0, d = 0.0;
#pragma unroll
    for (int w = 0; w < kGateThreads / 32; ++w) {
      a += s_num[w];
      d += s_den[w];
    }
    partials[(size_t)c * kGateMaxBlocksPerChunk + b] = make_double2(a, d);
    __threadfence();  // publish the partial before counting this block done
    const unsigned prev = atomicAdd(&counters[c], 1u);
    s_last = (prev == (unsigned)(bpc - 1));
  }
  __syncthreads();
  if (!s_last) return;

  // Last block of chunk c: fixed-order sum of every block's partial.
  __threadfence();
  if (warp == 0) {
    // Every lane sums partials lane, lane + 32, ... in that order; the loads
    // of eight of them are issued before the first is added.
    constexpr int kBatch = 8;
    const double2* pc = partials + (size_t)c * kGateMaxBlocksPerChunk;
    double a = 0.0, d = 0.0;
    for (int i0 = 0; i0 < bpc; i0 += 32 * kBatch) {
      double2 p[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * 32 + lane;
        p[u] = i < bpc ? __ldcg(pc + i) : make_double2(0.0, 0.0);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        a += p[u].x;
        d += p[u].y;
      }
    }
    a = warp_sum(a);
    d = warp_sum(d);
    if (lane == 0) {
      gate_finalize<kHist>(c, st, m, eps, a, d, f, l1, mask);
      counters[c] = 0u;  // ready for the next call
    }
  }
}
}  // namespace

// Workspace: completion counters [n_chunks], an error word (the gate has no
// device-side waits, so it stays zero), then the per-block partial sums
// [n_chunks][kGateMaxBlocksPerChunk].
static size_t counters_bytes(int n_chunks) {
  return align_up((size_t)(n_chunks + 1) * sizeof(unsigned), 256);
}

size_t gate_ws_bytes(int n_chunks) {
  return counters_bytes(n_chunks) + (size_t)n_chunks * kGateMaxBlocksPerChunk * sizeof(double2);
}

cudaError_t launch_gate(float* x, const float* v, int n_chunks, int64_t N, const float* dt,
                        const int32_t* step, int m, float eps, float* f, float* l1,
                        uint8_t* mask, void* ws, cudaStream_t s, bool history) {
  unsigned* counters = static_cast<unsigned*>(ws);
  double2* partials =
      reinterpret_cast<double2*>(static_cast<char*>(ws) + counters_bytes(n_chunks));
  // kGateBlocksPerSm resident 256-thread blocks per SM over the whole grid.
  const int64_t target = (int64_t)sm_count() * kGateBlocksPerSm;
  int64_t bpc = ceil_div(target, n_chunks);
  const int64_t useful = ceil_div(N / 4 + 1, kGateThreads);  // >= one vector per thread
  if (bpc > useful) bpc = useful;
  if (bpc < 1) bpc = 1;
  if (bpc > kGateMaxBlocksPerChunk) bpc = kGateMaxBlocksPerChunk;
  dim3 grid((unsigned)bpc, (unsigned)n_chunks);
  auto kern = history ? gate_kernel<true> : gate_kernel<false>;
  kern<<<grid, kGateThreads, 0, s>>>(x, v, N, dt, step, m, eps, f, l1, mask, counters, partials,
                                     (int)bpc);
  add_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the gate.
//
// Some callers cannot allocate device memory when they run the gate: a host
// runtime that gives its plugins only their input and output buffers and
// forbids cudaMalloc while work is being enqueued (an allocation may
// synchronize the device, or fail under a fixed memory budget), or code that
// has nowhere to keep a workspace alive between denoising steps.  For them
// the gate's scratch (completion counters and per-block partial sums) lives in
// one file-scope device array of a fixed size: every GPU that loads this
// library holds it until the process exits.  It serves at most
// kGateNoAllocMaxChunks chunks per call.  Every call shares the array, so
// calls that overlap on the GPU (other streams, other host threads) race;
// they must be ordered.
// ---------------------------------------------------------------------------
namespace {
constexpr int kGateNoAllocMaxChunks = 32;
constexpr size_t kGateNoAllocBytes =
    256 + (size_t)kGateNoAllocMaxChunks * kGateMaxBlocksPerChunk * sizeof(double2);  // 512.25 KiB

static __device__ __align__(256) unsigned char g_gate_scratch[kGateNoAllocBytes];

// Device address of g_gate_scratch per device ordinal, together with the id
// of the context it was looked up in.  In host code the array's name is only
// a host-side stand-in, so the address must come from cudaGetSymbolAddress,
// made with that device current.  The first call on a device (and the first
// after its primary context was destroyed, e.g. by cudaDeviceReset, which
// gives the array a new address) looks it up; later calls reuse it.  A mutex
// orders host threads that make their first call at the same time.
struct ScratchAddr {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kMaxDevices = 128;
ScratchAddr g_gate_scratch_addr[kMaxDevices] = {};
std::mutex g_gate_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id (for the life of the process) of the current context, or 0.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}
}  // namespace

int gate_noalloc_max_chunks() { return kGateNoAllocMaxChunks; }

cudaError_t gate_noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // Before the runtime has made a context current the id is 0, and the
  // address is looked up (which creates the primary context) on every call
  // until it has.
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_gate_scratch_mu);
  ScratchAddr& s = g_gate_scratch_addr[dev];
  if (s.addr == nullptr || ctx == 0 || s.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gate_scratch);
    if (e != cudaSuccess) return e;
    s.addr = p;
    s.ctx_id = ctx;
  }
  *out = s.addr;
  return cudaSuccess;
}

cudaError_t launch_gate_noalloc(float* x, const float* v, int n_chunks, int64_t N,
                                const float* dt, const int32_t* step, int m, float eps, float* f,
                                float* l1, uint8_t* mask, cudaStream_t s) {
  if (n_chunks < 1 || n_chunks > kGateNoAllocMaxChunks) return cudaErrorInvalidValue;
  void* ws = nullptr;
  cudaError_t e = gate_noalloc_scratch(&ws);
  if (e != cudaSuccess) return e;
  // The completion counters and the error word must start at zero; the array
  // keeps whatever the previous call left, so clear them on the caller's
  // stream first.
  e = cudaMemsetAsync(ws, 0, (size_t)(n_chunks + 1) * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  add_launches(1);
  return launch_gate(x, v, n_chunks, N, dt, step, m, eps, f, l1, mask, ws, s, false);
}

}  // namespace fc

// C-ABI of libflowcache: argument validation on the host, then launches.
// The declarations and their contracts are in include/flowcache.h.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "../../include/flowcache.h"
#include "../../include/flowcache_selftest.h"
#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

thread_local int g_launches = 0;
void add_launches(int n) { g_launches += n; }

}  // namespace fc

namespace {

thread_local char g_err[512] = "";

fc_status fail(fc_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

// An NVTX range around each compute call, named after it, so that a profiler
// timeline shows the library's calls (no cost without a profiler attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

fc_status ok() {
  g_err[0] = '\0';
  return FC_OK;
}

// Null, misalignment and host-memory checks for one tensor argument.
fc_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(FC_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
    return fail(FC_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  cudaPointerAttributes a;
  const cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FC_ERR_CUDA, "cudaPointerGetAttributes(%s): %s", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(FC_ERR_INVALID_ARG, "%s is not device memory", name);
  return FC_OK;
}

#define FC_CHECK_PTR(p)                        \
  do {                                         \
    fc_status _st = check_ptr((p), #p);        \
    if (_st != FC_OK) return _st;              \
  } while (0)

fc_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) fc::g_launches = 0;
  if (e != cudaSuccess) return fail(FC_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const char* pa = static_cast<const char*>(a);
  const char* pb = static_cast<const char*>(b);
  return pa < pb + nb && pb < pa + na;
}

size_t elem_bytes(fc_dtype t) { return t == FC_BF16 ? 2 : 4; }

// Two [n][N] float32 latent arrays, one written in place while the other is
// read, must be disjoint (the kernel reads v through a non-aliasing pointer).
bool latents_overlap(const float* x, const float* v, int n, int64_t N) {
  const size_t bytes = (size_t)n * (size_t)N * sizeof(float);
  return ranges_overlap(x, bytes, v, bytes);
}

fc_status check_kv_shape(fc_dtype dtype, int H, int L1, int L2, int d) {
  if (dtype != FC_F32 && dtype != FC_BF16) return fail(FC_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (H < 1 || L1 < 1 || L2 < 1) return fail(FC_ERR_INVALID_ARG, "sizes must be >= 1");
  if (H > 65535) return fail(FC_ERR_INVALID_ARG, "H must be <= 65535");
  if (d != 64 && d != 128) return fail(FC_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  return FC_OK;
}

// Workspace of fc_kv_cache_commit: the importance stage's own workspace first
// (so bytes 0..3 are its error word, as for fc_kv_importance), then Imp, Red
// and the selection, then the redundancy and score/top-B workspaces.
struct CacheWs {
  size_t imp, red, idx, red_ws, score_ws, total;
};

CacheWs cache_ws(int H, int Lq, int B_budget, int C, int d) {
  const size_t cap = (size_t)B_budget + C;
  CacheWs w;
  size_t o = fc::align_up(fc::importance_ws_bytes(H, Lq), 256);
  w.imp = o;
  o = fc::align_up(o + (size_t)H * cap * sizeof(float), 256);
  w.red = o;
  o = fc::align_up(o + (size_t)H * cap * sizeof(float), 256);
  w.idx = o;
  o = fc::align_up(o + (size_t)H * B_budget * sizeof(int32_t), 256);
  w.red_ws = o;
  o = fc::align_up(o + fc::redundancy_ws_bytes(H, (int)cap, d), 256);
  w.score_ws = o;
  w.total = fc::align_up(o + fc::score_topb_ws_bytes(H, (int)cap), 256);
  return w;
}

}  // namespace

extern "C" {

const char* fc_last_error(void) { return g_err; }

int fc_last_launches(void) { return fc::g_launches; }

int fc_version(void) { return 100; }

size_t fc_gate_workspace_size(int n_chunks, int64_t n_per_chunk) {
  (void)n_per_chunk;
  return n_chunks < 1 ? 0 : fc::gate_ws_bytes(n_chunks);
}

fc_status fc_chunk_l1_gate(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                           const float* dt, const int32_t* step, int32_t m, float eps, float* f,
                           float* l1_rel, uint8_t* recompute, void* ws, size_t ws_bytes,
                           void* stream) {
  NvtxRange _range("fc_chunk_l1_gate");
  fc::g_launches = 0;
  if (n_chunks < 1 || n_chunks > 65535)
    return fail(FC_ERR_INVALID_ARG, "n_chunks must be in [1, 65535] (got %d)", n_chunks);
  if (n_per_chunk < 0) return fail(FC_ERR_INVALID_ARG, "n_per_chunk must be >= 0");
  if (m < 0) return fail(FC_ERR_INVALID_ARG, "m must be >= 0");
  if (ws == nullptr || ws_bytes < fc::gate_ws_bytes(n_chunks))
    return fail(FC_ERR_WORKSPACE, "gate workspace needs %zu bytes", fc::gate_ws_bytes(n_chunks));
  if (n_per_chunk > 0) {  // empty chunks touch no latent memory
    FC_CHECK_PTR(x);
    FC_CHECK_PTR(v);
    if (latents_overlap(x, v, n_chunks, n_per_chunk))
      return fail(FC_ERR_INVALID_ARG, "x and v overlap (x is updated in place while v is read)");
  }
  FC_CHECK_PTR(dt);
  FC_CHECK_PTR(step);
  FC_CHECK_PTR(f);
  FC_CHECK_PTR(l1_rel);
  FC_CHECK_PTR(recompute);
  FC_CHECK_PTR(ws);
  return launched(fc::launch_gate(x, v, n_chunks, n_per_chunk, dt, step, m, eps, f, l1_rel,
                                  recompute, ws, static_cast<cudaStream_t>(stream), false),
                  "fc_chunk_l1_gate");
}

fc_status fc_history_l1_gate(float* h_old, const float* h_new, int n_segments,
                             int64_t n_per_segment, const int32_t* step, int32_t m, float delta,
                             float* f, float* d_rel, uint8_t* refresh, void* ws, size_t ws_bytes,
                             void* stream) {
  NvtxRange _range("fc_history_l1_gate");
  fc::g_launches = 0;
  if (n_segments < 1 || n_segments > 65535)
    return fail(FC_ERR_INVALID_ARG, "n_segments must be in [1, 65535] (got %d)", n_segments);
  if (n_per_segment < 0) return fail(FC_ERR_INVALID_ARG, "n_per_segment must be >= 0");
  if (m < 0) return fail(FC_ERR_INVALID_ARG, "m must be >= 0");
  if (ws == nullptr || ws_bytes < fc::gate_ws_bytes(n_segments))
    return fail(FC_ERR_WORKSPACE, "gate workspace needs %zu bytes", fc::gate_ws_bytes(n_segments));
  if (n_per_segment > 0) {
    FC_CHECK_PTR(h_old);
    FC_CHECK_PTR(h_new);
    if (latents_overlap(h_old, h_new, n_segments, n_per_segment))
      return fail(FC_ERR_INVALID_ARG,
                  "h_old and h_new overlap (h_old is overwritten while h_new is read)");
  }
  FC_CHECK_PTR(step);
  FC_CHECK_PTR(f);
  FC_CHECK_PTR(d_rel);
  FC_CHECK_PTR(refresh);
  FC_CHECK_PTR(ws);
  return launched(fc::launch_gate(h_old, h_new, n_segments, n_per_segment, nullptr, step, m, delta,
                                  f, d_rel, refresh, ws, static_cast<cudaStream_t>(stream), true),
                  "fc_history_l1_gate");
}

fc_status fc_chunk_l1_gate_noalloc(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                                   const float* dt, const int32_t* step, int32_t m, float eps,
                                   float* f, float* l1_rel, uint8_t* recompute, void* stream) {
  NvtxRange _range("fc_chunk_l1_gate_noalloc");
  fc::g_launches = 0;
  const int max_chunks = fc::gate_noalloc_max_chunks();
  if (n_chunks < 1 || n_chunks > max_chunks)
    return fail(FC_ERR_INVALID_ARG,
                "fc_chunk_l1_gate_noalloc serves 1 to %d chunks per call (got %d); use "
                "fc_chunk_l1_gate with a workspace for more",
                max_chunks, n_chunks);
  if (n_per_chunk < 0) return fail(FC_ERR_INVALID_ARG, "n_per_chunk must be >= 0");
  if (m < 0) return fail(FC_ERR_INVALID_ARG, "m must be >= 0");
  if (n_per_chunk > 0) {
    FC_CHECK_PTR(x);
    FC_CHECK_PTR(v);
    if (latents_overlap(x, v, n_chunks, n_per_chunk))
      return fail(FC_ERR_INVALID_ARG, "x and v overlap (x is updated in place while v is read)");
  }
  FC_CHECK_PTR(dt);
  FC_CHECK_PTR(step);
  FC_CHECK_PTR(f);
  FC_CHECK_PTR(l1_rel);
  FC_CHECK_PTR(recompute);
  return launched(fc::launch_gate_noalloc(x, v, n_chunks, n_per_chunk, dt, step, m, eps, f,
                                          l1_rel, recompute, static_cast<cudaStream_t>(stream)),
                  "fc_chunk_l1_gate_noalloc");
}

fc_status fc_gather_recompute(const float* x, const uint8_t* recompute, int n_chunks,
                              int64_t n_per_chunk, float* dense, int32_t* ids, int32_t* count,
                              void* stream) {
  NvtxRange _range("fc_gather_recompute");
  fc::g_launches = 0;
  if (n_chunks < 1 || n_chunks > 65535)
    return fail(FC_ERR_INVALID_ARG, "n_chunks must be in [1, 65535] (got %d)", n_chunks);
  if (n_per_chunk < 0) return fail(FC_ERR_INVALID_ARG, "n_per_chunk must be >= 0");
  if (n_per_chunk > 0) {
    FC_CHECK_PTR(x);
    FC_CHECK_PTR(dense);
  }
  FC_CHECK_PTR(recompute);
  FC_CHECK_PTR(ids);
  FC_CHECK_PTR(count);
  return launched(fc::launch_gather_recompute(x, recompute, n_chunks, n_per_chunk, dense, ids,
                                              count, static_cast<cudaStream_t>(stream)),
                  "fc_gather_recompute");
}

fc_status fc_scatter_velocity(const float* v_dense, const int32_t* ids, const int32_t* count,
                              int n_chunks, int64_t n_per_chunk, float* v_cache, void* stream) {
  NvtxRange _range("fc_scatter_velocity");
  fc::g_launches = 0;
  if (n_chunks < 1 || n_chunks > 65535)
    return fail(FC_ERR_INVALID_ARG, "n_chunks must be in [1, 65535] (got %d)", n_chunks);
  if (n_per_chunk < 0) return fail(FC_ERR_INVALID_ARG, "n_per_chunk must be >= 0");
  if (n_per_chunk > 0) {
    FC_CHECK_PTR(v_dense);
    FC_CHECK_PTR(v_cache);
  }
  FC_CHECK_PTR(ids);
  FC_CHECK_PTR(count);
  const size_t bytes = (size_t)n_chunks * n_per_chunk * sizeof(float);
  if (n_per_chunk > 0 && ranges_overlap(v_dense, bytes, v_cache, bytes))
    return fail(FC_ERR_INVALID_ARG, "v_dense and v_cache overlap");
  return launched(fc::launch_scatter_velocity(v_dense, ids, count, n_chunks, n_per_chunk, v_cache,
                                              static_cast<cudaStream_t>(stream)),
                  "fc_scatter_velocity");
}

fc_status fc_check_workspace(fc_ws_kind kind, const void* ws, int n_chunks, int clear,
                             void* stream) {
  fc::g_launches = 0;
  size_t off = 0;
  const char* base = static_cast<const char*>(ws);
  switch (kind) {
    case FC_WS_GATE:
      if (n_chunks < 1) return fail(FC_ERR_INVALID_ARG, "n_chunks must be >= 1");
      FC_CHECK_PTR(ws);
      off = (size_t)n_chunks * sizeof(unsigned);
      break;
    case FC_WS_GATE_NOALLOC: {
      if (n_chunks < 1 || n_chunks > fc::gate_noalloc_max_chunks())
        return fail(FC_ERR_INVALID_ARG, "n_chunks must be in [1, %d]",
                    fc::gate_noalloc_max_chunks());
      void* p = nullptr;
      const cudaError_t e = fc::gate_noalloc_scratch(&p);
      if (e != cudaSuccess) return fail(FC_ERR_CUDA, "scratch address: %s", cudaGetErrorString(e));
      base = static_cast<const char*>(p);
      off = (size_t)n_chunks * sizeof(unsigned);
      break;
    }
    case FC_WS_IMPORTANCE:
    case FC_WS_CACHE:
      FC_CHECK_PTR(ws);
      break;
    default:
      return fail(FC_ERR_INVALID_ARG, "unknown workspace kind %d", (int)kind);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, base + off, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear && word != 0) {
    e = cudaMemsetAsync(const_cast<char*>(base) + off, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return fail(FC_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (word != 0)
    return fail(FC_ERR_TIMEOUT, "a bounded device-side wait gave up: the outputs of the "
                                "calls since the word was last clear are not valid");
  return ok();
}

size_t fc_importance_workspace_size(fc_dtype dtype, int H, int Lq, int Lk, int d) {
  (void)dtype;
  (void)Lk;
  (void)d;
  return (H < 1 || Lq < 1) ? 0 : fc::importance_ws_bytes(H, Lq);
}

fc_status fc_kv_importance(const void* q, const void* k, fc_dtype dtype, int H, int Lq, int Lk,
                           int d, float scale, float* imp, void* ws, size_t ws_bytes,
                           void* stream) {
  NvtxRange _range("fc_kv_importance");
  fc::g_launches = 0;
  fc_status st = check_kv_shape(dtype, H, Lq, Lk, d);
  if (st != FC_OK) return st;
  if (ws == nullptr || ws_bytes < fc::importance_ws_bytes(H, Lq))
    return fail(FC_ERR_WORKSPACE, "importance workspace needs %zu bytes",
                fc::importance_ws_bytes(H, Lq));
  FC_CHECK_PTR(q);
  FC_CHECK_PTR(k);
  FC_CHECK_PTR(imp);
  FC_CHECK_PTR(ws);
  if (!(scale > 0.0f)) scale = 1.0f / sqrtf((float)d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == FC_BF16 && fc::importance_tc_supported(d))
    return launched(fc::launch_importance_tc(q, k, H, Lq, Lk, d, scale, imp, ws, s),
                    "fc_kv_importance");
  return launched(fc::launch_importance_simt(q, k, dtype == FC_BF16, H, Lq, Lk, d, scale, imp,
                                             ws, s),
                  "fc_kv_importance");
}

size_t fc_redundancy_workspace_size(fc_dtype dtype, int H, int Lk, int d) {
  (void)dtype;
  return (H < 1 || Lk < 1 || (d != 64 && d != 128)) ? 0 : fc::redundancy_ws_bytes(H, Lk, d);
}

fc_status fc_kv_redundancy(const void* k, fc_dtype dtype, int H, int Lk, int d, float* red,
                           void* ws, size_t ws_bytes, void* stream) {
  NvtxRange _range("fc_kv_redundancy");
  fc::g_launches = 0;
  fc_status st = check_kv_shape(dtype, H, Lk, Lk, d);
  if (st != FC_OK) return st;
  if (Lk > fc::redundancy_max_lk())
    return fail(FC_ERR_UNSUPPORTED, "Lk must be <= %d (got %d)", fc::redundancy_max_lk(), Lk);
  if (ws == nullptr || ws_bytes < fc::redundancy_ws_bytes(H, Lk, d))
    return fail(FC_ERR_WORKSPACE, "redundancy workspace needs %zu bytes",
                fc::redundancy_ws_bytes(H, Lk, d));
  FC_CHECK_PTR(k);
  FC_CHECK_PTR(red);
  FC_CHECK_PTR(ws);
  return launched(fc::launch_redundancy(k, dtype == FC_BF16, H, Lk, d, red, ws,
                                        static_cast<cudaStream_t>(stream)),
                  "fc_kv_redundancy");
}

size_t fc_score_topb_workspace_size(int H, int Lk, int B) {
  (void)B;
  return (H < 1 || Lk < 1) ? 0 : fc::score_topb_ws_bytes(H, Lk);
}

fc_status fc_kv_score_topb(const float* imp, const float* red, int H, int Lk, int pool_window,
                           float lambda, int B, float* score, int32_t* idx, void* ws,
                           size_t ws_bytes, void* stream) {
  NvtxRange _range("fc_kv_score_topb");
  fc::g_launches = 0;
  if (H < 1 || H > 65535 || Lk < 1) return fail(FC_ERR_INVALID_ARG, "H and Lk must be >= 1");
  if (B < 1) return fail(FC_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  if (pool_window < 1 || pool_window % 2 == 0 || pool_window > 511)
    return fail(FC_ERR_INVALID_ARG, "pool_window must be odd and in [1, 511] (got %d)",
                pool_window);
  if (ws == nullptr || ws_bytes < fc::score_topb_ws_bytes(H, Lk))
    return fail(FC_ERR_WORKSPACE, "score/top-B workspace needs %zu bytes",
                fc::score_topb_ws_bytes(H, Lk));
  FC_CHECK_PTR(imp);
  FC_CHECK_PTR(red);
  FC_CHECK_PTR(idx);
  FC_CHECK_PTR(ws);
  if (score != nullptr) FC_CHECK_PTR(score);
  return launched(fc::launch_score_topb(imp, red, H, Lk, pool_window, lambda, B, score, idx, ws,
                                        static_cast<cudaStream_t>(stream)),
                  "fc_kv_score_topb");
}

fc_status fc_kv_compact(const void* k, const void* v, fc_dtype dtype, int H, int Lk, int d,
                        const int32_t* idx, int B, void* k_out, void* v_out, void* stream) {
  NvtxRange _range("fc_kv_compact");
  fc::g_launches = 0;
  fc_status st = check_kv_shape(dtype, H, Lk, Lk, d);
  if (st != FC_OK) return st;
  if (B < 1) return fail(FC_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  FC_CHECK_PTR(k);
  FC_CHECK_PTR(v);
  FC_CHECK_PTR(idx);
  FC_CHECK_PTR(k_out);
  FC_CHECK_PTR(v_out);
  const size_t in_bytes = (size_t)H * Lk * d * elem_bytes(dtype);
  const size_t out_bytes = (size_t)H * B * d * elem_bytes(dtype);
  if (ranges_overlap(k_out, out_bytes, k, in_bytes) || ranges_overlap(k_out, out_bytes, v, in_bytes) ||
      ranges_overlap(v_out, out_bytes, k, in_bytes) || ranges_overlap(v_out, out_bytes, v, in_bytes) ||
      ranges_overlap(k_out, out_bytes, v_out, out_bytes))
    return fail(FC_ERR_INVALID_ARG, "k_out / v_out overlap an input or each other");
  return launched(fc::launch_compact(k, v, (int)elem_bytes(dtype), H, Lk, d, idx, B, B, k_out,
                                     v_out, static_cast<cudaStream_t>(stream)),
                  "fc_kv_compact");
}

size_t fc_kv_cache_workspace_size(fc_dtype dtype, int H, int Lq, int B_budget, int C, int d) {
  (void)dtype;
  if (H < 1 || Lq < 1 || B_budget < 1 || C < 1 || (d != 64 && d != 128)) return 0;
  return cache_ws(H, Lq, B_budget, C, d).total;
}

fc_status fc_kv_cache_commit(const void* q, const void* k_buf, const void* v_buf, void* k_next,
                             void* v_next, fc_dtype dtype, int H, int Lq, int d, int B_budget,
                             int C, int n_clean, float scale, int pool_window, float lambda,
                             int32_t* idx, void* ws, size_t ws_bytes, int* n_next,
                             int* compressed, void* stream) {
  NvtxRange _range("fc_kv_cache_commit");
  fc::g_launches = 0;
  if (n_next == nullptr || compressed == nullptr)
    return fail(FC_ERR_INVALID_ARG, "n_next and compressed must be host pointers");
  if (C < 1 || B_budget < C)
    return fail(FC_ERR_INVALID_ARG, "need 1 <= C <= B_budget (got C=%d, B_budget=%d)", C, B_budget);
  if ((int64_t)B_budget + C > INT32_MAX / 2) return fail(FC_ERR_INVALID_ARG, "B_budget + C too large");
  if ((int64_t)B_budget + C > fc::redundancy_max_lk())
    return fail(FC_ERR_UNSUPPORTED, "B_budget + C must be <= %d", fc::redundancy_max_lk());
  const int cap = B_budget + C;
  fc_status st = check_kv_shape(dtype, H, Lq, cap, d);
  if (st != FC_OK) return st;
  if (n_clean < 0 || n_clean > B_budget)
    return fail(FC_ERR_INVALID_ARG, "n_clean must be in [0, B_budget] (got %d)", n_clean);
  if (pool_window < 1 || pool_window % 2 == 0 || pool_window > 511)
    return fail(FC_ERR_INVALID_ARG, "pool_window must be odd and in [1, 511] (got %d)",
                pool_window);
  if (n_clean + C <= B_budget) {  // the chunk fits: it stays where it is
    *n_next = n_clean + C;
    *compressed = 0;
    return ok();
  }
  const CacheWs lay = cache_ws(H, Lq, B_budget, C, d);
  if (ws == nullptr || ws_bytes < lay.total)
    return fail(FC_ERR_WORKSPACE, "cache workspace needs %zu bytes", lay.total);
  FC_CHECK_PTR(q);
  FC_CHECK_PTR(k_buf);
  FC_CHECK_PTR(v_buf);
  FC_CHECK_PTR(k_next);
  FC_CHECK_PTR(v_next);
  FC_CHECK_PTR(ws);
  if (idx != nullptr) FC_CHECK_PTR(idx);
  const size_t buf_bytes = (size_t)H * cap * d * elem_bytes(dtype);
  if (ranges_overlap(k_next, buf_bytes, k_buf, buf_bytes) ||
      ranges_overlap(k_next, buf_bytes, v_buf, buf_bytes) ||
      ranges_overlap(v_next, buf_bytes, k_buf, buf_bytes) ||
      ranges_overlap(v_next, buf_bytes, v_buf, buf_bytes) ||
      ranges_overlap(k_next, buf_bytes, v_next, buf_bytes))
    return fail(FC_ERR_INVALID_ARG, "k_next / v_next overlap the current buffers or each other");
  if (!(scale > 0.0f)) scale = 1.0f / sqrtf((float)d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  float* imp = reinterpret_cast<float*>(w + lay.imp);
  float* red = reinterpret_cast<float*>(w + lay.red);
  int32_t* sel = idx != nullptr ? idx : reinterpret_cast<int32_t*>(w + lay.idx);
  const bool bf16 = dtype == FC_BF16;
  // The candidates are the first n_clean + C rows of each head; the heads are
  // cap rows apart.
  const int L = n_clean + C;
  cudaError_t e =
      (bf16 && fc::importance_tc_supported(d))
          ? fc::launch_importance_tc(q, k_buf, H, Lq, L, d, scale, imp, w, s, cap)
          : fc::launch_importance_simt(q, k_buf, bf16, H, Lq, L, d, scale, imp, w, s, cap);
  if (e == cudaSuccess)
    e = fc::launch_redundancy(k_buf, bf16, H, L, d, red, w + lay.red_ws, s, cap);
  if (e == cudaSuccess)
    e = fc::launch_score_topb(imp, red, H, L, pool_window, lambda, B_budget, nullptr, sel,
                              w + lay.score_ws, s);
  if (e == cudaSuccess)
    e = fc::launch_compact(k_buf, v_buf, (int)elem_bytes(dtype), H, L, d, sel, B_budget, cap,
                           k_next, v_next, s, cap);
  st = launched(e, "fc_kv_cache_commit");
  if (st == FC_OK) {
    *n_next = B_budget;
    *compressed = 1;
  }
  return st;
}

fc_status fc_selftest_exp2(const float* x, float* y_mufu, float* y_poly, int n, void* stream) {
  fc::g_launches = 0;
  if (n < 0 || n % 2 != 0) return fail(FC_ERR_INVALID_ARG, "n must be even and >= 0");
  if (n == 0) return ok();
  FC_CHECK_PTR(x);
  FC_CHECK_PTR(y_mufu);
  FC_CHECK_PTR(y_poly);
  return launched(fc::launch_exp2_selftest(x, y_mufu, y_poly, n, static_cast<cudaStream_t>(stream)),
                  "fc_selftest_exp2");
}

fc_status fc_selftest_wait_timeout(long long limit_cycles, int* err, void* stream) {
  fc::g_launches = 0;
  if (limit_cycles < 0 || limit_cycles > 4000000000ll)
    return fail(FC_ERR_INVALID_ARG, "limit_cycles must be in [0, 4e9]");
  FC_CHECK_PTR(err);
  return launched(fc::launch_wait_selftest(limit_cycles, err, static_cast<cudaStream_t>(stream)),
                  "fc_selftest_wait_timeout");
}

}  // extern "C"

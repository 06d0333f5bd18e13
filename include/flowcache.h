/*
 * libflowcache -- FlowCache's per-step hot path for NVIDIA B200 (sm_100a).
 *
 * Method: "Flow Caching for Autoregressive Video Generation" (paper notes on
 * papernotes.org, ICLR 2026), section 方法详解 / 关键设计 (method details / key
 * designs) 1-3.  Two parts:
 *   - the chunkwise cache gate (key designs 1 and 2): a fused Euler update with
 *     per-chunk relative-L1 reductions and the recursive accumulator f that
 *     decides, per chunk, whether the next forward recomputes or reuses;
 *   - the joint importance-redundancy KV-cache compression (key design 3):
 *     importance, redundancy, pooled joint score, per-head top-B, and the
 *     compaction of the kept K/V rows into the fixed B_budget buffer.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer (cudaMalloc / torch CUDA
 *     memory / managed memory) owned by the caller.  The library allocates
 *     nothing and keeps no state between calls, except the static scratch
 *     array that fc_chunk_l1_gate_noalloc uses instead of a workspace.  Host
 *     pointers are rejected with FC_ERR_INVALID_ARG before anything is
 *     launched.
 *   - Tensors are dense, row-major, with the stated layout, and their base
 *     address is 16-byte aligned.  "[H][L][d]" means head-major.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: they enqueue kernels and return.
 *   - Arguments are validated on the host before any launch.  On any error
 *     status nothing has been launched and no output was touched, except
 *     FC_ERR_CUDA, which reports a failed launch (the message names it).
 *     fc_last_error() returns a thread-local description of the last error.
 *   - `ws` is caller-owned device scratch of at least the size returned by the
 *     matching *_workspace_size() query.  Its contents are clobbered, except
 *     where a call says otherwise.  Two calls that run at the same time on the
 *     GPU must not share a workspace.
 *   - Results are deterministic: the same inputs and sizes give bitwise the
 *     same outputs (no floating-point atomics).
 */
#ifndef FLOWCACHE_H
#define FLOWCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FC_OK = 0,
  FC_ERR_INVALID_ARG = 1, /* a null / host / misaligned pointer or a bad size     */
  FC_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement         */
  FC_ERR_WORKSPACE = 3,   /* ws is null or smaller than the *_workspace_size()     */
  FC_ERR_CUDA = 4,        /* a CUDA call failed; see fc_last_error()               */
  FC_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (fc_check_workspace) */
} fc_status;

typedef enum { FC_F32 = 0, FC_BF16 = 1 } fc_dtype;

/* Thread-local text of the last error reported on this thread ("" if none). */
const char* fc_last_error(void);

/* Library version, as major*10000 + minor*100 + patch. */
int fc_version(void);

/*
 * Failure detection for the calls whose kernels wait on the device (the
 * importance and the cache commit; the gate's kernel has no device-side waits
 * and leaves its word zero, but its workspace keeps the word): every such
 * wait is bounded, and a wait that gives up sets a 32-bit error word in the
 * call's workspace and lets the kernel return instead of hanging.  The calls
 * are asynchronous, so the word is read here, after the work is done.
 *
 *   kind      which call's workspace ws is (the word's place differs)
 *   ws        the workspace passed to that call (ignored for FC_WS_GATE_NOALLOC,
 *             whose scratch is the library's own on the current device)
 *   n_chunks  the call's n_chunks (gate kinds only)
 *   clear     nonzero: reset a set word to zero after reading it
 * Synchronises `stream`, then returns FC_OK if the word is zero and
 * FC_ERR_TIMEOUT if it is set (the outputs of the calls made since it was last
 * zero are not valid).  Bad arguments -> FC_ERR_INVALID_ARG; a failed read ->
 * FC_ERR_CUDA.  The pages have no counterpart: this is the library's own.
 */
typedef enum {
  FC_WS_GATE = 0,          /* fc_chunk_l1_gate / fc_history_l1_gate workspace  */
  FC_WS_GATE_NOALLOC = 1,  /* fc_chunk_l1_gate_noalloc's static scratch       */
  FC_WS_IMPORTANCE = 2,    /* fc_kv_importance workspace                      */
  FC_WS_CACHE = 3          /* fc_kv_cache_commit workspace                    */
} fc_ws_kind;
fc_status fc_check_workspace(fc_ws_kind kind, const void* ws, int n_chunks, int clear,
                             void* stream);

/* Kernel launches (memsets included) that the last compute call made on this
 * host thread enqueued; 0 after an error.  For accounting in benchmarks. */
int fc_last_launches(void);

/* ------------------------------------------------------------------------ */
/* Chunkwise cache gate (key design 1: relative L1 distance; key design 2:  */
/* the accumulator f)                                                       */
/* ------------------------------------------------------------------------ */

/* Workspace bytes for fc_chunk_l1_gate. */
size_t fc_gate_workspace_size(int n_chunks, int64_t n_per_chunk);

/*
 * One denoising step of the chunkwise cache gate for every chunk.
 *
 * Key design 1 defines, for chunk i at step t, the relative L1 distance
 *   L1_rel = ||X_{t-1} - X_t||_1 / ||X_t||_1 = ||v*dt||_1 / ||X_t||_1.
 * Key design 2 keeps a per-chunk accumulator f: the first m steps of a chunk
 * recompute (f = 0); afterwards, if f + L1_rel > eps the chunk recomputes
 * and f resets to 0, otherwise f += L1_rel and the chunk reuses its cached
 * activations.
 *
 * In one pass this call applies the Euler update X <- X + v*dt (float32:
 * the product rounded once, then the sum rounded once; no fused
 * multiply-add), forms ||v*dt||_1 and ||X_t||_1 (pre-update X) in float64,
 * and runs the recurrence (in float32, compare strictly greater).
 *
 *   x          [n_chunks][n_per_chunk] float32, in/out: X_t in, X_{t-1} out
 *   v          [n_chunks][n_per_chunk] float32, velocity applied this step
 *   dt         [n_chunks] float32, signed step of each chunk
 *   step       [n_chunks] int32, steps chunk c has taken since it started;
 *              step < 0 marks an inactive chunk: x, f untouched, l1 = 0,
 *              recompute = 0
 *   m          forced-recompute steps (>= 0)
 *   eps        threshold
 *   f          [n_chunks] float32, in/out accumulator
 *   l1_rel     [n_chunks] float32, out: L1_rel (+inf when ||X_t||_1 = 0 and
 *              the update is not zero; 0 when both are zero)
 *   recompute  [n_chunks] uint8, out: 1 = recompute at the chunk's next
 *              forward, 0 = reuse
 *   ws         fc_gate_workspace_size() bytes.  Its first 4*(n_chunks+1)
 *              bytes (completion counters and an error word) must be zero
 *              before the first call (e.g. cudaMemsetAsync once); every call
 *              leaves the counters zero again.  The error word (the 32-bit
 *              word after the n_chunks counters) is reserved: this kernel
 *              has no device-side waits and never sets it.
 * x and v may be NULL when n_per_chunk == 0 (then L1_rel = 0 for every
 * active chunk).  x and v must not overlap (x is written while v is read).
 * Errors: n_chunks < 1, n_per_chunk < 0, m < 0, null/host/misaligned
 * pointers, overlapping x and v -> FC_ERR_INVALID_ARG; small ws ->
 * FC_ERR_WORKSPACE.
 */
fc_status fc_chunk_l1_gate(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                           const float* dt, const int32_t* step, int32_t m, float eps,
                           float* f, float* l1_rel, uint8_t* recompute, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * History-guided variant of the gate, for the neighbouring method of the notes
 * "Accelerating Autoregressive Video Diffusion via History-Guided Cache and
 * Residual Correction" (papernotes.org), 关键设计 1 (HGC).  Per segment:
 *   Delta = ||h_t - h_{t+1}||_1 / ||h_{t+1}||_1  (denominator: the older step),
 * and the cache refreshes at the step where the deviations summed since the
 * last refresh step t_ref (inclusive) first exceed delta:
 *   sum_{i=t+1}^{t_ref} Delta <= delta < sum_{i=t}^{t_ref} Delta.
 * The refresh step becomes t_ref, so f restarts at that step's own Delta
 * (where fc_chunk_l1_gate resets to 0).  The first m steps of a segment
 * refresh unconditionally.  Same kernels, reductions and precision as
 * fc_chunk_l1_gate: h_t - h_{t+1} is rounded once in float32, both norms are
 * summed in float64, the recurrence runs in float32.
 *
 *   h_old     [n][N] float32, in/out: h_{t+1} in, h_t out (for active segments)
 *   h_new     [n][N] float32, h_t; must not overlap h_old
 *   step      [n] int32, steps since the segment started; < 0: inactive, untouched
 *   m, delta  forced refresh steps, threshold
 *   f         [n] float32, in/out window sum
 *   d_rel     [n] float32, out: Delta
 *   refresh   [n] uint8, out: 1 = refresh (recompute) at this step
 *   ws        fc_gate_workspace_size(n, N) bytes, same contract as the gate's
 * Errors as for fc_chunk_l1_gate.
 */
fc_status fc_history_l1_gate(float* h_old, const float* h_new, int n_segments,
                             int64_t n_per_segment, const int32_t* step, int32_t m, float delta,
                             float* f, float* d_rel, uint8_t* refresh, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * Allocation-free variant of fc_chunk_l1_gate.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory when
 * they run the gate -- for example a host runtime that hands its plugins only
 * input and output buffers and forbids cudaMalloc while work is enqueued (an
 * allocation can synchronize the device or fail under a fixed memory budget),
 * or code with nowhere to keep a workspace alive between steps.
 *
 * Same arguments, results and errors as fc_chunk_l1_gate, without ws/ws_bytes.
 * The scratch (completion counters and per-block partial sums) is one static
 * device array of about 512 KiB inside the library, which every GPU that loads
 * the library holds until the process exits.  Limits and behaviour:
 *   - n_chunks must be in [1, 32]; larger counts return FC_ERR_INVALID_ARG
 *     before anything is launched (use fc_chunk_l1_gate with a workspace).
 *   - The call allocates nothing: no cudaMalloc, cudaFree or allocating
 *     library routine.  It clears the counters it needs with an asynchronous
 *     memset on `stream`, then launches the gate kernel.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept per device together
 *     with the id of the context it belongs to; a call made after the
 *     device's context was destroyed and created again (cudaDeviceReset)
 *     looks it up again, so make the first call after a reset outside
 *     stream capture too.  Host threads may make their first calls at the
 *     same time: the lookup is serialised by a lock.
 *   - Every call shares the one array: calls whose work overlaps on the GPU
 *     (other streams, other host threads) race and give wrong results; order
 *     them on one stream or with events.
 */
fc_status fc_chunk_l1_gate_noalloc(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                                   const float* dt, const int32_t* step, int32_t m, float eps,
                                   float* f, float* l1_rel, uint8_t* recompute, void* stream);

/*
 * Consumer of the recompute mask (the flowchart of 整体框架 and key design 2:
 * chunks marked for recompute run the model forward, the others reuse their
 * cached activations).  Gathers, in chunk order, the latents of the chunks
 * with recompute[c] != 0 into the first rows of a dense batch.
 *
 *   x          [n_chunks][n_per_chunk] float32
 *   recompute  [n_chunks] uint8 (the gate's output)
 *   dense      [n_chunks][n_per_chunk] float32 out: rows 0..count-1 are the
 *              recompute chunks' latents; rows >= count are not written
 *   ids        [n_chunks] int32 out: ids[i] = chunk of dense row i, -1 past count
 *   count      [1] int32 out (device): number of recompute chunks
 * Everything stays on the device (no host synchronisation).  Bitwise copy.
 * Errors: bad sizes or pointers -> FC_ERR_INVALID_ARG.
 */
fc_status fc_gather_recompute(const float* x, const uint8_t* recompute, int n_chunks,
                              int64_t n_per_chunk, float* dense, int32_t* ids, int32_t* count,
                              void* stream);

/*
 * The other half: after the forward of the dense batch, v_cache[ids[i]] =
 * v_dense[i] for i < *count; the reused chunks keep their cached velocity.
 *
 *   v_dense  [n_chunks][n_per_chunk] float32, fresh velocities of the batch
 *   ids, count  as written by fc_gather_recompute
 *   v_cache  [n_chunks][n_per_chunk] float32 in/out; must not overlap v_dense
 */
fc_status fc_scatter_velocity(const float* v_dense, const int32_t* ids, const int32_t* count,
                              int n_chunks, int64_t n_per_chunk, float* v_cache, void* stream);

/* ------------------------------------------------------------------------ */
/* Joint importance-redundancy KV compression (key design 3)                */
/* ------------------------------------------------------------------------ */

/* Workspace bytes for fc_kv_importance. */
size_t fc_importance_workspace_size(fc_dtype dtype, int H, int Lq, int Lk, int d);

/*
 * Pre-pooling importance of every clean key, per head (key design 3):
 *   Imp[h][j] = (1/Lq) * sum_q softmax_j(scale * q_q . k_j),
 * the attention softmax of the current denoising queries over the Lk clean
 * candidate keys, averaged over the queries.  Computed in two passes over
 * Q K^T: the row log-sum-exp of every query, then the column sums of
 * exp(s - lse).  Accumulation and softmax in float32.
 *
 *   q      [H][Lq][d] dtype, denoising queries
 *   k      [H][Lk][d] dtype, clean keys
 *   dtype  FC_BF16 (tensor-core path) or FC_F32 (CUDA-core path)
 *   d      64 or 128
 *   scale  logit scale; <= 0 selects 1/sqrt(d)
 *   imp    [H][Lk] float32, out; each row sums to 1
 *   ws     fc_importance_workspace_size() bytes: bytes 0..3 are an error
 *          word that the tensor-core path sets to nonzero if one of its
 *          bounded device-side waits gave up (the call never clears it; zero
 *          it once; read it with fc_check_workspace); the per-query log-sum-exp
 *          normalisers (split into bf16 terms) follow from byte 256
 * Errors: H, Lq, Lk < 1 or d not in {64, 128} -> FC_ERR_INVALID_ARG /
 * FC_ERR_UNSUPPORTED; bad pointers -> FC_ERR_INVALID_ARG; small ws ->
 * FC_ERR_WORKSPACE.
 */
fc_status fc_kv_importance(const void* q, const void* k, fc_dtype dtype, int H, int Lq, int Lk,
                           int d, float scale, float* imp, void* ws, size_t ws_bytes,
                           void* stream);

/* Workspace bytes for fc_kv_redundancy. */
size_t fc_redundancy_workspace_size(fc_dtype dtype, int H, int Lk, int d);

/*
 * Redundancy of every clean key, per head (key design 3):
 *   Red[h][j] = softmax_j( (1/Lk) * sum_{i != j} khat_i . khat_j ),
 * khat the l2-normalised keys (a zero key stays zero), i.e. the softmax of the
 * column means of the cosine-similarity matrix with its diagonal zeroed.
 * Evaluated with the exact identity sum_{i != j} khat_i.khat_j =
 * khat_j.(sum_i khat_i) - ||khat_j||^2, so that K is streamed instead of the
 * Lk x Lk matrix being formed.  The sums over a head's keys (of khat, and of
 * exp(r_j) for the softmax) are accumulated in 2^-32 fixed point in 64-bit
 * integers, so the result is bitwise the same whatever the order in which
 * the GPU finishes the pieces, and does not depend on H.  Heads are processed
 * in groups, one group's sum overlapping the previous group's logits.
 *
 *   k    [H][Lk][d] dtype
 *   red  [H][Lk] float32, out; each row sums to 1
 *   ws   fc_redundancy_workspace_size() bytes; no contents carried between
 *        calls (the call clears what it uses)
 * Errors as for fc_kv_importance; Lk > 2^26 -> FC_ERR_UNSUPPORTED.
 */
fc_status fc_kv_redundancy(const void* k, fc_dtype dtype, int H, int Lk, int d, float* red,
                           void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes for fc_kv_score_topb. */
size_t fc_score_topb_workspace_size(int H, int Lk, int B);

/*
 * Joint score and per-head top-B selection (key design 3):
 *   Imp~ = 1D max filter of imp along the token axis (odd `pool_window`,
 *          stride 1, output length Lk, taps outside [0, Lk) ignored),
 *   Score[h][j] = lambda*Imp~[h][j] - (1-lambda)*Red[h][j], evaluated in
 *          float32 as fl(fl(lambda*Imp~) - fl(fl(1-lambda)*Red)),
 *   idx[h] = the B tokens with the largest Score; equal scores keep the lower
 *          token index (-0 and +0 are equal); indices written ascending, which
 *          keeps the temporal order of the kept tokens.
 * B >= Lk keeps every token: idx[h][r] = r for r < Lk, -1 for r >= Lk.
 *
 *   imp, red     [H][Lk] float32 (outputs of the two calls above)
 *   pool_window  odd, in [1, 511]
 *   lambda       mixing weight (not clamped)
 *   B            >= 1, tokens kept per head
 *   score        [H][Lk] float32 out, or NULL to skip writing it
 *   idx          [H][B] int32 out
 * Errors: B < 1, pool_window even or out of range, bad pointers ->
 * FC_ERR_INVALID_ARG;
 * small ws -> FC_ERR_WORKSPACE.
 */
fc_status fc_kv_score_topb(const float* imp, const float* red, int H, int Lk, int pool_window,
                           float lambda, int B, float* score, int32_t* idx, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Compaction of the kept rows into the fixed-budget buffer (key design 3: the
 * compressed clean region B_budget of the fixed KV buffer):
 *   k_out[h][r] = k[h][idx[h][r]],  v_out[h][r] = v[h][idx[h][r]],
 * rows whose index is -1 are written as zeros.  Bitwise copy.
 *
 *   k, v          [H][Lk][d] dtype
 *   idx           [H][B] int32, each entry in [0, Lk) or -1
 *   k_out, v_out  [H][B][d] dtype, out; must not overlap k or v
 * Errors: bad sizes or pointers, overlapping buffers -> FC_ERR_INVALID_ARG.
 * An index outside [-1, Lk) is not read: the row is written as zeros.
 */
fc_status fc_kv_compact(const void* k, const void* v, fc_dtype dtype, int H, int Lk, int d,
                        const int32_t* idx, int B, void* k_out, void* v_out, void* stream);

/* ------------------------------------------------------------------------ */
/* Cache buffer management around compression (key design 3 and the         */
/* flowchart: finished chunks enter the KV cache; when the reserved cache  */
/* is full the new chunk is merged and every head keeps its top-B tokens)  */
/* ------------------------------------------------------------------------ */

/*
 * Bytes of workspace fc_kv_cache_commit needs (0 for invalid sizes).
 * Bytes 0..3 of that workspace are the importance stage's error word, with
 * the meaning and zero-initialisation rule of fc_kv_importance's.
 */
size_t fc_kv_cache_workspace_size(fc_dtype dtype, int H, int Lq, int B_budget, int C, int d);

/*
 * One chunk that has finished denoising enters the cache.
 *
 * The fixed buffer per head holds cap = B_budget + C rows: rows [0, n_clean)
 * are the compressed clean tokens, rows [n_clean, n_clean + C) the chunk that
 * just finished (the denoising forward wrote its K/V there, so the merge
 * moves nothing).
 *   - If n_clean + C <= B_budget the chunk is kept where it is: *n_next =
 *     n_clean + C, *compressed = 0, nothing is launched and no device pointer
 *     is read (they may be NULL).
 *   - Otherwise the n_clean + C candidates (n_clean + C <= cap) are scored as
 *     fc_kv_importance (queries q), fc_kv_redundancy and fc_kv_score_topb with
 *     B = B_budget would score them,
 *     and the kept rows of every head are written once, in candidate order, to
 *     rows [0, B_budget) of the other buffer (k_next, v_next); rows
 *     [B_budget, cap) of that buffer are not written (the next chunk's K/V go
 *     there).  *n_next = B_budget, *compressed = 1: the caller swaps buffers.
 *
 *   q              [H][Lq][d] dtype, queries of the chunk now denoising
 *   k_buf, v_buf   [H][cap][d] dtype, the current buffer (read only)
 *   k_next, v_next [H][cap][d] dtype, the other buffer; no overlap with the
 *                  current one or with each other
 *   d              64 or 128
 *   C              tokens per chunk, 1 <= C <= B_budget
 *   n_clean        clean rows in [0, B_budget]
 *   scale          softmax scale, <= 0 means 1/sqrt(d)
 *   pool_window, lambda  as for fc_kv_score_topb
 *   idx            [H][B_budget] int32 out (the kept candidate rows,
 *                  ascending), or NULL to keep them in the workspace only
 *   n_next, compressed   host ints, out
 * Errors: bad sizes or pointers, overlapping buffers -> FC_ERR_INVALID_ARG;
 * d not 64/128 -> FC_ERR_UNSUPPORTED; small ws -> FC_ERR_WORKSPACE.  On an
 * error *n_next and *compressed are unchanged.
 */
fc_status fc_kv_cache_commit(const void* q, const void* k_buf, const void* v_buf, void* k_next,
                             void* v_next, fc_dtype dtype, int H, int Lq, int d, int B_budget,
                             int C, int n_clean, float scale, int pool_window, float lambda,
                             int32_t* idx, void* ws, size_t ws_bytes, int* n_next,
                             int* compressed, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLOWCACHE_H */

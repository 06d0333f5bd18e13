// Internal launchers of libflowcache.  Each returns the CUDA error of its
// launches (cudaSuccess when everything was enqueued).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fc {

// ---- chunkwise gate --------------------------------------------------------
size_t gate_ws_bytes(int n_chunks);
// history = false: FlowCache (x += v*dt); true: history gate (x: older
// snapshot, v: newer snapshot, dt unused; x <- v after the step).
cudaError_t launch_gate(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                        const float* dt, const int32_t* step, int m, float eps, float* f,
                        float* l1, uint8_t* mask, void* ws, cudaStream_t s, bool history);

// Same kernel with its scratch in a static device array (no allocation, at
// most gate_noalloc_max_chunks() chunks; calls must not overlap on the GPU).
int gate_noalloc_max_chunks();
// Device address of the no-alloc gate's static scratch on the current device.
cudaError_t gate_noalloc_scratch(void** out);
cudaError_t launch_gate_noalloc(float* x, const float* v, int n_chunks, int64_t n_per_chunk,
                                const float* dt, const int32_t* step, int m, float eps, float* f,
                                float* l1, uint8_t* mask, cudaStream_t s);

// ---- consumer of the recompute mask ------------------------------------------
cudaError_t launch_gather_recompute(const float* x, const uint8_t* mask, int n_c, int64_t N,
                                    float* dense, int32_t* ids, int32_t* count, cudaStream_t s);
cudaError_t launch_scatter_velocity(const float* v_dense, const int32_t* ids, const int32_t* count,
                                    int n_c, int64_t N, float* v_cache, cudaStream_t s);

// ---- importance --------------------------------------------------------------
size_t importance_ws_bytes(int H, int Lq);
// bf16 tensor-core path (tcgen05 + TMEM + TMA)
// ldk (here and below): rows between consecutive heads of k (and v); <= 0
// means Lk (dense heads).  Only the first Lk rows of a head are read.
cudaError_t launch_importance_tc(const void* q, const void* k, int H, int Lq, int Lk, int d,
                                 float scale, float* imp, void* ws, cudaStream_t s, int ldk = 0);
bool importance_tc_supported(int d);
// A bounded mbarrier wait that nothing completes, for the self-test
cudaError_t launch_wait_selftest(long long limit_cycles, int* err, cudaStream_t s);
// 2^x on the special-function unit and on the FMA pipes, for the self-test
cudaError_t launch_exp2_selftest(const float* x, float* y_mufu, float* y_poly, int n,
                                 cudaStream_t s);
// CUDA-core path (float32 or bf16 inputs)
cudaError_t launch_importance_simt(const void* q, const void* k, bool bf16, int H, int Lq,
                                   int Lk, int d, float scale, float* imp, void* ws,
                                   cudaStream_t s, int ldk = 0);

// ---- redundancy ----------------------------------------------------------------
size_t redundancy_ws_bytes(int H, int Lk, int d);
// Largest L_k the redundancy's fixed-point accumulators serve.
int redundancy_max_lk();
cudaError_t launch_redundancy(const void* k, bool bf16, int H, int Lk, int d, float* red,
                              void* ws, cudaStream_t s, int ldk = 0);

// ---- score + top-B ---------------------------------------------------------------
size_t score_topb_ws_bytes(int H, int Lk);
cudaError_t launch_score_topb(const float* imp, const float* red, int H, int Lk, int pool,
                              float lambda, int B, float* score, int32_t* idx, void* ws,
                              cudaStream_t s);

// ---- compaction ------------------------------------------------------------------
cudaError_t launch_compact(const void* k, const void* v, int elem_bytes, int H, int Lk, int d,
                           const int32_t* idx, int B, int ldo, void* k_out, void* v_out,
                           cudaStream_t s, int ldk = 0);

}  // namespace fc

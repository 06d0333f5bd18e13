/*
 * A plain C consumer of libflowcache: no Python, no PyTorch, only the header
 * and the CUDA runtime.  Mode "host" checks what needs no GPU (version,
 * workspace sizes, argument validation and its messages).  Mode "gpu" also
 * runs the hand-worked gate trace of the Flow Caching notes (key designs 1
 * and 2: X = 1, v = 1, dt = -1/64 over 1024 elements gives L1_rel = 1/64 per
 * step; with m = 2 and eps = 0.05 the masks are 1,1,0,0,0,1,0,0,0,1) on
 * cudaMalloc'd buffers and compares every step exactly.
 * Exit status 0 on success; the first failed check is printed.
 */
#include <stdio.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "flowcache.h"

#define CHECK(cond, what)                                   \
  do {                                                      \
    if (!(cond)) {                                          \
      fprintf(stderr, "FAILED: %s (%s:%d)\n", what, __FILE__, __LINE__); \
      return 1;                                             \
    }                                                       \
  } while (0)

static int host_checks(void) {
  CHECK(fc_version() >= 100, "fc_version");
  CHECK(fc_gate_workspace_size(4, 1024) > 0, "gate workspace size");
  CHECK(fc_gate_workspace_size(0, 1024) == 0, "gate workspace size of 0 chunks");
  CHECK(fc_importance_workspace_size(FC_BF16, 2, 64, 64, 128) > 0, "importance workspace");
  CHECK(fc_redundancy_workspace_size(FC_BF16, 2, 64, 96) == 0, "redundancy d = 96");
  /* validation happens on the host and names the bad argument */
  fc_status st = fc_chunk_l1_gate(NULL, NULL, 0, 16, NULL, NULL, 1, 0.1f, NULL, NULL, NULL,
                                  NULL, 0, NULL);
  CHECK(st == FC_ERR_INVALID_ARG, "n_chunks = 0 rejected");
  CHECK(strstr(fc_last_error(), "n_chunks") != NULL, "message names n_chunks");
  st = fc_kv_importance(NULL, NULL, FC_BF16, 2, 8, 8, 96, 0.0f, NULL, NULL, 0, NULL);
  CHECK(st == FC_ERR_UNSUPPORTED, "d = 96 unsupported");
  st = fc_kv_score_topb(NULL, NULL, 2, 8, 6, 0.5f, 4, NULL, NULL, NULL, 1 << 20, NULL);
  CHECK(st == FC_ERR_INVALID_ARG, "even pool window rejected");
  CHECK(fc_last_launches() == 0, "nothing launched on an error");
  return 0;
}

static int gpu_trace(void) {
  enum { N = 1024, STEPS = 10 };
  const int m = 2;
  const float eps = 0.05f, dt_h = -0.015625f;
  const unsigned char want_mask[STEPS] = {1, 1, 0, 0, 0, 1, 0, 0, 0, 1};
  const float want_f[STEPS] = {0.0f, 0.0f, 0.015625f, 0.03125f, 0.046875f,
                               0.0f, 0.015625f, 0.03125f, 0.046875f, 0.0f};
  float ones[N], x_h[N];
  for (int i = 0; i < N; ++i) ones[i] = 1.0f;
  float *x, *v, *dt, *f, *l1;
  int *step;
  unsigned char* mask;
  void* ws;
  size_t ws_bytes = fc_gate_workspace_size(1, N);
  CHECK(cudaMalloc((void**)&x, N * sizeof(float)) == cudaSuccess, "cudaMalloc x");
  CHECK(cudaMalloc((void**)&v, N * sizeof(float)) == cudaSuccess, "cudaMalloc v");
  CHECK(cudaMalloc((void**)&dt, 16) == cudaSuccess && cudaMalloc((void**)&f, 16) == cudaSuccess &&
            cudaMalloc((void**)&l1, 16) == cudaSuccess &&
            cudaMalloc((void**)&step, 16) == cudaSuccess &&
            cudaMalloc((void**)&mask, 16) == cudaSuccess && cudaMalloc(&ws, ws_bytes) == cudaSuccess,
        "cudaMalloc small buffers");
  CHECK(cudaMemset(ws, 0, ws_bytes) == cudaSuccess && cudaMemset(f, 0, 16) == cudaSuccess,
        "zero ws and f");
  CHECK(cudaMemcpy(v, ones, sizeof(ones), cudaMemcpyHostToDevice) == cudaSuccess, "copy v");
  CHECK(cudaMemcpy(dt, &dt_h, sizeof(float), cudaMemcpyHostToDevice) == cudaSuccess, "copy dt");
  for (int t = 0; t < STEPS; ++t) {
    CHECK(cudaMemcpy(x, ones, sizeof(ones), cudaMemcpyHostToDevice) == cudaSuccess, "reset x");
    CHECK(cudaMemcpy(step, &t, sizeof(int), cudaMemcpyHostToDevice) == cudaSuccess, "copy step");
    fc_status st = fc_chunk_l1_gate(x, v, 1, N, dt, step, m, eps, f, l1, mask, ws, ws_bytes, NULL);
    CHECK(st == FC_OK, fc_last_error());
    float l1_h, f_h;
    unsigned char mask_h;
    CHECK(cudaMemcpy(&l1_h, l1, 4, cudaMemcpyDeviceToHost) == cudaSuccess &&
              cudaMemcpy(&f_h, f, 4, cudaMemcpyDeviceToHost) == cudaSuccess &&
              cudaMemcpy(&mask_h, mask, 1, cudaMemcpyDeviceToHost) == cudaSuccess &&
              cudaMemcpy(x_h, x, sizeof(x_h), cudaMemcpyDeviceToHost) == cudaSuccess,
          "read back");
    CHECK(l1_h == 0.015625f, "L1_rel = 1/64");
    CHECK(mask_h == want_mask[t], "recompute mask");
    CHECK(f_h == want_f[t], "accumulator f");
    for (int i = 0; i < N; ++i) CHECK(x_h[i] == 0.984375f, "Euler update 1 - 1/64");
  }
  CHECK(fc_check_workspace(FC_WS_GATE, ws, 1, 0, NULL) == FC_OK, "no wait gave up");
  cudaFree(x);
  cudaFree(v);
  cudaFree(dt);
  cudaFree(f);
  cudaFree(l1);
  cudaFree(step);
  cudaFree(mask);
  cudaFree(ws);
  return 0;
}

int main(int argc, char** argv) {
  if (host_checks() != 0) return 1;
  if (argc > 1 && strcmp(argv[1], "gpu") == 0 && gpu_trace() != 0) return 1;
  printf("ok\n");
  return 0;
}

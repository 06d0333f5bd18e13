/*
 * libflowcache self-test entry points.  Not part of the method: they expose
 * internal device arithmetic so that tests can check it against known error
 * bounds.  Same conventions as flowcache.h (device pointers, asynchronous on
 * `stream`, host-side validation, fc_last_error()).
 */
#ifndef FLOWCACHE_SELFTEST_H
#define FLOWCACHE_SELFTEST_H

#include "flowcache.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Evaluate 2^x for n inputs (n even) with the two exponentials the
 * tensor-core importance kernel mixes: y_mufu from the special-function unit
 * (ex2.approx.ftz.f32) and y_poly from the FMA-pipe range reduction +
 * polynomial the kernel uses (degree 3, relative error below 7.6e-5).
 * x, y_mufu, y_poly: [n] float32 device buffers.
 * The polynomial path clamps x below -125 to -125 and requires x <= 126.
 * Errors: n odd or negative, bad pointers -> FC_ERR_INVALID_ARG.
 */
fc_status fc_selftest_exp2(const float* x, float* y_mufu, float* y_poly, int n, void* stream);

/*
 * Failure-path self-test of the bounded device-side waits the tensor-core and
 * streaming kernels use: one CTA waits on an mbarrier that nothing arrives on,
 * gives up after `limit_cycles` SM clocks, and adds 1 to *err (a device int
 * the caller zeroes).  The kernel then returns normally: the context stays
 * usable.  limit_cycles in [0, 4e9] (4e9 ~ 2 s at 1.9 GHz).
 */
fc_status fc_selftest_wait_timeout(long long limit_cycles, int* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLOWCACHE_SELFTEST_H */

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
 * degree-5 polynomial.  x, y_mufu, y_poly: [n] float32 device buffers.
 * The polynomial path clamps x below -125 to -125 and requires x <= 126.
 * Errors: n odd or negative, bad pointers -> FC_ERR_INVALID_ARG.
 */
fc_status fc_selftest_exp2(const float* x, float* y_mufu, float* y_poly, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLOWCACHE_SELFTEST_H */

/*
 * qlinear_testing.h - hooks that let tests exercise the library's failure
 * detection without faulting a GPU.  Not part of the layer's computation.
 *
 * Every pipeline wait in the library's kernels is bounded: instead of
 * spinning forever on a barrier that never completes (a lost copy, a bug),
 * the kernel gives up after a time limit, sets QL_ERR_TIMEOUT in the
 * caller's device status word, releases what it holds and returns, so the
 * CUDA context stays usable.
 */
#ifndef QLINEAR_TESTING_H
#define QLINEAR_TESTING_H

#include <stdint.h>

#include "qlinear.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Launch one small kernel whose thread waits, through the same bounded
 * mbarrier wait the GEMM and streaming kernels use, on a barrier that nothing
 * ever arrives at, with a limit of limit_us microseconds (1 .. 10^7).  The
 * wait runs out, the kernel ORs (1u << QL_ERR_TIMEOUT) into *d_status and
 * returns.  Asynchronous on `stream`; returns QL_ERR_ARG for a bad limit or
 * NULL status, QL_ERR_CUDA if the launch fails. */
QL_API int ql_test_wait_timeout(int32_t *d_status, uint32_t limit_us, void *stream);

/* The float32 reciprocal and quotient steps the SwiGLU gate kernels and the
 * optimizer updates use (Markstein's correction steps on the approximate
 * hardware reciprocal), applied elementwise to device arrays of n values:
 * y[i] = 1/d[i] and q[i] = a[i]/d[i], each meant to equal the correctly
 * rounded (IEEE round-to-nearest-even) result.  Operands outside the steps'
 * ranges (the gate's: 1 <= d <= 2^24 with 2^-90 <= |a| <= 2^100; the wide
 * one: d in [2^-60, 2^60] with a zero or in +-[2^-60, 2^60]) take the IEEE
 * division; y[i] is then 1/d[i] by IEEE division
 * too.  A zero a may give a zero of either sign.  Asynchronous on `stream`;
 * QL_ERR_ARG for n < 0 or a NULL pointer with n > 0, QL_ERR_CUDA if the
 * launch fails. */
QL_API int ql_test_divrn(const float *a, const float *d, int64_t n, float *q, float *y,
                         void *stream);

/* The float32 square-root steps of the optimizer updates (Markstein's
 * correction on the approximate reciprocal square root), elementwise on n
 * device values: s_plain[i] from the approximate root as it comes,
 * s_refined[i] after one Newton step on it; each meant to equal the
 * correctly rounded sqrt(v[i]).  Values outside the steps' range (negative,
 * below 2^-100 other than zero, above 2^100, inf, NaN) take the IEEE square
 * root.  Asynchronous on `stream`; QL_ERR_ARG for n < 0 or a NULL pointer
 * with n > 0, QL_ERR_CUDA if the launch fails. */
QL_API int ql_test_sqrtrn(const float *v, int64_t n, float *s_plain, float *s_refined,
                          void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_TESTING_H */

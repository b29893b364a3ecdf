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

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_TESTING_H */

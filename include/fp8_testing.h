/*
 * fp8_testing.h -- a testing entry point of libfp8.so.  Not for production use.
 *
 * The source pages have no counterpart: this hook exists so that tests can drive
 * the failure path of the kernels' bounded waits without faulting or hanging a GPU.
 *
 * Every mbarrier wait in the GEMM kernels (fp8_scaled_gemm, fp8_linear_forward and
 * their _ex forms, fp8_weight_only_linear) is bounded by a time limit, 4 s by
 * default.  When a wait runs out, the CTA sets FP8_ERR_TIMEOUT in dev_status, tells
 * its other warps to stop, waits (itself bounded) until the TMA copies and the
 * tensor-core operations it has already issued are complete, frees its tensor
 * memory and exits; the CUDA context stays usable and the outputs of that call are
 * unspecified.
 */
#ifndef FP8_B200_TESTING_H
#define FP8_B200_TESTING_H

#include "fp8.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fp8_testing_set_wait_limit_ns -- the limit, in nanoseconds, of each pipeline wait
 * in the GEMM kernels launched after this call from any thread of the process; 0
 * restores the default (4 s).  A limit shorter than the kernel's own pipeline
 * latency makes the waits run out, which is what a test of the failure path wants.
 * The setting is process-wide and not synchronised with launches on other threads.
 */
FP8_API void fp8_testing_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* FP8_B200_TESTING_H */

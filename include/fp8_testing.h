/*
 * fp8_testing.h -- testing entry points of libfp8.so.  Not for production use.
 *
 * The source pages have no counterpart for either: the first exists so that tests
 * can drive the failure path of the kernels' bounded waits without faulting or
 * hanging a GPU, the second so that they can sweep the encode step over every fp32
 * pattern of a range.
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

/*
 * fp8_testing_encode_f32_range -- q[i] = the FP8 code (format fmt) that the quantize
 * kernels' encode step gives the fp32 value whose bit pattern is first_bits + i, for
 * 0 <= i < n: round to nearest even, saturating to +-F_max ([FFS] "Scale 怎样把
 * Tensor 塞进 E4M3": X_fp8 = cast(clip(X / s)); here the value is already X / s).
 *   first_bits  bit pattern of the first value; first_bits + n <= 2^32
 *   n           number of values (0: nothing happens)
 *   fmt         FP8_E4M3 or FP8_E5M2
 *   q           device pointer to n bytes, caller-owned
 *   stream      cudaStream_t or NULL; asynchronous on it
 * Returns FP8_OK, FP8_ERR_INVALID_ARG (format, range, null q), FP8_ERR_UNSUPPORTED_DEVICE
 * or FP8_ERR_CUDA (launch failure).
 */
FP8_API int32_t fp8_testing_encode_f32_range(uint32_t first_bits, int64_t n, int32_t fmt, uint8_t* q, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FP8_B200_TESTING_H */

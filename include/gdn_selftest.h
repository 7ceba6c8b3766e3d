/*
 * gdn_selftest.h -- self-test entry point of the tensor-core building blocks
 * used by the GDN kernels (include/gdn.h).  The pages describe no such call: it
 * checks this library's own operand layouts on the device it runs on.
 */
#ifndef GDN_SELFTEST_H
#define GDN_SELFTEST_H

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * gdn_selftest_umma -- D = init + (+/-A) * B on one CTA with tcgen05.mma
 * (kind::f16, fp16 operands, fp32 accumulation in tensor memory).
 *
 *   A     [128, K] fp16 row-major, device      (K in {64, 128})
 *   B     [K, N]   fp16 row-major, device      (N in {64, 128})
 *   init  [128, N] fp32 device or NULL (then D = +/-A*B)
 *   D     [128, N] fp32 device, written
 *   a_mn        A in shared memory MN-major (1) or K-major (0), or in tensor
 *               memory (2: row m in lane m, elements 2c, 2c+1 in column c)
 *   b_mn        B in shared memory MN-major (1) or K-major (0)
 *   negate_a    use -A (A in shared memory only)
 *
 * Synchronises `stream`.  Returns GDN_ERR_TIMEOUT if the MMA completion wait
 * expired, GDN_ERR_INVALID_ARG for unsupported sizes or NULL buffers.
 */
GDN_API gdn_status_t gdn_selftest_umma(int a_mn, int b_mn, int negate_a, int N, int K,
                                       const void *A, const void *B, const float *init,
                                       float *D, gdn_stream_t stream);

/*
 * gdn_selftest_wait_timeout -- failure-detection check of one kernel family's
 * bounded wait.  Launches one CTA that waits, through the family's own wait
 * routine, for an mbarrier phase that nothing completes; after `max_polls`
 * polls the wait gives up and raises the family's device error word, which
 * gdn_device_error_status then reports.  Nothing faults and the context stays
 * usable.
 *
 *   family     GDN_ERRF_PREP, GDN_ERRF_CHAIN, GDN_ERRF_DECODE, GDN_ERRF_QSA or
 *              GDN_ERRF_GEMM (one bit)
 *   max_polls  1 .. 65536
 *
 * Asynchronous on `stream`.  GDN_ERR_INVALID_ARG for another family value or
 * max_polls out of range, GDN_ERR_CUDA if the launch fails.
 */
GDN_API gdn_status_t gdn_selftest_wait_timeout(unsigned family, unsigned max_polls,
                                               gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_SELFTEST_H */

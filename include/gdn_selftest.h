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
 *   a_mn, b_mn  stage A / B MN-major (1) or K-major (0) in shared memory
 *   negate_a    use -A
 *
 * Synchronises `stream`.  Returns GDN_ERR_TIMEOUT if the MMA completion wait
 * expired, GDN_ERR_INVALID_ARG for unsupported sizes or NULL buffers.
 */
GDN_API gdn_status_t gdn_selftest_umma(int a_mn, int b_mn, int negate_a, int N, int K,
                                       const void *A, const void *B, const float *init,
                                       float *D, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_SELFTEST_H */

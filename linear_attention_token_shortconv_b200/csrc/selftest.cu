// Self-test of the tcgen05 operand layouts the GDN kernels rely on: one CTA
// stages A [128 x K] and B [K x N] (fp16, row-major in global memory) into
// shared memory in the requested K-major or MN-major 128-byte-swizzled layout
// (A alternatively into tensor memory, row m in lane m, K pairs per column),
// runs K/16 tcgen05.mma (kind::f16, fp32 accumulation in TMEM, optionally onto
// an initial value written with tcgen05.st, optionally with A negated) and
// writes D [128 x N] back.  The host compares D with a plain matmul.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/gdn_selftest.h"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

__device__ unsigned int g_selftest_err;

constexpr int kStA = 0;            // A region (64 KB reserved)
constexpr int kStB = 65536;        // B region (64 KB reserved)
constexpr int kStMisc = 131072;    // mbarrier + TMEM slot
constexpr int kStSmem = kStMisc + 64 + 1024;

__global__ void __launch_bounds__(128)
umma_selftest_kernel(int a_mn, int b_mn, int neg_a, int N, int K, const __half *__restrict__ A,
                     const __half *__restrict__ B, const float *__restrict__ init,
                     float *__restrict__ D) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint8_t *As = sm + kStA, *Bs = sm + kStB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kStMisc);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + kStMisc + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) umma::tmem_alloc(tslot, 256);
    if (tid == 0) {
        umma::mbar_init(bar, 1);
        umma::fence_mbar_init();
    }
    // stage A (logical [128][K]) and B (logical [K][N]) as 8-element chunks
    for (int idx = tid; idx < 128 * K / 8; idx += 128) {
        const int m = idx / (K / 8), k8 = idx % (K / 8);
        const uint4 v = reinterpret_cast<const uint4 *>(A + (size_t)m * K)[k8];
        if (a_mn == 2) {      // tensor memory: staged after the allocation below
        } else if (!a_mn) {   // K-major: k-block k/64, row m
            umma::st_chunk(As + (k8 / 8) * 16384, m, k8 % 8, v);
        } else {              // MN-major: rows = k, mn-block m/64 -- scatter the 8 k values
            const __half *hv = reinterpret_cast<const __half *>(&v);
            for (int e = 0; e < 8; ++e) {
                const int k = k8 * 8 + e;
                uint8_t *blk = As + (m / 64) * (K * 128);
                *reinterpret_cast<__half *>(blk + umma::sw128_offset(k, (m % 64) / 8) + (m % 8) * 2) = hv[e];
            }
        }
    }
    for (int idx = tid; idx < K * N / 8; idx += 128) {
        const int k = idx / (N / 8), n8 = idx % (N / 8);
        const uint4 v = reinterpret_cast<const uint4 *>(B + (size_t)k * N)[n8];
        if (b_mn) {           // MN-major: rows = k, mn-block n/64
            umma::st_chunk(Bs + (n8 / 8) * (K * 128), k, n8 % 8, v);
        } else {              // K-major: rows = n, k-block k/64 -- scatter the 8 n values
            const __half *hv = reinterpret_cast<const __half *>(&v);
            for (int e = 0; e < 8; ++e) {
                const int n = n8 * 8 + e;
                uint8_t *blk = Bs + (k / 64) * (N * 128);
                *reinterpret_cast<__half *>(blk + umma::sw128_offset(n, (k % 64) / 8) + (k % 8) * 2) = hv[e];
            }
        }
    }
    __syncthreads();
    const uint32_t tbase = *tslot;
    const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
    if (a_mn == 2) {          // A rows into lanes, K pairs into columns [128, 128 + K/2)
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 32) {
            float v[32];
            for (int j = 0; j < 32; ++j) {
                const __half2 h2 = *reinterpret_cast<const __half2 *>(A + (size_t)m * K + 2 * (c0 + j));
                v[j] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&h2));
            }
            umma::tmem_st32(trow + 128 + c0, v);
        }
        umma::tmem_st_wait();
    }
    if (init) {
        for (int c = 0; c < N; c += 32) {
            float v[32];
            for (int j = 0; j < 32; ++j) v[j] = init[(size_t)(warp * 32 + lane) * N + c + j];
            umma::tmem_st32(trow + c, v);
        }
        umma::tmem_st_wait();
    }
    umma::fence_proxy_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        umma::tc_fence_after();
        const uint32_t idesc = umma::idesc_f16(128, N, a_mn == 1, b_mn != 0, neg_a != 0);   // A from TMEM: K-major only
        const uint32_t a0 = umma::smem_u32(As), b0 = umma::smem_u32(Bs);
        for (int s = 0; s < K / 16; ++s) {
            uint64_t ad = 0, bd;
            if (a_mn == 0)      ad = umma::sw128_desc(a0 + (s / 4) * 16384 + (s % 4) * 32, 16, 1024);
            else if (a_mn == 1) ad = umma::sw128_desc(a0 + s * 2048, K * 128, 1024);
            if (b_mn)  bd = umma::sw128_desc(b0 + s * 2048, K * 128, 1024);
            else       bd = umma::sw128_desc(b0 + (s / 4) * (N * 128) + (s % 4) * 32, 16, 1024);
            if (a_mn == 2) umma::mma_f16_ts(tbase, tbase + 128 + s * 8, bd, idesc, (s > 0 || init) ? 1u : 0u);
            else           umma::mma_f16(tbase, ad, bd, idesc, (s > 0 || init) ? 1u : 0u);
        }
        umma::mma_commit(bar);
    }
    const bool ok = umma::mbar_wait_bounded(bar, 0, 1u << 22);
    umma::tc_fence_after();
    if (!ok) {
        if (lane == 0) atomicOr(&g_selftest_err, 1u);
    } else {
        for (int c = 0; c < N; c += 32) {
            float v[32];
            umma::tmem_ld32(trow + c, v);
            for (int j = 0; j < 32; ++j) D[(size_t)(warp * 32 + lane) * N + c + j] = v[j];
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tbase, 256);
}

}  // namespace gdn

extern "C" gdn_status_t gdn_selftest_umma(int a_mn, int b_mn, int negate_a, int N, int K,
                                          const void *A, const void *B, const float *init,
                                          float *D, gdn_stream_t stream) {
    if ((N != 64 && N != 128) || (K != 64 && K != 128) || !A || !B || !D) return GDN_ERR_INVALID_ARG;
    if (a_mn < 0 || a_mn > 2 || (a_mn == 2 && negate_a)) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned int zero = 0, err = 0;
    if (cudaMemcpyToSymbolAsync(gdn::g_selftest_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaFuncSetAttribute(gdn::umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gdn::kStSmem) != cudaSuccess)
        return GDN_ERR_CUDA;
    gdn::umma_selftest_kernel<<<1, 128, gdn::kStSmem, s>>>(a_mn, b_mn, negate_a, N, K,
                                                           static_cast<const __half *>(A),
                                                           static_cast<const __half *>(B), init, D);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&err, gdn::g_selftest_err, sizeof err, 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    return err ? GDN_ERR_TIMEOUT : GDN_OK;
}

extern "C" gdn_status_t gdn_selftest_wait_timeout(unsigned family, unsigned max_polls,
                                                  gdn_stream_t stream) {
    if (max_polls < 1 || max_polls > 65536) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (family) {
    case GDN_ERRF_PREP: e = gdn::prep_wait_selftest(max_polls, s); break;
    case GDN_ERRF_CHAIN: e = gdn::chain_wait_selftest(max_polls, s); break;
    case GDN_ERRF_DECODE: e = gdn::decode_wait_selftest(max_polls, s); break;
    case GDN_ERRF_QSA: e = gdn::qsa_wait_selftest(max_polls, s); break;
    case GDN_ERRF_GEMM: e = gdn::gemm_wait_selftest(max_polls, s); break;
    default: return GDN_ERR_INVALID_ARG;
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

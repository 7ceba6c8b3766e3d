// K2b -- the state-dependent part of the chunked gated delta rule, sequential
// over the chunks of one (sequence, head), with the output gate and the
// zero-centred RMSNorm fused (slinene.github.io write-up of "On the Design of
// Qwen3.8-Next Architecture", 模块 A: 递归状态 and 参数化).
//
// Per chunk, with the per-chunk tensors of the chunk-prep kernel
// (-W, U', Qt, Kt, Aqk, e^{G_C}) and the state S before the chunk:
//     P[0:64]   = U' + (-W) S        = U            (tcgen05, M=128 with rows 64..127)
//     P[64:128] = Qt S                               (... = diag(e^G) Q S)
//     P[64:128] += Aqk U             = Y            (tcgen05)
//     dS        = Kt^T U                              (tcgen05)
//     S         = e^{G_C} S + dS                      (fp32, registers)
//     out       = sigmoid(z) * Y / sqrt(mean(Y^2) + eps) * (1 + w)
// One CTA of 128 threads: thread r holds row r of the fp32 state S [dk=128][dv]
// (TMEM lane r of dS), and an fp16 copy of S in shared memory is the B operand
// of the next chunk.  All accumulators live in tensor memory.
#include <cuda_fp16.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

__device__ unsigned int g_chain_err;

namespace chain {
constexpr int C = 64;
constexpr int DK = 128;
constexpr int OFF_AP = 0;                // [-W; Qt] K-major: 2 k-blocks x 16 KB
constexpr int OFF_BP = 32768;            // S MN-major: rows = dk, DV/64 mn-blocks x 16 KB
constexpr int OFF_AS = 65536;            // Kt MN-major: rows = tokens, 2 mn-blocks x 8 KB
constexpr int OFF_AY = 81920;            // [0; Aqk] K-major: 1 k-block x 16 KB
constexpr int OFF_BU = 98304;            // U MN-major: rows = tokens, DV/64 mn-blocks x 8 KB
constexpr int OFF_MISC = 114688;
constexpr int SMEM = OFF_MISC + 1024 + 1024;
}  // namespace chain

__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(umma::pack_half2(x[0], x[1]), umma::pack_half2(x[2], x[3]),
                      umma::pack_half2(x[4], x[5]), umma::pack_half2(x[6], x[7]));
}

__device__ __forceinline__ void unpack8(uint4 u, float *x) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

template <typename T> __device__ __forceinline__ void load8_any(const T *p, float (&x)[8]) { load8(p, x); }

template <typename Tout> __device__ __forceinline__ void store8_out(Tout *p, const float (&x)[8]);
template <> __device__ __forceinline__ void store8_out<float>(float *p, const float (&x)[8]) {
    store8(p, x);
}
template <> __device__ __forceinline__ void store8_out<bf16>(bf16 *p, const float (&x)[8]) {
    uint4 u;
    uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t *>(&b);
    }
    *reinterpret_cast<uint4 *>(p) = u;
}

template <int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(128, 1)
chunk_chain_kernel(const __half *__restrict__ Qt, const __half *__restrict__ Kt,
                   const __half *__restrict__ Wn, const __half *__restrict__ Up,
                   const __half *__restrict__ Aqk, const float *__restrict__ decay,
                   const Tin *__restrict__ z, const float *__restrict__ norm_w,
                   const float *__restrict__ S0, const int32_t *__restrict__ cu_seqlens,
                   int n_seq, int n_tok, int H, Tout *__restrict__ out,
                   float *__restrict__ S_final) {
    using namespace chain;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sAP = sm + OFF_AP, *sBP = sm + OFF_BP, *sAS = sm + OFF_AS, *sAY = sm + OFF_AY,
            *sBU = sm + OFF_BU;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 16);
    constexpr uint32_t TMEM_COLS = 2 * DV;   // P [0, DV), dS [DV, 2 DV)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, n = blockIdx.y;
    int s_begin, s_end;
    if (cu_seqlens) { s_begin = __ldg(cu_seqlens + n); s_end = __ldg(cu_seqlens + n + 1); }
    else { const int L = n_tok / n_seq; s_begin = n * L; s_end = s_begin + L; }
    const int n_chunks = (s_end - s_begin + C - 1) / C;

    if (warp == 0) umma::tmem_alloc(tslot, TMEM_COLS);
    if (tid == 0) { umma::mbar_init(bar, 1); umma::fence_mbar_init(); }
    // rows 0..63 of the A operand of Aqk U stay zero
    for (int idx = tid; idx < 64 * 8; idx += 128)
        umma::st_chunk(sAY, idx / 8, idx % 8, make_uint4(0, 0, 0, 0));

    // fp32 master state: thread r owns row r of S; fp16 copy into sBP (rows = dk)
    const size_t sbase = ((size_t)n * H + h) * DK * DV;
    float S[DV];
    {
        const int r = tid;
#pragma unroll
        for (int c8 = 0; c8 < DV / 8; ++c8) {
            float x[8];
            if (S0) load8(S0 + sbase + (size_t)r * DV + c8 * 8, x);
            else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) S[c8 * 8 + e] = x[e];
            umma::st_chunk(sBP + (c8 / 8) * 16384, r, c8 % 8, pack8(x));
        }
    }
    __syncthreads();
    const uint32_t tbase = *tslot;
    const uint32_t tP = tbase, tS = tbase + DV;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t phase = 0;
    bool ok = true;

    for (int c = 0; c < n_chunks && ok; ++c) {
        const int t0 = s_begin + c * C;
        const int len = min(C, s_end - t0);
        const float dec = __ldg(decay + (size_t)t0 * H + h);
        // ---- 1. stage -W, Qt (A of P), Kt (A of dS), Aqk (A of Y); U' / 0 into TMEM P
        for (int idx = tid; idx < C * (DK / 8); idx += 128) {
            const int i = idx / (DK / 8), ch = idx % (DK / 8);
            uint4 w = make_uint4(0, 0, 0, 0), q = w, k = w;
            if (i < len) {
                const size_t g = ((size_t)(t0 + i) * H + h) * DK + ch * 8;
                w = *reinterpret_cast<const uint4 *>(Wn + g);
                q = *reinterpret_cast<const uint4 *>(Qt + g);
                k = *reinterpret_cast<const uint4 *>(Kt + g);
            }
            umma::st_chunk(sAP + (ch / 8) * 16384, i, ch % 8, w);
            umma::st_chunk(sAP + (ch / 8) * 16384, 64 + i, ch % 8, q);
            umma::st_chunk(sAS + (ch / 8) * 8192, i, ch % 8, k);
        }
        for (int idx = tid; idx < C * 8; idx += 128) {
            const int i = idx / 8, ch = idx % 8;
            uint4 a = make_uint4(0, 0, 0, 0);
            if (i < len) a = *reinterpret_cast<const uint4 *>(Aqk + ((size_t)(t0 + i) * H + h) * C + ch * 8);
            umma::st_chunk(sAY, 64 + i, ch, a);
        }
        {
            const int i = (warp * 32 + lane) & 63;
            const bool has = warp < 2 && i < len;
            const __half *src = Up + ((size_t)(t0 + i) * H + h) * DV;
#pragma unroll
            for (int c0 = 0; c0 < DV; c0 += 32) {
                float v[32];
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    if (has) unpack8(*reinterpret_cast<const uint4 *>(src + c0 + q8 * 8), v + q8 * 8);
                    else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[q8 * 8 + e] = 0.f;
                    }
                }
                umma::tmem_st32(tP + lane_off + c0, v);
            }
            umma::tmem_st_wait();
        }
        umma::fence_proxy_async_smem();
        umma::tc_fence_before();
        __syncthreads();

        // ---- 2. P += [-W; Qt] S    (M=128, N=DV, K=dk)
        if (tid == 0) {
            umma::tc_fence_after();
            const uint32_t a0 = umma::smem_u32(sAP), b0 = umma::smem_u32(sBP);
            const uint32_t idesc = umma::idesc_f16(128, DV, false, true);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                umma::mma_f16(tP, umma::sw128_desc(a0 + (s / 4) * 16384 + (s % 4) * 32, 16, 1024),
                              umma::sw128_desc(b0 + s * 2048, 16384, 1024), idesc, 1u);
            umma::mma_commit(bar);
        }
        ok = __syncthreads_and(umma::mbar_wait_bounded(bar, phase, 1u << 22));
        phase ^= 1;
        umma::tc_fence_after();
        if (!ok) break;

        // ---- 3. U = P[0:64] -> fp16 MN-major (rows = tokens) as the B operand
        if (warp < 2) {
            const int i = warp * 32 + lane;
#pragma unroll
            for (int c0 = 0; c0 < DV; c0 += 32) {
                float v[32];
                umma::tmem_ld32(tP + lane_off + c0, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const int col = c0 + q8 * 8;
                    umma::st_chunk(sBU + (col / 64) * 8192, i, (col % 64) / 8, pack8(v + q8 * 8));
                }
            }
        }
        umma::fence_proxy_async_smem();
        umma::tc_fence_before();
        __syncthreads();

        // ---- 4. P += [0; Aqk] U  (Y in rows 64..127);  dS = Kt^T U
        if (tid == 0) {
            umma::tc_fence_after();
            const uint32_t aY = umma::smem_u32(sAY), aS = umma::smem_u32(sAS), bU = umma::smem_u32(sBU);
            const uint32_t idy = umma::idesc_f16(128, DV, false, true);
            const uint32_t ids = umma::idesc_f16(128, DV, true, true);
#pragma unroll
            for (int s = 0; s < C / 16; ++s) {
                const uint64_t bd = umma::sw128_desc(bU + s * 2048, 8192, 1024);
                umma::mma_f16(tP, umma::sw128_desc(aY + s * 32, 16, 1024), bd, idy, 1u);
                umma::mma_f16(tS, umma::sw128_desc(aS + s * 2048, 8192, 1024), bd, ids, s > 0);
            }
            umma::mma_commit(bar);
        }
        ok = __syncthreads_and(umma::mbar_wait_bounded(bar, phase, 1u << 22));
        phase ^= 1;
        umma::tc_fence_after();
        if (!ok) break;

        // ---- 5a. S = e^{G_C} S + dS; fp16 copy for the next chunk
        {
            const int r = tid;
#pragma unroll
            for (int c0 = 0; c0 < DV; c0 += 32) {
                float v[32];
                umma::tmem_ld32(tS + lane_off + c0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[c0 + j] = fmaf(dec, S[c0 + j], v[j]);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const int col = c0 + q8 * 8;
                    umma::st_chunk(sBP + (col / 64) * 16384, r, (col % 64) / 8, pack8(S + col));
                }
            }
        }
        // ---- 5b. output stage on Y = P[64:128] (warps 2, 3): two passes over TMEM
        if (warp >= 2) {
            const int i = (warp - 2) * 32 + lane;
            float ss = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < DV; c0 += 32) {
                float v[32];
                umma::tmem_ld32(tP + lane_off + c0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
            }
            const float rr = 1.0f / sqrtf(ss / DV + kNormEps);
            const size_t g = ((size_t)(t0 + i) * H + h) * DV;
#pragma unroll
            for (int c0 = 0; c0 < DV; c0 += 32) {
                float v[32];
                umma::tmem_ld32(tP + lane_off + c0, v);
                if (i < len) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        const int col = c0 + q8 * 8;
                        float zz[8], o[8];
                        load8(z + g + col, zz);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float w1 = 1.0f + __ldg(norm_w + col + e);
                            o[e] = sigmoid_acc(zz[e]) * v[q8 * 8 + e] * rr * w1;
                        }
                        store8_out<Tout>(out + g + col, o);
                    }
                }
            }
        }
        umma::fence_proxy_async_smem();
        umma::tc_fence_before();
        __syncthreads();
    }
    if (!ok && tid == 0) atomicOr(&g_chain_err, 1u);
    if (ok && S_final) {
        const int r = tid;
#pragma unroll
        for (int c8 = 0; c8 < DV / 8; ++c8) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = S[c8 * 8 + e];
            store8(S_final + sbase + (size_t)r * DV + c8 * 8, x);
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tbase, TMEM_COLS);
}

cudaError_t launch_chunk_chain(const PrefillArgs &a, const TcWorkspace &w) {
    dim3 grid(a.H, a.n_seq);
    cudaError_t e;
#define GDN_CHAIN(DV_, TIN, TOUT)                                                                 \
    e = cudaFuncSetAttribute(chunk_chain_kernel<DV_, TIN, TOUT>,                                  \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, chain::SMEM);            \
    if (e != cudaSuccess) return e;                                                               \
    chunk_chain_kernel<DV_, TIN, TOUT><<<grid, 128, chain::SMEM, a.stream>>>(                     \
        w.Qt, w.Kt, w.Wn, w.Up, w.Aqk, w.decay, (const TIN *)a.z, a.norm_w, a.S0, a.cu_seqlens, \
        a.n_seq, a.n_tok, a.H, (TOUT *)a.out, a.S_final)
    if (a.dv == 128) {
        if (a.in_bf16) { if (a.out_bf16) { GDN_CHAIN(128, bf16, bf16); } else { GDN_CHAIN(128, bf16, float); } }
        else { if (a.out_bf16) { GDN_CHAIN(128, float, bf16); } else { GDN_CHAIN(128, float, float); } }
    } else {
        if (a.in_bf16) { if (a.out_bf16) { GDN_CHAIN(64, bf16, bf16); } else { GDN_CHAIN(64, bf16, float); } }
        else { if (a.out_bf16) { GDN_CHAIN(64, float, bf16); } else { GDN_CHAIN(64, float, float); } }
    }
#undef GDN_CHAIN
    return cudaGetLastError();
}

}  // namespace gdn

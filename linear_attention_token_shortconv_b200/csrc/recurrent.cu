// K2f -- the gated delta rule token by token in fp32 (SIMT), with the gates and
// the output stage fused (slinene.github.io write-up of "On the Design of
// Qwen3.8-Next Architecture", 模块 A: 递归状态 and 参数化).
//
// One CTA per (sequence, head); thread j owns column j of the state S [dk][dv]
// in dk registers, so S^T k, the rank-1 write and S^T q are thread-local and need
// no reduction.  Tokens are staged through shared memory in blocks of 16; the
// output RMSNorm of a block is done after its 16 recurrence steps.  This is the
// path of the fp32 workload, where tensor-core operand rounding would exceed the
// 1e-5 bound.
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kRecBlock = 16;  // tokens staged per block

template <int DK, int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(DV)
recurrent_kernel(const float *__restrict__ qn, const float *__restrict__ kn,
                 const float *__restrict__ vn, const Tin *__restrict__ a_logit,
                 const Tin *__restrict__ b_logit, const float *__restrict__ A,
                 const float *__restrict__ b_alpha, const Tin *__restrict__ z,
                 const float *__restrict__ norm_w, const float *__restrict__ S0,
                 const int32_t *__restrict__ cu_seqlens, int n_seq, int n_tok, int H,
                 Tout *__restrict__ out, float *__restrict__ S_final) {
    __shared__ __align__(16) float qs[kRecBlock][DK];
    __shared__ __align__(16) float ks[kRecBlock][DK];
    __shared__ __align__(16) float vs[kRecBlock][DV];
    __shared__ __align__(16) float ys[kRecBlock][DV];
    __shared__ float alpha_s[kRecBlock], beta_s[kRecBlock];

    const int h = blockIdx.x, n = blockIdx.y, j = threadIdx.x;
    const int lane = j & 31, warp = j >> 5;
    constexpr int NW = DV / 32;
    int t_begin, t_end;
    if (cu_seqlens) {
        t_begin = __ldg(cu_seqlens + n);
        t_end = __ldg(cu_seqlens + n + 1);
    } else {
        const int L = n_tok / n_seq;
        t_begin = n * L;
        t_end = t_begin + L;
    }
    const size_t sbase = ((size_t)n * H + h) * DK * DV;
    float S[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i) S[i] = S0 ? __ldg(S0 + sbase + (size_t)i * DV + j) : 0.f;
    const float eA = expf(__ldg(A + h)), ba = __ldg(b_alpha + h);

    for (int tb = t_begin; tb < t_end; tb += kRecBlock) {
        const int nb = min(kRecBlock, t_end - tb);
        // stage q, k (dk each) and v (dv) of nb tokens of head h
        for (int idx = j; idx < nb * DK / 4; idx += DV) {
            const int tt = idx / (DK / 4), c4 = idx % (DK / 4);
            const size_t g = ((size_t)(tb + tt) * H + h) * DK / 4 + c4;
            reinterpret_cast<float4 *>(qs[tt])[c4] = __ldg(reinterpret_cast<const float4 *>(qn) + g);
            reinterpret_cast<float4 *>(ks[tt])[c4] = __ldg(reinterpret_cast<const float4 *>(kn) + g);
        }
        for (int idx = j; idx < nb * DV / 4; idx += DV) {
            const int tt = idx / (DV / 4), c4 = idx % (DV / 4);
            const size_t g = ((size_t)(tb + tt) * H + h) * DV / 4 + c4;
            reinterpret_cast<float4 *>(vs[tt])[c4] = __ldg(reinterpret_cast<const float4 *>(vn) + g);
        }
        if (j < nb) {
            const size_t g = (size_t)(tb + j) * H + h;
            const float la = -eA * softplus_acc(to_f32(a_logit[g]) + ba);
            alpha_s[j] = expf(la);
            beta_s[j] = sigmoid_acc(to_f32(b_logit[g]));
        }
        __syncthreads();
        for (int tt = 0; tt < nb; ++tt) {
            const float al = alpha_s[tt], be = beta_s[tt];
            float sk = 0.f;
#pragma unroll
            for (int i = 0; i < DK; i += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&ks[tt][i]);
                sk = fmaf(S[i], kk.x, sk); sk = fmaf(S[i + 1], kk.y, sk);
                sk = fmaf(S[i + 2], kk.z, sk); sk = fmaf(S[i + 3], kk.w, sk);
            }
            // e = v - (alpha S)^T k ; S = alpha S + beta k e^T ; y = S^T q
            const float bee = be * (vs[tt][j] - al * sk);
            float y = 0.f;
#pragma unroll
            for (int i = 0; i < DK; i += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&ks[tt][i]);
                const float4 qq = *reinterpret_cast<const float4 *>(&qs[tt][i]);
                S[i] = fmaf(kk.x, bee, al * S[i]);         y = fmaf(S[i], qq.x, y);
                S[i + 1] = fmaf(kk.y, bee, al * S[i + 1]); y = fmaf(S[i + 1], qq.y, y);
                S[i + 2] = fmaf(kk.z, bee, al * S[i + 2]); y = fmaf(S[i + 2], qq.z, y);
                S[i + 3] = fmaf(kk.w, bee, al * S[i + 3]); y = fmaf(S[i + 3], qq.w, y);
            }
            ys[tt][j] = y;
        }
        __syncthreads();
        // output stage: warp w normalises tokens w, w + NW, ...
        for (int tt = warp; tt < nb; tt += NW) {
            float yv[DV / 32];
            float ss = 0.f;
#pragma unroll
            for (int m = 0; m < DV / 32; ++m) {
                yv[m] = ys[tt][lane + 32 * m];
                ss = fmaf(yv[m], yv[m], ss);
            }
            ss = group_sum<32>(ss);
            const float r = 1.0f / sqrtf(ss / DV + kNormEps);
            const size_t g = ((size_t)(tb + tt) * H + h) * DV;
#pragma unroll
            for (int m = 0; m < DV / 32; ++m) {
                const int col = lane + 32 * m;
                const float gate = sigmoid_acc(to_f32(z[g + col]));
                const float wc = 1.0f + __ldg(norm_w + col);
                out[g + col] = from_f32<Tout>(gate * yv[m] * r * wc);
            }
        }
        __syncthreads();
    }
    if (S_final) {
#pragma unroll
        for (int i = 0; i < DK; ++i) S_final[sbase + (size_t)i * DV + j] = S[i];
    }
}

template <int DK, int DV>
static cudaError_t launch_rec_dims(const PrefillArgs &a, const float *qn, const float *kn,
                                   const float *vn) {
    dim3 grid(a.H, a.n_seq);
#define GDN_REC(TIN, TOUT)                                                                      \
    recurrent_kernel<DK, DV, TIN, TOUT><<<grid, DV, 0, a.stream>>>(                            \
        qn, kn, vn, (const TIN *)a.a_logit, (const TIN *)a.b_logit, a.A, a.b_alpha,           \
        (const TIN *)a.z, a.norm_w, a.S0, a.cu_seqlens, a.n_seq, a.n_tok, a.H, (TOUT *)a.out,  \
        a.S_final)
    if (a.in_bf16) {
        if (a.out_bf16) GDN_REC(bf16, bf16); else GDN_REC(bf16, float);
    } else {
        if (a.out_bf16) GDN_REC(float, bf16); else GDN_REC(float, float);
    }
#undef GDN_REC
    return launched();
}

cudaError_t launch_recurrent(const PrefillArgs &a, const float *qn, const float *kn,
                             const float *vn) {
    if (a.dk == 128 && a.dv == 128) return launch_rec_dims<128, 128>(a, qn, kn, vn);
    if (a.dk == 64 && a.dv == 64) return launch_rec_dims<64, 64>(a, qn, kn, vn);
    if (a.dk == 128 && a.dv == 64) return launch_rec_dims<128, 64>(a, qn, kn, vn);
    return launch_rec_dims<64, 128>(a, qn, kn, vn);
}

}  // namespace gdn

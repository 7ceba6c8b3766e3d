// K3 -- one decode step of the GDN mixer: ShortConv over the raw history plus the
// current token, SiLU, L2Norm, the gates, the gated delta rule on the fp32 state
// (read once, written once, in place) and the gated RMSNorm output
// (slinene.github.io write-up of "On the Design of Qwen3.8-Next Architecture",
// 模块 A; the digest's remark that decode time is set by the bytes moved).
//
// One CTA of 256 threads per (sequence, head).  The CTA first issues all loads of
// its 64 KB state slice (16 x 128-bit per thread, a warp reads one 512-byte row
// per load), computes the prelude while they are in flight, then forms
// s_k = S^T k and s_q = S^T q with a block reduction, and writes
//   S' = alpha S + beta k e^T,  e = v - alpha s_k,
//   y  = S'^T q = alpha s_q + beta (k.q) e
// so the state is streamed through registers exactly once.
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kDecThreads = 256;

template <int DK, int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ conv_w, Tin *__restrict__ hist,
              const Tin *__restrict__ a_logit, const Tin *__restrict__ b_logit,
              const float *__restrict__ A, const float *__restrict__ b_alpha,
              const Tin *__restrict__ z, const float *__restrict__ norm_w, float *__restrict__ S,
              Tout *__restrict__ out, int H) {
    constexpr int NCH = 2 * DK + DV;           // channels of this head
    constexpr int F4_PER_ROW = DV / 4;          // float4 per state row
    constexpr int NV = DK * DV / 4 / kDecThreads;  // float4 per thread
    constexpr int ROWS_PER_PASS = kDecThreads / F4_PER_ROW;
    constexpr int NW = kDecThreads / 32;

    __shared__ __align__(16) float xs[NCH];     // conv+SiLU outputs: q | k | v
    __shared__ float red_k[ROWS_PER_PASS][DV], red_q[ROWS_PER_PASS][DV];
    __shared__ float e_s[DV], y_s[DV];
    __shared__ float scal[4];                   // 1/|q|, 1/|k|, alpha, beta

    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const size_t gi = (size_t)b * H + h;
    float4 *Sh = reinterpret_cast<float4 *>(S + gi * DK * DV);

    // 1. issue the state loads first
    float4 s[NV];
#pragma unroll
    for (int r = 0; r < NV; ++r) s[r] = __ldcs(Sh + tid + r * kDecThreads);

    // 2. prelude of this head: conv over [hist (3 taps), current], SiLU; shift history
    const size_t C = (size_t)H * NCH;
    for (int ch = tid; ch < NCH; ch += kDecThreads) {
        size_t c, src_i;
        const Tin *src;
        if (ch < DK) { c = (size_t)h * DK + ch; src = q; src_i = gi * DK + ch; }
        else if (ch < 2 * DK) { c = (size_t)H * DK + h * DK + (ch - DK); src = k; src_i = gi * DK + (ch - DK); }
        else { c = (size_t)2 * H * DK + h * DV + (ch - 2 * DK); src = v; src_i = gi * DV + (ch - 2 * DK); }
        const float4 w = __ldg(reinterpret_cast<const float4 *>(conv_w) + c);
        Tin *hb = hist + (size_t)b * 3 * C + c;
        const Tin x0 = hb[0], x1 = hb[C], x2 = hb[2 * C], xc = src[src_i];
        float acc = w.x * to_f32(x0);
        acc = fmaf(w.y, to_f32(x1), acc);
        acc = fmaf(w.z, to_f32(x2), acc);
        acc = fmaf(w.w, to_f32(xc), acc);
        xs[ch] = siluf_(acc);
        hb[0] = x1; hb[C] = x2; hb[2 * C] = xc;
    }
    __syncthreads();
    if (warp < 2) {  // warp 0: |q|^2, warp 1: |k|^2
        float ss = 0.f;
        for (int i = lane; i < DK; i += 32) { const float x = xs[warp * DK + i]; ss = fmaf(x, x, ss); }
        ss = group_sum<32>(ss);
        if (lane == 0) scal[warp] = rsqrtf(ss + kNormEps);
    } else if (warp == 2 && lane == 0) {
        const float la = log_decay(to_f32(a_logit[gi]), __ldg(A + h), __ldg(b_alpha + h));
        scal[2] = expf(la);
        scal[3] = sigmoid_acc(to_f32(b_logit[gi]));
    }
    __syncthreads();
    const float rq = scal[0], rk = scal[1], alpha = scal[2], beta = scal[3];

    // 3. partial S^T k and S^T q over this thread's rows (raw SiLU values; scaled later)
    const int cg = tid % F4_PER_ROW, row0 = tid / F4_PER_ROW;
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < NV; ++r) {
        const int i = row0 + r * ROWS_PER_PASS;
        const float kk = xs[DK + i], qq = xs[i];
        pk[0] = fmaf(s[r].x, kk, pk[0]); pk[1] = fmaf(s[r].y, kk, pk[1]);
        pk[2] = fmaf(s[r].z, kk, pk[2]); pk[3] = fmaf(s[r].w, kk, pk[3]);
        pq[0] = fmaf(s[r].x, qq, pq[0]); pq[1] = fmaf(s[r].y, qq, pq[1]);
        pq[2] = fmaf(s[r].z, qq, pq[2]); pq[3] = fmaf(s[r].w, qq, pq[3]);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        red_k[row0][cg * 4 + m] = pk[m];
        red_q[row0][cg * 4 + m] = pq[m];
    }
    __syncthreads();
    // 4. finish the reductions; e and y per column
    if (tid < DV) {
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int p = 0; p < ROWS_PER_PASS; ++p) { sk += red_k[p][tid]; sq += red_q[p][tid]; }
        sk *= rk;
        sq *= rq;
        float kq = 0.f;  // k.q of the normalised vectors
        for (int i = 0; i < DK; ++i) kq = fmaf(xs[DK + i], xs[i], kq);
        kq *= rk * rq;
        const float e = xs[2 * DK + tid] - alpha * sk;
        e_s[tid] = e;
        y_s[tid] = fmaf(beta * kq, e, alpha * sq);
    }
    __syncthreads();
    // 5. S' = alpha S + beta k e^T, written back in place
    {
        const float4 e4 = make_float4(e_s[cg * 4], e_s[cg * 4 + 1], e_s[cg * 4 + 2], e_s[cg * 4 + 3]);
#pragma unroll
        for (int r = 0; r < NV; ++r) {
            const int i = row0 + r * ROWS_PER_PASS;
            const float bk = beta * rk * xs[DK + i];
            float4 o;
            o.x = fmaf(bk, e4.x, alpha * s[r].x);
            o.y = fmaf(bk, e4.y, alpha * s[r].y);
            o.z = fmaf(bk, e4.z, alpha * s[r].z);
            o.w = fmaf(bk, e4.w, alpha * s[r].w);
            __stcs(Sh + tid + r * kDecThreads, o);
        }
    }
    // 6. output stage on warp NW-1 (its state stores are already issued)
    if (warp == NW - 1) {
        float yv[DV / 32], ss = 0.f;
#pragma unroll
        for (int m = 0; m < DV / 32; ++m) { yv[m] = y_s[lane + 32 * m]; ss = fmaf(yv[m], yv[m], ss); }
        ss = group_sum<32>(ss);
        const float r = 1.0f / sqrtf(ss / DV + kNormEps);
#pragma unroll
        for (int m = 0; m < DV / 32; ++m) {
            const int col = lane + 32 * m;
            const float gate = sigmoid_acc(to_f32(z[gi * DV + col]));
            out[gi * DV + col] = from_f32<Tout>(gate * yv[m] * r * (1.0f + __ldg(norm_w + col)));
        }
    }
}

template <int DK, int DV>
static cudaError_t launch_dec_dims(const DecodeArgs &a) {
    dim3 grid(a.H, a.B);
#define GDN_DEC(TIN, TOUT)                                                                    \
    decode_kernel<DK, DV, TIN, TOUT><<<grid, kDecThreads, 0, a.stream>>>(                    \
        (const TIN *)a.q, (const TIN *)a.k, (const TIN *)a.v, a.conv_w, (TIN *)a.conv_hist,  \
        (const TIN *)a.a_logit, (const TIN *)a.b_logit, a.A, a.b_alpha, (const TIN *)a.z,    \
        a.norm_w, a.S, (TOUT *)a.out, a.H)
    if (a.in_bf16) {
        if (a.out_bf16) GDN_DEC(bf16, bf16); else GDN_DEC(bf16, float);
    } else {
        if (a.out_bf16) GDN_DEC(float, bf16); else GDN_DEC(float, float);
    }
#undef GDN_DEC
    return launched();
}

cudaError_t launch_decode(const DecodeArgs &a) {
    if (a.dk == 128 && a.dv == 128) return launch_dec_dims<128, 128>(a);
    if (a.dk == 64 && a.dv == 64) return launch_dec_dims<64, 64>(a);
    if (a.dk == 128 && a.dv == 64) return launch_dec_dims<128, 64>(a);
    return launch_dec_dims<64, 128>(a);
}

}  // namespace gdn

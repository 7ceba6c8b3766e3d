// K1 -- the elementwise prelude of the GDN mixer for a packed prefill batch:
// ShortConv (causal depthwise, width 4) -> SiLU on q, k, v, then L2Norm on q and k
// (slinene.github.io write-up of "On the Design of Qwen3.8-Next Architecture",
// 模块 A, 参数化; the digest's Figure 2 caption).
//
// One thread owns 8 consecutive channels and walks a tile of tokens, keeping the
// last three raw rows of its channels in registers, so every raw element is read
// from HBM once (plus a 3-row halo per tile).  Loads and stores are 128-bit.  The
// L2Norm sum over a head's dk channels is a shuffle reduction inside the dk/8
// lanes that hold the head.  Output goes to a workspace in fp32 or fp16.
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kPreludeThreads = 256;
constexpr int kPreludeTile = 16;  // tokens per thread

template <typename Tin, typename Tws, int DK, int DV>
__global__ void __launch_bounds__(kPreludeThreads)
prelude_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
               const float *__restrict__ conv_w, const int32_t *__restrict__ cu_seqlens,
               int n_seq, int n_tok, int H, Tws *__restrict__ qn, Tws *__restrict__ kn,
               Tws *__restrict__ vn) {
    const int octets = H * (2 * DK + DV) / 8;
    const int co = blockIdx.x * kPreludeThreads + threadIdx.x;
    const bool active = co < octets;
    const int c = active ? co * 8 : 0;  // first conv channel of this thread
    // which tensor, and the column of the first channel inside a token row
    const Tin *src;
    Tws *dst;
    int row, col, kind;  // kind 0 = q, 1 = k, 2 = v
    if (c < H * DK) {
        src = q; dst = qn; row = H * DK; col = c; kind = 0;
    } else if (c < 2 * H * DK) {
        src = k; dst = kn; row = H * DK; col = c - H * DK; kind = 1;
    } else {
        src = v; dst = vn; row = H * DV; col = c - 2 * H * DK; kind = 2;
    }
    float w[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float4 t4 = active ? __ldg(reinterpret_cast<const float4 *>(conv_w) + (c + i))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        w[i][0] = t4.x; w[i][1] = t4.y; w[i][2] = t4.z; w[i][3] = t4.w;
    }
    const int t0 = blockIdx.y * kPreludeTile;
    const int t1 = min(t0 + kPreludeTile, n_tok);
    // sequence of the first token and where it starts / ends
    const int L = cu_seqlens ? 0 : n_tok / n_seq;
    int n = cu_seqlens ? seq_of_token(cu_seqlens, n_seq, t0) : t0 / L;
    int s_start = cu_seqlens ? __ldg(cu_seqlens + n) : n * L;
    int s_end = cu_seqlens ? __ldg(cu_seqlens + n + 1) : (n + 1) * L;
    // raw history rows t-3, t-2, t-1 (zero before the sequence start)
    float h0[8], h1[8], h2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h0[i] = h1[i] = h2[i] = 0.f;
    if (active) {
        if (t0 - 3 >= s_start) load8(src + (size_t)(t0 - 3) * row + col, h0);
        if (t0 - 2 >= s_start) load8(src + (size_t)(t0 - 2) * row + col, h1);
        if (t0 - 1 >= s_start) load8(src + (size_t)(t0 - 1) * row + col, h2);
    }
    for (int t = t0; t < t1; ++t) {
        while (t >= s_end) {  // entered the next (possibly after empty) sequence
            ++n;
            s_start = s_end;
            s_end = cu_seqlens ? __ldg(cu_seqlens + n + 1) : (n + 1) * L;
#pragma unroll
            for (int i = 0; i < 8; ++i) h0[i] = h1[i] = h2[i] = 0.f;
        }
        float x[8], y[8];
        if (active) load8(src + (size_t)t * row + col, x);
        else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float a = w[i][0] * h0[i];
            a = fmaf(w[i][1], h1[i], a);
            a = fmaf(w[i][2], h2[i], a);
            a = fmaf(w[i][3], x[i], a);
            y[i] = siluf_(a);
            ss = fmaf(y[i], y[i], ss);
            h0[i] = h1[i]; h1[i] = h2[i]; h2[i] = x[i];
        }
        // all lanes take part in the shuffle; only q/k lanes use the result
        ss = group_sum<DK / 8>(ss);
        if (kind < 2) {
            const float r = rsqrtf(ss + kNormEps);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] *= r;
        }
        if (active) store8(dst + (size_t)t * row + col, y);
    }
}

template <typename Tin, typename Tws>
cudaError_t launch_prelude_t(const PrefillArgs &a, Tws *qn, Tws *kn, Tws *vn) {
    const int octets = a.H * (2 * a.dk + a.dv) / 8;
    dim3 grid((octets + kPreludeThreads - 1) / kPreludeThreads,
              (a.n_tok + kPreludeTile - 1) / kPreludeTile);
    if (a.n_tok == 0) return cudaSuccess;
#define GDN_PRELUDE(DK_, DV_)                                                                  \
    prelude_kernel<Tin, Tws, DK_, DV_><<<grid, kPreludeThreads, 0, a.stream>>>(              \
        (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v, a.conv_w, a.cu_seqlens, a.n_seq, \
        a.n_tok, a.H, qn, kn, vn)
    if (a.dk == 128 && a.dv == 128) GDN_PRELUDE(128, 128);
    else if (a.dk == 64 && a.dv == 64) GDN_PRELUDE(64, 64);
    else if (a.dk == 128 && a.dv == 64) GDN_PRELUDE(128, 64);
    else GDN_PRELUDE(64, 128);
#undef GDN_PRELUDE
    return launched();
}

cudaError_t launch_prelude_f32(const PrefillArgs &a, float *qn, float *kn, float *vn) {
    return a.in_bf16 ? launch_prelude_t<bf16, float>(a, qn, kn, vn)
                     : launch_prelude_t<float, float>(a, qn, kn, vn);
}

cudaError_t launch_prelude_f16(const PrefillArgs &a, __half *qn, __half *kn, __half *vn) {
    return a.in_bf16 ? launch_prelude_t<bf16, __half>(a, qn, kn, vn)
                     : launch_prelude_t<float, __half>(a, qn, kn, vn);
}

}  // namespace gdn

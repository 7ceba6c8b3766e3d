// Device-side helpers shared by the GDN kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {

// eps inside the square root of both L2Norm (q, k) and the output RMSNorm.
constexpr float kNormEps = 1e-6f;

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Load 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32) as floats.
__device__ __forceinline__ void load8(const bf16 *p, float (&x)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
    x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store8(float *p, const float (&x)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8(__half *p, const float (&x)[8]) {
    __half2 h0 = __floats2half2_rn(x[0], x[1]), h1 = __floats2half2_rn(x[2], x[3]);
    __half2 h2 = __floats2half2_rn(x[4], x[5]), h3 = __floats2half2_rn(x[6], x[7]);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t *>(&h0); u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2); u.w = *reinterpret_cast<uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return x / (1.0f + __expf(-x)); }

// Accurate variants for the gates, where the fp32 path must stay within 1e-5.
__device__ __forceinline__ float sigmoid_acc(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float softplus_acc(float x) {
    return x > 0.0f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}
// Lower bound of the log-decay on the chunked (tensor-core) path.  That path
// forms e^{G_i - G_j} from in-chunk cumulative sums of log alpha, so a log-decay
// that overflows to -inf (a decay logit near the top of the bf16 range) would
// give -inf - (-inf) = NaN.  Every log-decay at or below -104 already makes
// e^g, and every product that contains it, exactly 0 in fp32, so clamping at
// -128 changes no result and keeps the sums finite.  A NaN logit stays NaN.
constexpr float kLogDecayFloor = -128.f;
__device__ __forceinline__ float clamp_log_decay(float g) { return g < kLogDecayFloor ? kLogDecayFloor : g; }

// log alpha = -exp(A) * softplus(a + b_alpha)
__device__ __forceinline__ float log_decay(float a_logit, float A, float b_alpha) {
    return -expf(A) * softplus_acc(a_logit + b_alpha);
}

// ---- packed fp32x2 arithmetic (sm_100): two lanes of work per instruction
union F2 {
    unsigned long long u;
    float2 f;
};
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    F2 x, y, z, r;
    x.f = a; y.f = b; z.f = c;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.u) : "l"(x.u), "l"(y.u), "l"(z.u));
    return r.f;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    F2 x, y, r;
    x.f = a; y.f = b;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.u) : "l"(x.u), "l"(y.u));
    return r.f;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    F2 x, y, r;
    x.f = a; y.f = b;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.u) : "l"(x.u), "l"(y.u));
    return r.f;
}

// Fast-math gates for the tensor-core path: softplus with the exp / log
// intrinsics (absolute error ~1e-7), sigmoid with the intrinsic exp.
__device__ __forceinline__ float softplus_fast(float x) {
    return fmaxf(x, 0.f) + __logf(1.0f + __expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

template <int W>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sequence index of packed token t: the largest n with cu[n] <= t (cu non-decreasing).
__device__ __forceinline__ int seq_of_token(const int32_t *cu, int n_seq, int t) {
    int lo = 0, hi = n_seq;  // answer in [0, n_seq)
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace gdn

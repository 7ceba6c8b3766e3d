// K2a -- prelude plus the state-independent part of the chunked gated delta
// rule, one 64-token chunk of one head per iteration, chunks of all sequences
// and heads in parallel.
//
// Prelude (slinene.github.io write-up of "On the Design of Qwen3.8-Next
// Architecture", 模块 A, 参数化): q = L2Norm(SiLU(ShortConv(q_raw))), k likewise,
// v = SiLU(ShortConv(v_raw)), beta = sigmoid(b), log alpha = -e^A softplus(a + b_alpha).
//
// Chunk form (derived from the erase-then-write update of the same section,
// 递归状态): with u_i = beta_i (v_i - alpha_i S_{i-1}^T k_i) the update is
// S_i = alpha_i S_{i-1} + k_i u_i^T.  With G_i = sum_{j<=i} log alpha_j inside
// the chunk and S the state before it,
//     (I + L) U = diag(beta) (V - diag(e^G) K S),
//     L_ij = beta_i (k_i . k_j) e^{G_i - G_j}  (j < i),
// so U = U' - W S with T = (I + L)^-1, W = T diag(beta e^G) K, U' = T diag(beta) V.
// The chain kernel needs, per chunk: -W, U', Qt = diag(e^G) Q,
// Kt = diag(e^{G_C - G}) K, Aqk_ij = (q_i . k_j) e^{G_i - G_j} (j <= i), e^{G_C}.
// Every decay is exp of a non-positive difference of log sums.
//
// The output RMSNorm is scale-invariant, so for short-memory heads the output
// is sensitive to the *relative* error of q_i . k_i, which can be tiny.  The
// q.k and k.k products therefore use a two-term fp16 split of the fp32 q and k
// (x = hi + lo): [Qh;Kh]Kh^T + [Qh;Kh]Kl^T + [Ql;Kl]Kh^T, fp32 accumulation.
//
// Per chunk: the gates and their in-chunk cumulative log decays first; then the
// prelude in registers -> fp16 hi/lo tiles in smem, with Qt and Kt written to
// global memory straight from it; the split [Q;K]K^T on tcgen05 (M=128, N=64) ->
// TMEM; Aqk and L from TMEM; T = (I + L)^-1 by 16 x 16 blocks (warp-level tensor
// cores, tf32 with a two-term split); [T diag(beta e^G); T diag(beta)] times K and
// V on tcgen05 -> TMEM; results to global memory in fp16.
//
// Device code only: the kernels that run it and the device error word it raises
// (g_prep_err, defined before this header is included) live in prefill_tc.cu.
#pragma once

#include <cuda_fp16.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

constexpr uint32_t kPrepMaxPolls = 1u << 22;

// Synchronisation of one prep worker: a whole CTA, or 256 threads of a larger
// CTA on a named barrier (two workers per CTA in the fused prefill kernel).
struct PrepBlockSync {
    __device__ __forceinline__ void sync() const { __syncthreads(); }
    __device__ __forceinline__ bool all(bool p) const { return __syncthreads_and(p); }
};
struct PrepGroupSync {
    int id;   // named barrier of the worker's 256 threads
    __device__ __forceinline__ void sync() const { umma::named_bar_sync(id, 256); }
    __device__ __forceinline__ bool all(bool p) const {
        uint32_t r;
        asm volatile(
            "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n"
            " bar.red.and.pred po, %2, 256, pi;\n selp.u32 %0, 1, 0, po;\n}\n"
            : "=r"(r) : "r"((uint32_t)p), "r"(id) : "memory");
        return r != 0;
    }
};

// Worker-wide bounded wait for phase `phase` of `bar`: true only if every thread
// saw it complete; on expiry the worker's thread 0 raises the device error word.
template <class Sync>
__device__ __forceinline__ bool prep_wait(const Sync &sy, uint64_t *bar, uint32_t phase, uint32_t max_polls,
                                          int tid) {
    const bool ok = sy.all(umma::mbar_wait_bounded(bar, phase, max_polls));
    if (!ok && tid == 0) atomicOr(&g_prep_err, 1u);
    return ok;
}

namespace prep {
constexpr int C = 64;          // chunk length
constexpr int DK = 128;
constexpr int OFF_HI = 0;      // [Qh;Kh] K-major, 2 k-blocks x 16 KB
constexpr int OFF_LO = 32768;  // [Ql;Kl] K-major, 2 k-blocks x 16 KB; later L and T fp32 [64][64]
constexpr int OFF_V = 65536;   // V MN-major, DV/64 mn-blocks x 8 KB
constexpr int OFF_T = 81920;   // [T'; T''] K-major, 1 k-block x 16 KB
constexpr int OFF_MISC = 98304;  // G, beta, barriers [0, 1024); block products [1024, 4096);
                                 // per-token factors e^G, e^{G_C - G}, beta e^G [4096, 4864)
constexpr int MISC_BYTES = 4864;
constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 256;
}  // namespace prep

// 2^x on the special-function unit (ex2.approx: about 2 ulp; inputs here are at
// most 60, and underflow to 0 is what the callers want)
__device__ __forceinline__ float ex2_fast(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Ask L2 to fetch the raw q, k and v rows of chunk c of head h (and the three rows
// before it): one 256-byte row per thread for the first 3 * (C + 3) threads.
template <int DV>
__device__ __forceinline__ void prefetch_chunk_rows(const bf16 *q, const bf16 *k, const bf16 *v, int H, int h,
                                                    int t0, int t_end, int tid) {
    constexpr int R = 64 + 3;
    if (tid >= 3 * R) return;
    const int which = tid / R, t = t0 - 3 + tid % R;
    if (t < 0 || t >= t_end) return;
    const bf16 *row = which == 0 ? q + ((size_t)t * H + h) * 128
                    : which == 1 ? k + ((size_t)t * H + h) * 128 : v + ((size_t)t * H + h) * DV;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row), "r"(which == 2 ? DV * 2 : 256) : "memory");
}

// Row staging for coalesced global stores.  A tile of 16-bit rows is staged in
// shared memory with its 16-byte chunks rotated by the row (chunk c of row r at
// position c ^ (r % 8)), so that both the row-per-lane writes out of tensor
// memory and the row-contiguous reads that follow are free of bank conflicts.
// RB: bytes per row.
template <int RB>
__device__ __forceinline__ uint32_t stage_off(int r, int c) {
    return (uint32_t)(r * RB + ((c ^ (r & 7)) << 4));
}
// Copy rows [0, len) of a staged tile of 64 rows to global memory, a warp storing
// whole rows (RB / 16 lanes per row), NT threads.  Row r goes to dst + r * stride.
template <int RB, int NT>
__device__ __forceinline__ void store_rows(const uint8_t *stage, __half *dst, size_t stride, int len, int tid) {
    constexpr int CPR = RB / 16;   // 16-byte chunks per row
    for (int e = tid; e < len * CPR; e += NT) {
        const int r = e / CPR, c = e % CPR;
        *reinterpret_cast<uint4 *>(dst + (size_t)r * stride + c * 8) =
            *reinterpret_cast<const uint4 *>(stage + stage_off<RB>(r, c));
    }
}

// Conv + SiLU of 8 channels (4 pairs) for tokens [i0, i0 + N) of a chunk: all
// N + 3 raw rows (zero before the sequence start and past its end) are loaded
// first, then a sliding window of converted rows produces y[N][4] (pairs).
template <int N>
__device__ __forceinline__ void conv_load(const bf16 *src, size_t row_stride, int col, int t0, int s_begin, int i0,
                                          int len, uint4 (&raw)[N + 3]) {
    const bf16 *base = src + (size_t)(t0 + i0 - 3) * row_stride + col;
#pragma unroll
    for (int r = 0; r < N + 3; ++r) {
        const int i = i0 + r - 3;            // chunk-relative row
        const bool ok = (i < len) && (t0 + i >= s_begin);
        raw[r] = ok ? __ldg(reinterpret_cast<const uint4 *>(base + (size_t)r * row_stride)) : make_uint4(0, 0, 0, 0);
    }
}

template <int N>
__device__ __forceinline__ void conv_silu(const uint4 (&raw)[N + 3], const float2 (&w)[4][4], int i0, int len,
                                          float2 (&y)[N][4]) {
    auto cvt = [](uint4 u, float2 (&x)[4]) {
        x[0] = make_float2(bf16lo(u.x), bf16hi(u.x));
        x[1] = make_float2(bf16lo(u.y), bf16hi(u.y));
        x[2] = make_float2(bf16lo(u.z), bf16hi(u.z));
        x[3] = make_float2(bf16lo(u.w), bf16hi(u.w));
    };
    float2 h0[4], h1[4], h2[4];
    cvt(raw[0], h0);
    cvt(raw[1], h1);
    cvt(raw[2], h2);
    const float2 nl2e = make_float2(-1.4426950408889634f, -1.4426950408889634f);
    const float2 one = make_float2(1.f, 1.f);
#pragma unroll
    for (int ii = 0; ii < N; ++ii) {
        float2 x[4];
        cvt(raw[ii + 3], x);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float2 a = fmul2(w[p][0], h0[p]);
            a = ffma2(w[p][1], h1[p], a);
            a = ffma2(w[p][2], h2[p], a);
            a = ffma2(w[p][3], x[p], a);
            // silu(a) = a / (1 + 2^(-a log2 e)); the pair shares one reciprocal,
            // 1 / (d.x d.y), with the exponents clamped to 60 so the product stays finite
            const float2 e = fmul2(a, nl2e);
            const float2 d = fadd2(one, make_float2(ex2_fast(fminf(e.x, 60.f)), ex2_fast(fminf(e.y, 60.f))));
            const float r = __fdividef(1.0f, d.x * d.y);
            y[ii][p] = fmul2(fmul2(a, make_float2(d.y, d.x)), make_float2(r, r));
            h0[p] = h1[p]; h1[p] = h2[p]; h2[p] = x[p];
        }
        if (i0 + ii >= len) {
#pragma unroll
            for (int p = 0; p < 4; ++p) y[ii][p] = make_float2(0.f, 0.f);
        }
    }
}

__device__ __forceinline__ void load_conv_w(const float *conv_w, int chan, float2 (&w)[4][4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(conv_w) + chan + 2 * p);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(conv_w) + chan + 2 * p + 1);
        w[p][0] = make_float2(a.x, b.x); w[p][1] = make_float2(a.y, b.y);
        w[p][2] = make_float2(a.z, b.z); w[p][3] = make_float2(a.w, b.w);
    }
}

// ---- T = (I + L)^-1 for the strictly lower triangular 64 x 64 L of a chunk.
//
// L and T are kept as their ten 16 x 16 blocks on or below the diagonal
// ("block-compact": block (bi, bj), bj <= bi, at index bi (bi + 1) / 2 + bj, rows
// of 20 floats so that the fragment loads below are free of bank conflicts).
// Diagonal blocks D_b = (I + L_bb)^-1 by forward substitution; then the 2 x 2
// block recursion on 32 x 32 halves,
//   T_10 = -D_1 L_10 D_0,  T_32 = -D_3 L_32 D_2,
//   X_a0 = L_{2+a,0} D_0 + L_{2+a,1} T_10,  X_a1 = L_{2+a,1} D_1   (a = 0, 1),
//   T_2b = -D_2 X_0b,  T_3b = -(T_32 X_0b + D_3 X_1b)               (b = 0, 1),
// whose 16 x 16 x 16 block products run on the warp-level tensor-core MMA
// (m16n8k8, tf32) with each operand split into two tf32 terms, x = hi + lo, and
// the three products hi*hi + hi*lo + lo*hi accumulated in fp32: about fp32
// accuracy, as the solve needs (T multiplies every row of W and U').  The
// products are far too small for tcgen05 (whose M is at least 64).
namespace tsolve {
constexpr int BS = 20;                 // row stride of a block (floats)
constexpr int BLK = 16 * BS;           // floats per block
__device__ __forceinline__ int bidx(int bi, int bj) { return bi * (bi + 1) / 2 + bj; }

__device__ __forceinline__ uint32_t tf32_hi(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32_hi(x);
    lo = tf32_hi(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// c += A B[:, 8 nt .. 8 nt + 8): A a 16 x 16 block (row stride BS), B a 16 x 16
// block (row stride bs) of which the n-tile nt is used.  Lane (g, t) = (lane / 4,
// lane % 4) holds c[0..3] = C(g, 2t), C(g, 2t + 1), C(g + 8, 2t), C(g + 8, 2t + 1).
__device__ __forceinline__ void prod(float (&c)[4], const float *A, const float *B, int bs, int nt, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t ah[4], al[4], bh[2], bl[2];
        split(A[g * BS + 8 * ks + t], ah[0], al[0]);
        split(A[(g + 8) * BS + 8 * ks + t], ah[1], al[1]);
        split(A[g * BS + 8 * ks + t + 4], ah[2], al[2]);
        split(A[(g + 8) * BS + 8 * ks + t + 4], ah[3], al[3]);
        split(B[(8 * ks + t) * bs + 8 * nt + g], bh[0], bl[0]);
        split(B[(8 * ks + t + 4) * bs + 8 * nt + g], bh[1], bl[1]);
        mma_tf32(c, al, bh);
        mma_tf32(c, ah, bl);
        mma_tf32(c, ah, bh);
    }
}

// Store -c (an n-tile of a 16 x 16 result) into a block of row stride bs.
__device__ __forceinline__ void store_neg(float *B, int bs, int nt, const float (&c)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2 *>(B + g * bs + 8 * nt + 2 * t) = make_float2(-c[0], -c[1]);
    *reinterpret_cast<float2 *>(B + (g + 8) * bs + 8 * nt + 2 * t) = make_float2(-c[2], -c[3]);
}
__device__ __forceinline__ void store_pos(float *B, int bs, int nt, const float (&c)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2 *>(B + g * bs + 8 * nt + 2 * t) = make_float2(c[0], c[1]);
    *reinterpret_cast<float2 *>(B + (g + 8) * bs + 8 * nt + 2 * t) = make_float2(c[2], c[3]);
}
}  // namespace tsolve

// T = (I + L)^-1 (block-compact L and T, see above) by 256 threads = 8 warps
// synchronised by `sy`; `scratch` holds 4 blocks plus 4 warp tiles of 16 x 8.
template <class Sync>
__device__ __forceinline__ void solve_unit_lower(const Sync &sy, const float *L, float *T, float *scratch, int tid) {
    using namespace tsolve;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < 64) {   // diagonal blocks: thread (b, cc) owns column cc of D_b
        const int b = tid >> 4, cc = tid & 15;
        const float *Lb = L + bidx(b, b) * BLK;
        float *Tb = T + bidx(b, b) * BLK;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < r; ++j) acc = fmaf(-Lb[r * BS + j], x[j], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * BS + cc] = x[r];
    }
    sy.sync();
    float *X = scratch;                     // X_ab at X + (2a + b) * BLK
    float *W8 = scratch + 4 * BLK;          // warp tiles 16 x 8 for the first level
    if (warp < 4) {
        // T_10 (warps 0, 1) and T_32 (warps 2, 3), n-tile warp & 1
        const int bi = warp < 2 ? 1 : 3, bj = bi - 1, nt = warp & 1;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        prod(c, L + bidx(bi, bj) * BLK, T + bidx(bj, bj) * BLK, BS, nt, lane);
        float *w8 = W8 + warp * 128;
        // the n-tile as a 16 x 8 B operand (columns 0..7 of a row stride 8)
        const int g = lane >> 2, t = lane & 3;
        *reinterpret_cast<float2 *>(w8 + g * 8 + 2 * t) = make_float2(c[0], c[1]);
        *reinterpret_cast<float2 *>(w8 + (g + 8) * 8 + 2 * t) = make_float2(c[2], c[3]);
        __syncwarp();
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        prod(d, T + bidx(bi, bi) * BLK, w8, 8, 0, lane);
        store_neg(T + bidx(bi, bj) * BLK, BS, nt, d, lane);
    }
    sy.sync();
    {   // X_ab, n-tile: warp = (a, b, nt)
        const int a = warp >> 2, b = (warp >> 1) & 1, nt = warp & 1;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if (b == 0) {
            prod(c, L + bidx(2 + a, 0) * BLK, T + bidx(0, 0) * BLK, BS, nt, lane);
            prod(c, L + bidx(2 + a, 1) * BLK, T + bidx(1, 0) * BLK, BS, nt, lane);
        } else {
            prod(c, L + bidx(2 + a, 1) * BLK, T + bidx(1, 1) * BLK, BS, nt, lane);
        }
        store_pos(X + (2 * a + b) * BLK, BS, nt, c, lane);
    }
    sy.sync();
    {   // T_{2+a, b}, n-tile: warp = (a, b, nt)
        const int a = warp >> 2, b = (warp >> 1) & 1, nt = warp & 1;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if (a == 0) {
            prod(c, T + bidx(2, 2) * BLK, X + b * BLK, BS, nt, lane);
        } else {
            prod(c, T + bidx(3, 2) * BLK, X + b * BLK, BS, nt, lane);
            prod(c, T + bidx(3, 3) * BLK, X + (2 + b) * BLK, BS, nt, lane);
        }
        store_neg(T + bidx(2 + a, b) * BLK, BS, nt, c, lane);
    }
    sy.sync();
}

// Inputs and outputs of the chunk prep.
struct PrepArgs {
    const bf16 *q, *k, *v;
    const float *conv_w;
    const bf16 *a_logit, *b_logit;
    const float *A, *b_alpha;
    int H;
    __half *Qt, *Kt, *Wn, *Up, *Aqk;
    float *decay;
};

// One 64-token chunk c of head h of the sequence [s_begin, s_end), by one worker
// of 256 threads (tid in [0, 256)) with its own shared memory `sm`, 256 TMEM
// columns at `tbase` and mbarrier `bar`.  Returns false when a bounded wait
// expired (the device error word is raised).  `publish` (optional) is the ready
// flag of the worker's previous chunk: it is set, with release semantics, once
// this chunk's prelude is done -- by then the previous chunk's stores have long
// drained, so the fence that orders them before the flag costs little.
template <int DV, class Sync>
__device__ __forceinline__ bool prep_one_chunk(const Sync &sy, const PrepArgs pa, uint8_t *sm,
                                               uint32_t tbase, uint64_t *bar, uint32_t &phase, int tid,
                                               int h, int s_begin, int s_end, int c, int *publish = nullptr) {
    using namespace prep;
    const bf16 *q = pa.q, *k = pa.k, *v = pa.v;
    const float *conv_w = pa.conv_w;
    const bf16 *a_logit = pa.a_logit, *b_logit = pa.b_logit;
    const int H = pa.H;
    __half *Qt = pa.Qt, *Kt = pa.Kt, *Wn = pa.Wn, *Up = pa.Up, *Aqk = pa.Aqk;
    float *decay = pa.decay;
    uint8_t *sHI = sm + OFF_HI, *sLO = sm + OFF_LO, *sV = sm + OFF_V, *sT = sm + OFF_T;
    // L and T block-compact fp32 (10 blocks of 16 x 20 each) alias [Ql;Kl] after the
    // q.k MMA; the solve's scratch uses the [T'; T''] tile's region, written after it
    float *sL = reinterpret_cast<float *>(sm + OFF_LO);
    float *sTf = sL + 10 * tsolve::BLK;
    float *sX = reinterpret_cast<float *>(sm + OFF_T);             // solve scratch: [0, 7 KB)
    uint8_t *sAqk = sm + OFF_T + 8192;                            // Aqk row stage: 64 x 128 B
    float *sG = reinterpret_cast<float *>(sm + OFF_MISC);        // 64
    float *sBeta = sG + 64;                                      // 64
    float *sTot = sBeta + 64;                                    // 2: partial sums of warps 0, 1
    float *sEG = reinterpret_cast<float *>(sm + OFF_MISC + 4096);  // 64: e^{G_i}
    float *sEK = sEG + 64;                                       // 64: e^{G_C - G_i}
    float *sBE = sEK + 64;                                       // 64: beta_i e^{G_i}
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t trow = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
    const float eA = expf(__ldg(pa.A + h)), ba = __ldg(pa.b_alpha + h);

    // this thread's prelude channels: q/k octet tid % 32 for tokens 8 * warp .. + 8,
    // and v octet tid % (DV / 8) for a 64 / VPARTS-token part of the chunk
    constexpr int NT = 256;
    const int qk_oct = tid & 31;                  // 0..15 q, 16..31 k
    const bool is_k = qk_oct >= 16;
    const int qk_col = h * DK + (qk_oct & 15) * 8;
    const int qk_chan = (is_k ? H * DK : 0) + qk_col;
    constexpr int VO = DV / 8;                    // v octets
    constexpr int VPARTS = NT / VO;               // token parts for v
    const int v_oct = tid % VO, v_part = tid / VO;
    const int v_col = h * DV + v_oct * 8;
    const int v_chan = 2 * H * DK + v_col;
    bool ok = true;
    const int t0 = s_begin + c * C;
    const int len = min(C, s_end - t0);
    // the token's gate logits (thread tid < len) and the first raw q/k rows are
    // loaded first, so that their latency passes while the gates are computed
    bf16 a_raw = __float2bfloat16(0.f), b_raw = __float2bfloat16(0.f);
    if (tid < len) {
        const size_t gi = (size_t)(t0 + tid) * H + h;
        a_raw = a_logit[gi];
        b_raw = b_logit[gi];
    }
    const bf16 *qk_src = is_k ? k : q;
    uint4 raw[7];
    conv_load<4>(qk_src, (size_t)H * DK, qk_col, t0, s_begin, 8 * warp, len, raw);

    // ---- 1. gates: beta, log alpha and their in-chunk cumulative sum G, then the
    //         per-token factors e^{G_i}, e^{G_C - G_i}, beta_i e^{G_i}
    if (tid < C) {
        float g = 0.f, be = 0.f;
        if (tid < len) {
            g = clamp_log_decay(-eA * softplus_fast(to_f32(a_raw) + ba));
            be = sigmoid_fast(to_f32(b_raw));
        }
        // inclusive scan of the log decays within each warp, then across the two
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, g, o);
            if (lane >= o) g += y;
        }
        if (tid == 31) sTot[0] = g;
        if (tid == 63) sTot[1] = g;
        sBeta[tid] = be;
        sG[tid] = g;
    }
    sy.sync();
    if (tid < C) {   // each thread finishes its own token: G_i, and the per-token factors
        const float w0 = sTot[0];
        const float Gi = sG[tid] + (tid >= 32 ? w0 : 0.f);
        const float GC = w0 + sTot[1];
        const float eg = __expf(Gi);
        sG[tid] = Gi;
        sEG[tid] = eg;
        sEK[tid] = __expf(GC - Gi);
        sBE[tid] = sBeta[tid] * eg;
        if (tid == 0) decay[(size_t)t0 * H + h] = __expf(GC);
    }
    sy.sync();

    // ---- 2. prelude: q, k -> L2-normalised fp32 -> hi/lo fp16 tiles, and Qt = e^G q,
    //         Kt = e^{G_C - G} k (fp16) straight to global memory; v -> fp16 tile
    // (conv weights re-read per chunk from L1/L2 to keep them out of the solve's registers)
    {
        float2 w[4][4];
        load_conv_w(conv_w, qk_chan, w);
        const int oc = qk_oct & 15;
        uint8_t *hb = sHI + (oc / 8) * 16384, *lb = sLO + (oc / 8) * 16384;
        const float *fac = is_k ? sEK : sEG;
        __half *dst_t = is_k ? Kt : Qt;
        // the warp's 8 tokens in two halves of 4 (a 7-row window each; the halo rows
        // are re-read from L1), which keeps the prelude's registers in bounds
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            if (hf == 1) conv_load<4>(qk_src, (size_t)H * DK, qk_col, t0, s_begin, 8 * warp + 4, len, raw);
            float2 y[4][4];
            conv_silu<4>(raw, w, 8 * warp + 4 * hf, len, y);
            // L2 norm over the 16 lanes that hold this head's q (or k): 4 tokens at once
            float ss[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                float2 acc = fmul2(y[ii][0], y[ii][0]);
#pragma unroll
                for (int p = 1; p < 4; ++p) acc = ffma2(y[ii][p], y[ii][p], acc);
                ss[ii] = acc.x + acc.y;
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) ss[ii] += __shfl_xor_sync(0xffffffffu, ss[ii], o);
            }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = 8 * warp + 4 * hf + ii;   // token of the chunk
                const float r = rsqrtf(ss[ii] + kNormEps);
                const float2 rr = make_float2(r, r);
                const float sc = fac[i];
                const float2 scs = make_float2(sc, sc);
                uint32_t hw[4], lw[4], tw[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 x = fmul2(y[ii][p], rr);
                    const __half2 hh = __floats2half2_rn(x.x, x.y);
                    const float2 hf2 = __half22float2(hh);
                    const __half2 ll = __floats2half2_rn(x.x - hf2.x, x.y - hf2.y);
                    hw[p] = *reinterpret_cast<const uint32_t *>(&hh);
                    lw[p] = *reinterpret_cast<const uint32_t *>(&ll);
                    const float2 xt = fmul2(x, scs);
                    tw[p] = umma::pack_half2(xt.x, xt.y);
                }
                const int row = (is_k ? 64 : 0) + i;
                umma::st_chunk(hb, row, oc % 8, make_uint4(hw[0], hw[1], hw[2], hw[3]));
                umma::st_chunk(lb, row, oc % 8, make_uint4(lw[0], lw[1], lw[2], lw[3]));
                if (i < len)
                    *reinterpret_cast<uint4 *>(dst_t + ((size_t)(t0 + i) * H + h) * DK + oc * 8) =
                        make_uint4(tw[0], tw[1], tw[2], tw[3]);
            }
        }
    }
    {
        float2 w[4][4];
        load_conv_w(conv_w, v_chan, w);
        constexpr int NV = C / VPARTS;
        uint4 vraw[NV + 3];
        conv_load<NV>(v, (size_t)H * DV, v_col, t0, s_begin, NV * v_part, len, vraw);
        float2 y[NV][4];
        conv_silu<NV>(vraw, w, NV * v_part, len, y);
#pragma unroll
        for (int ii = 0; ii < NV; ++ii)
            umma::st_chunk(sV + (v_oct / 8) * 8192, NV * v_part + ii, v_oct % 8,
                           make_uint4(umma::pack_half2(y[ii][0].x, y[ii][0].y), umma::pack_half2(y[ii][1].x, y[ii][1].y),
                                      umma::pack_half2(y[ii][2].x, y[ii][2].y), umma::pack_half2(y[ii][3].x, y[ii][3].y)));
    }
    umma::fence_proxy_async_smem();
    sy.sync();
    if (publish && tid == 32) {
        // the previous chunk's writes (every thread's) precede this worker's barriers;
        // a thread other than the MMA issuer makes them visible and sets the flag, so
        // that the fence's wait for the stores does not delay the MMA below
        __threadfence();
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(publish), "r"(1) : "memory");
    }

    // ---- 3. [Q;K] K^T = [Qh;Kh]Kh^T + [Qh;Kh]Kl^T + [Ql;Kl]Kh^T -> TMEM [0, 64)
    if (tid == 0) {
        umma::tc_fence_after();
        const uint32_t hi = umma::smem_u32(sHI), lo = umma::smem_u32(sLO);
        const uint32_t idesc = umma::idesc_f16(128, 64, false, false);
#pragma unroll
        for (int s = 0; s < DK / 16; ++s) {
            const uint32_t off = (s / 4) * 16384 + (s % 4) * 32;
            const uint64_t ah = umma::sw128_desc(hi + off, 16, 1024), al = umma::sw128_desc(lo + off, 16, 1024);
            const uint64_t bh = umma::sw128_desc(hi + off + 8192, 16, 1024), bl = umma::sw128_desc(lo + off + 8192, 16, 1024);
            umma::mma_f16(tbase, ah, bh, idesc, s > 0);
            umma::mma_f16(tbase, ah, bl, idesc, 1u);
            umma::mma_f16(tbase, al, bh, idesc, 1u);
        }
        umma::mma_commit(bar);
    }
    ok = prep_wait(sy, bar, phase, kPrepMaxPolls, tid);
    phase ^= 1;
    umma::tc_fence_after();
    if (!ok) return false;

    // ---- 4. rows 0..63: Aqk (masked, decayed q.k) -> global; rows 64..127: L -> smem
    //         warp w reads lane quadrant w % 4, columns [32 (w / 4), + 32)
    {
        float v[32];
        const int j0 = 32 * (warp >> 2);
        umma::tmem_ld32(trow + j0, v);
        const int i = (32 * (warp & 3) + lane) & 63;
        const float Gi = sG[i];
        if ((warp & 3) < 2) {
            // Aqk row i (its 32 columns j0..) into the row stage; stored after the barrier
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = j0 + q8 * 8 + e;
                    x[e] = (j <= i) ? v[q8 * 8 + e] * __expf(Gi - sG[j]) : 0.f;
                }
                *reinterpret_cast<uint4 *>(sAqk + stage_off<C * 2>(i, j0 / 8 + q8)) =
                    make_uint4(umma::pack_half2(x[0], x[1]), umma::pack_half2(x[2], x[3]),
                               umma::pack_half2(x[4], x[5]), umma::pack_half2(x[6], x[7]));
            }
        } else {
            // L_ij = beta_i (k_i . k_j) e^{G_i - G_j} (j < i) into the blocks (i / 16, jb)
            // on or below the diagonal (the solve reads the diagonal block's lower part only)
            const float bi = sBeta[i];
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int jb = (j0 >> 4) + hb;
                if (jb > (i >> 4)) continue;
                float4 *dst = reinterpret_cast<float4 *>(sL + tsolve::bidx(i >> 4, jb) * tsolve::BLK +
                                                         (i & 15) * tsolve::BS);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 16 * jb + q4 * 4 + e;
                        x[e] = (j < i) ? bi * v[16 * hb + q4 * 4 + e] * __expf(Gi - sG[j]) : 0.f;
                    }
                    dst[q4] = make_float4(x[0], x[1], x[2], x[3]);
                }
            }
        }
    }
    umma::tc_fence_before();
    sy.sync();
    // Aqk rows to global memory, whole rows per warp (its stage is not reused before
    // the barriers of the solve)
    store_rows<C * 2, NT>(sAqk, Aqk + ((size_t)t0 * H + h) * C, (size_t)H * C, len, tid);

    // ---- 5. T = (I + L)^-1 (fp32, blocked); then T' = T diag(beta e^G) in rows
    //         0..63 and T'' = T diag(beta) in rows 64..127 of an fp16 K-major tile
    solve_unit_lower(sy, sL, sTf, sX, tid);
    for (int idx = tid; idx < C * 8; idx += NT) {
        const int i = idx >> 3, ch = idx & 7;
        // only the blocks on or below the diagonal of T exist: the rest is zero
        const bool in = (ch >> 1) <= (i >> 4);
        float4 t0v = make_float4(0.f, 0.f, 0.f, 0.f), t1v = t0v;
        if (in) {
            const float4 *tr = reinterpret_cast<const float4 *>(sTf + tsolve::bidx(i >> 4, ch >> 1) * tsolve::BLK +
                                                                (i & 15) * tsolve::BS + (ch & 1) * 8);
            t0v = tr[0];
            t1v = tr[1];
        }
        const float tv[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
        float a1[8], a2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = ch * 8 + e;
            const float t = tv[e];
            a1[e] = t * sBE[j];
            a2[e] = t * sBeta[j];
        }
        umma::st_chunk(sT, i, ch, make_uint4(umma::pack_half2(a1[0], a1[1]), umma::pack_half2(a1[2], a1[3]),
                                             umma::pack_half2(a1[4], a1[5]), umma::pack_half2(a1[6], a1[7])));
        umma::st_chunk(sT, 64 + i, ch, make_uint4(umma::pack_half2(a2[0], a2[1]), umma::pack_half2(a2[2], a2[3]),
                                                  umma::pack_half2(a2[4], a2[5]), umma::pack_half2(a2[6], a2[7])));
    }
    umma::fence_proxy_async_smem();
    sy.sync();

    // ---- 6. W-part = T' K -> TMEM [0, DK);  U'-part = T'' V -> TMEM [DK, DK + DV)
    if (tid == 0) {
        umma::tc_fence_after();
        const uint32_t aT = umma::smem_u32(sT), aK = umma::smem_u32(sHI) + 8192, aV = umma::smem_u32(sV);
        const uint32_t idw = umma::idesc_f16(128, DK, false, true);
        const uint32_t idu = umma::idesc_f16(128, DV, false, true);
#pragma unroll
        for (int s = 0; s < C / 16; ++s) {
            const uint64_t ad = umma::sw128_desc(aT + s * 32, 16, 1024);
            umma::mma_f16(tbase, ad, umma::sw128_desc(aK + s * 2048, 16384, 1024), idw, s > 0);
            umma::mma_f16(tbase + DK, ad, umma::sw128_desc(aV + s * 2048, 8192, 1024), idu, s > 0);
        }
        umma::mma_commit(bar);
    }
    ok = prep_wait(sy, bar, phase, kPrepMaxPolls, tid);
    phase ^= 1;
    umma::tc_fence_after();
    if (!ok) return false;

    // ---- 7. rows 0..63 of the W-part -> -W; rows 64..127 of the U'-part -> U'
    //         (warp w: lane quadrant w % 4, column half w / 4; TMEM loads are
    //         warp-collective), through row stages in the [Ql;Kl] region (free since
    //         the T' build) so that the global stores are whole rows per warp
    {
        uint8_t *sW = sLO, *sU = sLO + 64 * DK * 2;
        const int i = (32 * (warp & 3) + lane) & 63;
        const int half = warp >> 2;
        if ((warp & 3) < 2) {
#pragma unroll
            for (int c0 = half * (DK / 2); c0 < (half + 1) * (DK / 2); c0 += 32) {
                float vv[32];
                umma::tmem_ld32(trow + c0, vv);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(sW + stage_off<DK * 2>(i, c0 / 8 + q8)) = make_uint4(
                        umma::pack_half2(-vv[q8 * 8 + 0], -vv[q8 * 8 + 1]), umma::pack_half2(-vv[q8 * 8 + 2], -vv[q8 * 8 + 3]),
                        umma::pack_half2(-vv[q8 * 8 + 4], -vv[q8 * 8 + 5]), umma::pack_half2(-vv[q8 * 8 + 6], -vv[q8 * 8 + 7]));
            }
        } else {
#pragma unroll
            for (int c0 = half * (DV / 2); c0 < (half + 1) * (DV / 2); c0 += 32) {
                float vv[32];
                umma::tmem_ld32(trow + DK + c0, vv);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(sU + stage_off<DV * 2>(i, c0 / 8 + q8)) = make_uint4(
                        umma::pack_half2(vv[q8 * 8 + 0], vv[q8 * 8 + 1]), umma::pack_half2(vv[q8 * 8 + 2], vv[q8 * 8 + 3]),
                        umma::pack_half2(vv[q8 * 8 + 4], vv[q8 * 8 + 5]), umma::pack_half2(vv[q8 * 8 + 6], vv[q8 * 8 + 7]));
            }
        }
        umma::tc_fence_before();
        sy.sync();
        store_rows<DK * 2, NT>(sW, Wn + ((size_t)t0 * H + h) * DK, (size_t)H * DK, len, tid);
        store_rows<DV * 2, NT>(sU, Up + ((size_t)t0 * H + h) * DV, (size_t)H * DV, len, tid);
    }
    umma::tc_fence_before();
    sy.sync();
    return true;
}

}  // namespace gdn

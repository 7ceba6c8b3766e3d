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
// Per chunk: prelude in registers -> fp16 hi/lo tiles in smem; the split
// [Q;K]K^T on tcgen05 (M=128, N=64) -> TMEM, with Qt and Kt written out while
// it runs; Aqk and L from TMEM; T by blocked forward substitution in fp32 over
// all 256 threads; [T diag(beta e^G); T diag(beta)] times K and V on tcgen05 ->
// TMEM; results to global memory in fp16.
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
constexpr int OFF_MISC = 98304;  // G, beta, barriers [0, 1024); block products [1024, 4096)
constexpr int SMEM = OFF_MISC + 4096 + 1024;
constexpr uint32_t TMEM_COLS = 256;
}  // namespace prep

// Conv + SiLU of 8 channels (4 pairs) for tokens [i0, i0 + N) of a chunk: all
// N + 3 raw rows (zero before the sequence start and past its end) are loaded
// first, then a sliding window of converted rows produces y[N][4] (pairs).
template <int N>
__device__ __forceinline__ void conv_silu(const bf16 *src, size_t row_stride, int col,
                                          const float2 (&w)[4][4], int t0, int s_begin, int i0,
                                          int len, float2 (&y)[N][4]) {
    uint4 raw[N + 3];
#pragma unroll
    for (int r = 0; r < N + 3; ++r) {
        const int i = i0 + r - 3;            // chunk-relative row
        const int t = t0 + i;
        const bool ok = (i < len) && (t >= s_begin);
        raw[r] = ok ? __ldg(reinterpret_cast<const uint4 *>(src + (size_t)t * row_stride + col))
                    : make_uint4(0, 0, 0, 0);
    }
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
            // silu(a) = a / (1 + 2^(-a log2 e))
            const float2 e = fmul2(a, nl2e);
            const float2 d = fadd2(one, make_float2(exp2f(e.x), exp2f(e.y)));
            y[ii][p] = make_float2(__fdividef(a.x, d.x), __fdividef(a.y, d.y));
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

// acc(r, c) += sum_k A[ar + r][ac + k] * B[br + k][bc + c] over a 16 x 16 block
// product, A and B row-major fp32 [64][64] in shared memory.
__device__ __forceinline__ float blk16(const float *A, int ar, int ac, const float *B, int br, int bc,
                                       int r, int c, float acc) {
    const float4 *a = reinterpret_cast<const float4 *>(A + (ar + r) * 64 + ac);
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const float4 av = a[k4];
        acc = fmaf(av.x, B[(br + 4 * k4 + 0) * 64 + bc + c], acc);
        acc = fmaf(av.y, B[(br + 4 * k4 + 1) * 64 + bc + c], acc);
        acc = fmaf(av.z, B[(br + 4 * k4 + 2) * 64 + bc + c], acc);
        acc = fmaf(av.w, B[(br + 4 * k4 + 3) * 64 + bc + c], acc);
    }
    return acc;
}

// T = (I + L)^-1 for a strictly lower triangular 64 x 64 L, by 16 x 16 blocks:
// diagonal blocks by forward substitution, then block row-diagonals
//   T_{b+d,b} = -D_{b+d} sum_{j=b}^{b+d-1} L_{b+d,j} T_{j,b},  D_b = (I + L_bb)^-1.
// NT threads synchronised by `sy` (the worker); X is a [3][16][16] scratch.  Only
// the block-lower part of T is written.
template <int NT, class Sync>
__device__ __forceinline__ void solve_unit_lower(const Sync &sy, const float *L, float *T, float *X, int tid) {
    if (tid < 64) {   // diagonal blocks: thread (b, c) owns column c of D_b
        const int b = tid >> 4, cc = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < r; ++j) acc = fmaf(-L[(o + r) * 64 + o + j], x[j], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T[(o + r) * 64 + o + cc] = x[r];
    }
    sy.sync();
    // d = 1: X_b = L_{b+1,b} D_b, then T_{b+1,b} = -D_{b+1} X_b   (b = 0, 1, 2)
    for (int e = tid; e < 3 * 256; e += NT) {
        const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15;
        X[e] = blk16(L, 16 * (b + 1), 16 * b, T, 16 * b, 16 * b, r, cc, 0.f);
    }
    sy.sync();
    for (int e = tid; e < 3 * 256; e += NT) {
        const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(T[(16 * (b + 1) + r) * 64 + 16 * (b + 1) + k], X[(b << 8) + k * 16 + cc], acc);
        T[(16 * (b + 1) + r) * 64 + 16 * b + cc] = -acc;
    }
    sy.sync();
    // d = 2: X_b = L_{b+2,b} D_b + L_{b+2,b+1} T_{b+1,b}, then T_{b+2,b} = -D_{b+2} X_b   (b = 0, 1)
    for (int e = tid; e < 2 * 256; e += NT) {
        const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15;
        float acc = blk16(L, 16 * (b + 2), 16 * b, T, 16 * b, 16 * b, r, cc, 0.f);
        X[e] = blk16(L, 16 * (b + 2), 16 * (b + 1), T, 16 * (b + 1), 16 * b, r, cc, acc);
    }
    sy.sync();
    for (int e = tid; e < 2 * 256; e += NT) {
        const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(T[(16 * (b + 2) + r) * 64 + 16 * (b + 2) + k], X[(b << 8) + k * 16 + cc], acc);
        T[(16 * (b + 2) + r) * 64 + 16 * b + cc] = -acc;
    }
    sy.sync();
    // d = 3: X = L_30 D_0 + L_31 T_10 + L_32 T_20, then T_30 = -D_3 X
    for (int e = tid; e < 256; e += NT) {
        const int r = e >> 4, cc = e & 15;
        float acc = blk16(L, 48, 0, T, 0, 0, r, cc, 0.f);
        acc = blk16(L, 48, 16, T, 16, 0, r, cc, acc);
        X[e] = blk16(L, 48, 32, T, 32, 0, r, cc, acc);
    }
    sy.sync();
    for (int e = tid; e < 256; e += NT) {
        const int r = e >> 4, cc = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(T[(48 + r) * 64 + 48 + k], X[k * 16 + cc], acc);
        T[(48 + r) * 64 + cc] = -acc;
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
    float *sL = reinterpret_cast<float *>(sm + OFF_LO);          // aliases [Ql;Kl] after the q.k MMA
    float *sTf = sL + 64 * 64;                                   // fp32 T, same region
    float *sX = reinterpret_cast<float *>(sm + OFF_MISC + 1024); // [3][16][16]
    float *sG = reinterpret_cast<float *>(sm + OFF_MISC);        // 64
    float *sBeta = sG + 64;                                      // 64
    float *sTot = sBeta + 64;                                    // 1
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
    // the token's gate logits (thread tid < len), loaded first so that their latency
    // passes while the convolutions run
    bf16 a_raw = __float2bfloat16(0.f), b_raw = __float2bfloat16(0.f);
    if (tid < len) {
        const size_t gi = (size_t)(t0 + tid) * H + h;
        a_raw = a_logit[gi];
        b_raw = b_logit[gi];
    }
    // ---- 1. prelude: q, k -> L2-normalised fp32 -> hi/lo fp16 tiles; v -> fp16 tile
    // (conv weights re-read per chunk from L1/L2 to keep them out of the solve's registers)
    {
        float2 w[4][4];
        load_conv_w(conv_w, qk_chan, w);
        const int oc = qk_oct & 15;
        uint8_t *hb = sHI + (oc / 8) * 16384, *lb = sLO + (oc / 8) * 16384;
        // the warp's 8 tokens in two halves of 4 (a 7-row window each; the halo rows
        // are re-read from L1), which keeps the prelude's registers in bounds
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            float2 y[4][4];
            conv_silu<4>(is_k ? k : q, (size_t)H * DK, qk_col, w, t0, s_begin, 8 * warp + 4 * hf, len, y);
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
                const float r = rsqrtf(ss[ii] + kNormEps);
                const float2 rr = make_float2(r, r);
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 x = fmul2(y[ii][p], rr);
                    const __half2 hh = __floats2half2_rn(x.x, x.y);
                    const float2 hf2 = __half22float2(hh);
                    const __half2 ll = __floats2half2_rn(x.x - hf2.x, x.y - hf2.y);
                    hw[p] = *reinterpret_cast<const uint32_t *>(&hh);
                    lw[p] = *reinterpret_cast<const uint32_t *>(&ll);
                }
                const int row = (is_k ? 64 : 0) + 8 * warp + 4 * hf + ii;
                umma::st_chunk(hb, row, oc % 8, make_uint4(hw[0], hw[1], hw[2], hw[3]));
                umma::st_chunk(lb, row, oc % 8, make_uint4(lw[0], lw[1], lw[2], lw[3]));
            }
        }
    }
    {
        float2 w[4][4];
        load_conv_w(conv_w, v_chan, w);
        constexpr int NV = C / VPARTS;
        float2 y[NV][4];
        conv_silu<NV>(v, (size_t)H * DV, v_col, w, t0, s_begin, NV * v_part, len, y);
#pragma unroll
        for (int ii = 0; ii < NV; ++ii)
            umma::st_chunk(sV + (v_oct / 8) * 8192, NV * v_part + ii, v_oct % 8,
                           make_uint4(umma::pack_half2(y[ii][0].x, y[ii][0].y), umma::pack_half2(y[ii][1].x, y[ii][1].y),
                                      umma::pack_half2(y[ii][2].x, y[ii][2].y), umma::pack_half2(y[ii][3].x, y[ii][3].y)));
    }
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
        if (tid == 31) *sTot = g;
        sBeta[tid] = be;
        sG[tid] = g;
    }
    sy.sync();
    if (tid >= 32 && tid < C) sG[tid] += *sTot;
    umma::fence_proxy_async_smem();
    sy.sync();
    if (publish && tid == 0) {   // the previous chunk's writes precede this worker's barriers
        __threadfence();
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(publish), "r"(1) : "memory");
    }

    // ---- 2. [Q;K] K^T = [Qh;Kh]Kh^T + [Qh;Kh]Kl^T + [Ql;Kl]Kh^T -> TMEM [0, 64)
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
    // while the MMA runs: Qt = e^{G_i} q_i, Kt = e^{G_C - G_i} k_i (fp16) and e^{G_C}
    {
        const float GC = sG[C - 1];
        for (int idx = tid; idx < len * (DK / 8); idx += NT) {
            const int i = idx / (DK / 8), ch = idx % (DK / 8);
            const float sq = __expf(sG[i]), sk = __expf(GC - sG[i]);
            const uint4 qv = *reinterpret_cast<const uint4 *>(sHI + (ch / 8) * 16384 + umma::sw128_offset(i, ch % 8));
            const uint4 kv = *reinterpret_cast<const uint4 *>(sHI + (ch / 8) * 16384 + umma::sw128_offset(64 + i, ch % 8));
            const __half2 *q2 = reinterpret_cast<const __half2 *>(&qv);
            const __half2 *k2 = reinterpret_cast<const __half2 *>(&kv);
            uint4 qo, ko;
            uint32_t *qo32 = reinterpret_cast<uint32_t *>(&qo), *ko32 = reinterpret_cast<uint32_t *>(&ko);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 qf = __half22float2(q2[e]), kf = __half22float2(k2[e]);
                qo32[e] = umma::pack_half2(qf.x * sq, qf.y * sq);
                ko32[e] = umma::pack_half2(kf.x * sk, kf.y * sk);
            }
            const size_t g = ((size_t)(t0 + i) * H + h) * DK + ch * 8;
            *reinterpret_cast<uint4 *>(Qt + g) = qo;
            *reinterpret_cast<uint4 *>(Kt + g) = ko;
        }
        if (tid == 0) decay[(size_t)t0 * H + h] = __expf(GC);
    }
    ok = prep_wait(sy, bar, phase, kPrepMaxPolls, tid);
    phase ^= 1;
    umma::tc_fence_after();
    if (!ok) return false;

    // ---- 3. rows 0..63: Aqk (masked, decayed q.k) -> global; rows 64..127: L -> smem
    //         warp w reads lane quadrant w % 4, columns [32 (w / 4), + 32)
    {
        float v[32];
        const int j0 = 32 * (warp >> 2);
        umma::tmem_ld32(trow + j0, v);
        const int i = (32 * (warp & 3) + lane) & 63;
        const float Gi = sG[i];
        if ((warp & 3) < 2) {
            if (i < len) {
                uint4 *dst = reinterpret_cast<uint4 *>(Aqk + ((size_t)(t0 + i) * H + h) * C + j0);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = j0 + q8 * 8 + e;
                        x[e] = (j <= i) ? v[q8 * 8 + e] * __expf(Gi - sG[j]) : 0.f;
                    }
                    dst[q8] = make_uint4(umma::pack_half2(x[0], x[1]), umma::pack_half2(x[2], x[3]),
                                         umma::pack_half2(x[4], x[5]), umma::pack_half2(x[6], x[7]));
                }
            }
        } else {
            const float bi = sBeta[i];
            float4 *dst = reinterpret_cast<float4 *>(sL + i * C + j0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                float x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + q4 * 4 + e;
                    x[e] = (j < i) ? bi * v[q4 * 4 + e] * __expf(Gi - sG[j]) : 0.f;
                }
                dst[q4] = make_float4(x[0], x[1], x[2], x[3]);
            }
        }
    }
    umma::tc_fence_before();
    sy.sync();

    // ---- 4. T = (I + L)^-1 (fp32, blocked); then T' = T diag(beta e^G) in rows
    //         0..63 and T'' = T diag(beta) in rows 64..127 of an fp16 K-major tile
    solve_unit_lower<NT>(sy, sL, sTf, sX, tid);
    for (int idx = tid; idx < C * 8; idx += NT) {
        const int i = idx >> 3, ch = idx & 7;
        const float4 *tr = reinterpret_cast<const float4 *>(sTf + i * C + ch * 8);
        const float4 t0v = tr[0], t1v = tr[1];
        const float tv[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
        float a1[8], a2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = ch * 8 + e;
            // only the block-lower part of T was written: zero the rest
            const float t = ((j >> 4) <= (i >> 4)) ? tv[e] : 0.f;
            const float bj = sBeta[j];
            a1[e] = t * bj * __expf(sG[j]);
            a2[e] = t * bj;
        }
        umma::st_chunk(sT, i, ch, make_uint4(umma::pack_half2(a1[0], a1[1]), umma::pack_half2(a1[2], a1[3]),
                                             umma::pack_half2(a1[4], a1[5]), umma::pack_half2(a1[6], a1[7])));
        umma::st_chunk(sT, 64 + i, ch, make_uint4(umma::pack_half2(a2[0], a2[1]), umma::pack_half2(a2[2], a2[3]),
                                                  umma::pack_half2(a2[4], a2[5]), umma::pack_half2(a2[6], a2[7])));
    }
    umma::fence_proxy_async_smem();
    sy.sync();

    // ---- 5. W-part = T' K -> TMEM [0, DK);  U'-part = T'' V -> TMEM [DK, DK + DV)
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

    // ---- 6. rows 0..63 of the W-part -> -W; rows 64..127 of the U'-part -> U'
    //         (warp w: lane quadrant w % 4, column half w / 4; TMEM loads are
    //         warp-collective: every lane loads, valid rows store)
    {
        const int i = (32 * (warp & 3) + lane) & 63;
        const int half = warp >> 2;
        if ((warp & 3) < 2) {
            __half *dst = Wn + ((size_t)(t0 + i) * H + h) * DK;
#pragma unroll
            for (int c0 = half * (DK / 2); c0 < (half + 1) * (DK / 2); c0 += 32) {
                float vv[32];
                umma::tmem_ld32(trow + c0, vv);
                if (i < len) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        reinterpret_cast<uint4 *>(dst + c0)[q8] = make_uint4(
                            umma::pack_half2(-vv[q8 * 8 + 0], -vv[q8 * 8 + 1]), umma::pack_half2(-vv[q8 * 8 + 2], -vv[q8 * 8 + 3]),
                            umma::pack_half2(-vv[q8 * 8 + 4], -vv[q8 * 8 + 5]), umma::pack_half2(-vv[q8 * 8 + 6], -vv[q8 * 8 + 7]));
                }
            }
        } else {
            __half *dst = Up + ((size_t)(t0 + i) * H + h) * DV;
#pragma unroll
            for (int c0 = half * (DV / 2); c0 < (half + 1) * (DV / 2); c0 += 32) {
                float vv[32];
                umma::tmem_ld32(trow + DK + c0, vv);
                if (i < len) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        reinterpret_cast<uint4 *>(dst + c0)[q8] = make_uint4(
                            umma::pack_half2(vv[q8 * 8 + 0], vv[q8 * 8 + 1]), umma::pack_half2(vv[q8 * 8 + 2], vv[q8 * 8 + 3]),
                            umma::pack_half2(vv[q8 * 8 + 4], vv[q8 * 8 + 5]), umma::pack_half2(vv[q8 * 8 + 6], vv[q8 * 8 + 7]));
                }
            }
        }
    }
    umma::tc_fence_before();
    sy.sync();
    return true;
}

}  // namespace gdn

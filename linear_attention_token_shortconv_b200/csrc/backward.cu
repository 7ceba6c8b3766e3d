// K4 -- the prefill backward (fp32 inputs, d_k = d_v = D in {64, 128}): gradients
// of <d_out, out> + <d_S_final, S_final> with respect to every prefill input.
//
// Reverse-mode derivative of the forward of the same write-ups (slinene.github.io
// write-up of "On the Design of Qwen3.8-Next Architecture", 模块 A: 递归状态 and
// 参数化; paper.rainbus.top digest, 方法步骤详情 step (1)).  Per token, with P the
// state before it, e = v - alpha P^T k, S = alpha P + beta k e^T, y = S^T q, the
// output o = sigmoid(z) y r (1 + w), r = (mean y^2 + eps)^{-1/2}, and D the
// gradient of S:
//   dy = r dn - r^3 y mean(dn y),  dn = do sigmoid(z) (1 + w);
//   D += q dy^T;  dq = alpha P dy + beta (e . dy) k;
//   de = beta D^T k = dv;  dk = beta D e - alpha P de;  dbeta = k^T D e;
//   dalpha = <D, P> - k^T P de;  dg = alpha dalpha (g = log alpha);
//   gradient of P = alpha (D - k de^T).
// Then the gates (g = -e^A softplus(a + b_alpha), beta = sigmoid(b)), L2Norm,
// SiLU and the short convolution in reverse.
//
// Kernels (one launch each):
//  (prelude)  q_hat, k_hat, v_hat in fp32: the forward's fp32 prelude kernel.
//  K4a bwd_ckpt_kernel: the forward recurrence of one (sequence, head) per CTA,
//      storing the state before every 16-token interval (checkpoints).
//  K4b bwd_recurrence_kernel: one (sequence, head) per CTA, intervals in reverse.
//      Per interval: the checkpoint is loaded and the interval run forward once,
//      each state before a token going to a per-CTA scratch (16 x 64 KB, which
//      stays in L2) with the token's e and y; the output-stage backward of the 16
//      tokens (one warp per two tokens); then the token steps in reverse, the
//      state gradient held in registers.  The state is laid out as in the decode
//      kernel: thread (warp w, lane l) holds rows w + 8 r and columns
//      (D / 32) l + m.  Column sums go through shared memory across the 8 warps;
//      row sums are a reduce-scatter across the 32 lanes of a warp.
//  K4c bwd_prelude_kernel: L2Norm, SiLU and conv backward per channel octet and
//      64-token tile: d_q, d_k, d_v and per-tile partial sums of d_conv_w.
//  K4d bwd_gates_kernel: d_a_logit, d_b_logit, and d_A, d_b_alpha per head.
//  K4e bwd_reduce_kernel: the partial sums of d_conv_w and d_norm_w.
// Every partial sum has a fixed order: the results do not depend on scheduling.
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace bwd {
constexpr int NT = 256;
constexpr int IV = 16;   // tokens per checkpoint interval
constexpr int PT = 64;   // tokens per prelude-backward tile
}  // namespace bwd

__device__ __forceinline__ void bwd_seq_bounds(const int32_t *cu, int n_seq, int n_tok, int n, int &s0, int &s1) {
    if (cu) {
        s0 = __ldg(cu + n);
        s1 = __ldg(cu + n + 1);
    } else {
        const int L = n_tok / n_seq;
        s0 = n * L;
        s1 = s0 + L;
    }
}

// Checkpoint slot of interval 0 of sequence n: the sequence uses ceil(len / 16)
// consecutive slots from floor(start / 16) + n, which never reaches the next
// sequence's first slot; floor(N_tok / 16) + N_seq slots in all.
__device__ __forceinline__ size_t ckpt_base(int s0, int n) { return (size_t)(s0 / bwd::IV) + n; }

__device__ __forceinline__ void bwd_gates(float a_l, float b_l, float A, float ba, float &al, float &be) {
    al = expf(log_decay(a_l, A, ba));
    be = sigmoid_acc(b_l);
}

// Reduce-scatter of N values across the 32 lanes of a warp (N a multiple of 32):
// afterwards v[i], i < N / 32, of lane l holds the warp-wide sum of entry
// (N / 32) l + i.  Each round halves the array: a lane keeps the half selected by
// its lane bit and adds the partner lane's copy of that half.
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
#pragma unroll
    for (int rd = 0; rd < 5; ++rd) {
        const int o = 16 >> rd;
        const bool up = (lane & o) != 0;
        const int half = N >> (rd + 1);
#pragma unroll
        for (int i = 0; i < (N >> 1); ++i) {
            if (i < half) {
                const float send = up ? v[i] : v[i + half];
                const float keep = up ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
    }
}

// ---------------------------------------------------------------- K4a: checkpoints
template <int D>
__global__ void __launch_bounds__(bwd::NT, 1)
bwd_ckpt_kernel(const float *__restrict__ kn, const float *__restrict__ vn, const float *__restrict__ a_logit,
                const float *__restrict__ b_logit, const float *__restrict__ A, const float *__restrict__ b_alpha,
                const float *__restrict__ S0, const int32_t *__restrict__ cu, int n_seq, int n_tok, int H,
                float *__restrict__ ckpt) {
    constexpr int RPT = D / 8, CPT = D / 32, IV = bwd::IV;
    __shared__ float kk[IV][D], vv[IV][D], al[IV], be[IV];
    __shared__ float red[2][8][D];
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int s0, s1;
    bwd_seq_bounds(cu, n_seq, n_tok, n, s0, s1);
    float S[RPT][CPT];
    const float *S0h = S0 ? S0 + ((size_t)n * H + h) * D * D : nullptr;
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int m = 0; m < CPT; ++m) S[r][m] = S0h ? S0h[(warp + 8 * r) * D + CPT * lane + m] : 0.f;
    const size_t base = ckpt_base(s0, n);
    const float Ah = __ldg(A + h), bah = __ldg(b_alpha + h);
    for (int t0 = s0, I = 0; t0 < s1; t0 += IV, ++I) {
        const int cnt = min(IV, s1 - t0);
        float *ck = ckpt + ((base + I) * H + h) * (size_t)D * D;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int m = 0; m < CPT; ++m) ck[(warp + 8 * r) * D + CPT * lane + m] = S[r][m];
        __syncthreads();   // the previous interval's reads of the tile are done
        for (int idx = tid; idx < cnt * D; idx += bwd::NT) {
            const int t = idx / D, i = idx % D;
            const size_t g = ((size_t)(t0 + t) * H + h) * D + i;
            kk[t][i] = kn[g];
            vv[t][i] = vn[g];
        }
        if (tid < cnt) {
            const size_t gi = (size_t)(t0 + tid) * H + h;
            bwd_gates(a_logit[gi], b_logit[gi], Ah, bah, al[tid], be[tid]);
        }
        __syncthreads();
        for (int t = 0; t < cnt; ++t) {
            float p[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) p[m] = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kr = kk[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) p[m] = fmaf(S[r][m], kr, p[m]);
            }
#pragma unroll
            for (int m = 0; m < CPT; ++m) red[t & 1][warp][CPT * lane + m] = p[m];
            __syncthreads();
            float e[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) s += red[t & 1][w][CPT * lane + m];
                e[m] = vv[t][CPT * lane + m] - al[t] * s;
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float bk = be[t] * kk[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) S[r][m] = fmaf(bk, e[m], al[t] * S[r][m]);
            }
        }
    }
}

// ------------------------------------------------------------- K4b: recurrence
namespace bwd {
template <int D> struct RecLayout {
    // floats: q, k, v, e, y, dy [IV][D]; red [2][2][8][D]; rowsum [2][3][D];
    // alpha, beta, k.q, e.dy [IV]; per-token scalar partials [IV][8][3]
    static constexpr int TILE = IV * D;
    static constexpr int OFF_RED = 6 * TILE;
    static constexpr int OFF_ROW = OFF_RED + 2 * 2 * 8 * D;
    static constexpr int OFF_SMALL = OFF_ROW + 2 * 3 * D;
    static constexpr int OFF_SC = OFF_SMALL + 4 * IV;
    static constexpr int FLOATS = OFF_SC + IV * 8 * 3;
    static constexpr int BYTES = FLOATS * 4;
};
}  // namespace bwd

template <int D>
__global__ void __launch_bounds__(bwd::NT, 1)
bwd_recurrence_kernel(const float *__restrict__ qn, const float *__restrict__ kn, const float *__restrict__ vn,
                      const float *__restrict__ a_logit, const float *__restrict__ b_logit,
                      const float *__restrict__ A, const float *__restrict__ b_alpha, const float *__restrict__ z,
                      const float *__restrict__ norm_w, const float *__restrict__ d_out,
                      const float *__restrict__ d_S_final, const int32_t *__restrict__ cu, int n_seq, int n_tok,
                      int H, const float *__restrict__ ckpt, float *__restrict__ scratch, float *__restrict__ dqn,
                      float *__restrict__ dkn, float *__restrict__ dvn, float *__restrict__ dg,
                      float *__restrict__ dbeta, float *__restrict__ d_z, float *__restrict__ dnorm_part,
                      float *__restrict__ d_S0) {
    using L = bwd::RecLayout<D>;
    constexpr int RPT = D / 8, CPT = D / 32, IV = bwd::IV;
    constexpr int NV = (3 * RPT + 31) / 32 * 32;   // row sums per thread, padded for the reduce-scatter
    extern __shared__ float smf[];
    float(*qq)[D] = reinterpret_cast<float(*)[D]>(smf);
    float(*kk)[D] = qq + IV;
    float(*vv)[D] = kk + IV;
    float(*ee)[D] = vv + IV;
    float(*yy)[D] = ee + IV;
    float(*dyy)[D] = yy + IV;
    float *red = smf + L::OFF_RED;      // [parity][quantity][warp][D]
    float *rowsum = smf + L::OFF_ROW;   // [parity][A, B, C][D]
    float *al = smf + L::OFF_SMALL, *be = al + IV, *kq = be + IV, *edy = kq + IV;
    float *sc = smf + L::OFF_SC;        // [token][warp][<D,P>, k.(D e), k.(P de)]

    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int s0, s1;
    bwd_seq_bounds(cu, n_seq, n_tok, n, s0, s1);
    const int nI = (s1 - s0 + IV - 1) / IV;
    const size_t base = ckpt_base(s0, n);
    const float Ah = __ldg(A + h), bah = __ldg(b_alpha + h);
    float *scr = scratch + ((size_t)n * H + h) * IV * D * D;
    float gain[CPT], dwacc[CPT];
#pragma unroll
    for (int m = 0; m < CPT; ++m) {
        gain[m] = 1.0f + __ldg(norm_w + CPT * lane + m);
        dwacc[m] = 0.f;
    }
    // the gradient of the state after the current token
    float Dg[RPT][CPT];
    const float *dSf = d_S_final ? d_S_final + ((size_t)n * H + h) * D * D : nullptr;
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int m = 0; m < CPT; ++m) Dg[r][m] = dSf ? dSf[(warp + 8 * r) * D + CPT * lane + m] : 0.f;

    for (int I = nI - 1; I >= 0; --I) {
        const int t0 = s0 + I * IV, cnt = min(IV, s1 - t0);
        auto finish_rows = [&](int t, int par) {   // threads tid < D: row tid of token t
            const int i = tid;
            const float Ai = rowsum[(par * 3 + 0) * D + i], Bi = rowsum[(par * 3 + 1) * D + i];
            const float Ci = rowsum[(par * 3 + 2) * D + i], ki = kk[t][i];
            const size_t g = ((size_t)(t0 + t) * H + h) * D + i;
            dqn[g] = fmaf(al[t], Ai, be[t] * edy[t] * ki);
            dkn[g] = fmaf(be[t], Ci, -al[t] * Bi);
            const float kc = group_sum<32>(ki * Ci), kb = group_sum<32>(ki * Bi);
            if (lane == 0) {
                sc[(t * 8 + warp) * 3 + 1] = kc;
                sc[(t * 8 + warp) * 3 + 2] = kb;
            }
        };
        // (a) the state before the interval
        float S[RPT][CPT];
        {
            const float *ck = ckpt + ((base + I) * H + h) * (size_t)D * D;
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int m = 0; m < CPT; ++m) S[r][m] = ck[(warp + 8 * r) * D + CPT * lane + m];
        }
        __syncthreads();   // the previous interval's shared-memory reads are done
        // (b) the interval's q, k, v, gates and k.q: warp w stages tokens 2w, 2w + 1
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int t = 2 * warp + u;
            if (t < cnt) {
                const size_t row = ((size_t)(t0 + t) * H + h) * D;
                float dot = 0.f;
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    const int j = CPT * lane + m;
                    const float qv = qn[row + j], kv = kn[row + j];
                    qq[t][j] = qv;
                    kk[t][j] = kv;
                    vv[t][j] = vn[row + j];
                    dot = fmaf(qv, kv, dot);
                }
                dot = group_sum<32>(dot);
                if (lane == 0) {
                    kq[t] = dot;
                    const size_t gi = (size_t)(t0 + t) * H + h;
                    bwd_gates(a_logit[gi], b_logit[gi], Ah, bah, al[t], be[t]);
                }
            }
        }
        for (int idx = tid; idx < IV * 8 * 3; idx += bwd::NT) sc[idx] = 0.f;
        __syncthreads();
        // (c) forward over the interval: the state before each token to the scratch;
        //     e and y of each token
        for (int t = 0; t < cnt; ++t) {
            float *st = scr + (size_t)t * D * D;
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int m = 0; m < CPT; ++m) st[(warp + 8 * r) * D + CPT * lane + m] = S[r][m];
            float p[CPT], pq[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) p[m] = pq[m] = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kr = kk[t][warp + 8 * r], qr = qq[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    p[m] = fmaf(S[r][m], kr, p[m]);
                    pq[m] = fmaf(S[r][m], qr, pq[m]);
                }
            }
            float *rd = red + (t & 1) * 2 * 8 * D;
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                rd[warp * D + CPT * lane + m] = p[m];
                rd[8 * D + warp * D + CPT * lane + m] = pq[m];
            }
            __syncthreads();
            float e[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                const int j = CPT * lane + m;
                float s = 0.f, sq = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    s += rd[w * D + j];
                    sq += rd[8 * D + w * D + j];
                }
                e[m] = vv[t][j] - al[t] * s;
                if (warp == 0) {
                    ee[t][j] = e[m];
                    yy[t][j] = fmaf(al[t], sq, be[t] * kq[t] * e[m]);
                }
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float bk = be[t] * kk[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) S[r][m] = fmaf(bk, e[m], al[t] * S[r][m]);
            }
        }
        __syncthreads();   // e and y of the interval are complete
        // (c') output-stage backward: warp w takes tokens 2w, 2w + 1
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int t = 2 * warp + u;
            if (t < cnt) {
                const size_t row = ((size_t)(t0 + t) * H + h) * D;
                float yv[CPT], sz[CPT], dov[CPT], dn[CPT], ssq = 0.f, dny = 0.f;
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    const int j = CPT * lane + m;
                    yv[m] = yy[t][j];
                    sz[m] = sigmoid_acc(z[row + j]);
                    dov[m] = d_out[row + j];
                    ssq = fmaf(yv[m], yv[m], ssq);
                    dn[m] = dov[m] * sz[m] * gain[m];
                    dny = fmaf(dn[m], yv[m], dny);
                }
                ssq = group_sum<32>(ssq);
                dny = group_sum<32>(dny);
                const float r = 1.0f / sqrtf(ssq / D + kNormEps);
                float edot = 0.f;
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    const int j = CPT * lane + m;
                    const float nj = yv[m] * r;
                    d_z[row + j] = dov[m] * nj * gain[m] * sz[m] * (1.0f - sz[m]);
                    dwacc[m] = fmaf(dov[m] * sz[m], nj, dwacc[m]);
                    const float dyv = r * dn[m] - r * r * r * yv[m] * (dny / D);
                    dyy[t][j] = dyv;
                    edot = fmaf(ee[t][j], dyv, edot);
                }
                edot = group_sum<32>(edot);
                if (lane == 0) edy[t] = edot;
            }
        }
        __syncthreads();
        // (d) token steps in reverse
        for (int t = cnt - 1; t >= 0; --t) {
            const int par = t & 1;
            const float *st = scr + (size_t)t * D * D;
            float P[RPT][CPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int m = 0; m < CPT; ++m) P[r][m] = st[(warp + 8 * r) * D + CPT * lane + m];
            float dyl[CPT], el[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                dyl[m] = dyy[t][CPT * lane + m];
                el[m] = ee[t][CPT * lane + m];
            }
            // D += q dy^T, then the column partials of D^T k
            float dp[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) dp[m] = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float qr = qq[t][warp + 8 * r], kr = kk[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    Dg[r][m] = fmaf(qr, dyl[m], Dg[r][m]);
                    dp[m] = fmaf(Dg[r][m], kr, dp[m]);
                }
            }
            float *rd = red + par * 2 * 8 * D;
#pragma unroll
            for (int m = 0; m < CPT; ++m) rd[warp * D + CPT * lane + m] = dp[m];
            __syncthreads();
            // the rows of token t + 1 (their sums were completed before this barrier)
            if (t + 1 < cnt && tid < D) finish_rows(t + 1, par ^ 1);
            float de[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) s += rd[w * D + CPT * lane + m];
                de[m] = be[t] * s;
            }
            if (warp == 0) {
#pragma unroll
                for (int m = 0; m < CPT; ++m) dvn[((size_t)(t0 + t) * H + h) * D + CPT * lane + m] = de[m];
            }
            // row sums: A = P dy, B = P de, C = D e; and <D, P>
            float v[NV];
            float dDP = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                float a_ = 0.f, b_ = 0.f, c_ = 0.f;
#pragma unroll
                for (int m = 0; m < CPT; ++m) {
                    a_ = fmaf(P[r][m], dyl[m], a_);
                    b_ = fmaf(P[r][m], de[m], b_);
                    c_ = fmaf(Dg[r][m], el[m], c_);
                    dDP = fmaf(Dg[r][m], P[r][m], dDP);
                }
                v[r] = a_;
                v[RPT + r] = b_;
                v[2 * RPT + r] = c_;
            }
#pragma unroll
            for (int x = 3 * RPT; x < NV; ++x) v[x] = 0.f;
            warp_reduce_scatter<NV>(v, lane);
#pragma unroll
            for (int i = 0; i < NV / 32; ++i) {
                const int idx = (NV / 32) * lane + i;
                if (idx < 3 * RPT) rowsum[(par * 3 + idx / RPT) * D + warp + 8 * (idx % RPT)] = v[i];
            }
            dDP = group_sum<32>(dDP);
            if (lane == 0) sc[(t * 8 + warp) * 3 + 0] = dDP;
            // the gradient of the state before token t
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kr = kk[t][warp + 8 * r];
#pragma unroll
                for (int m = 0; m < CPT; ++m) Dg[r][m] = al[t] * fmaf(-kr, de[m], Dg[r][m]);
            }
        }
        __syncthreads();
        if (cnt > 0 && tid < D) finish_rows(0, 0);
        __syncthreads();
        if (tid < cnt) {
            float dp_ = 0.f, kc = 0.f, kb = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                dp_ += sc[(tid * 8 + w) * 3 + 0];
                kc += sc[(tid * 8 + w) * 3 + 1];
                kb += sc[(tid * 8 + w) * 3 + 2];
            }
            const size_t gi = (size_t)(t0 + tid) * H + h;
            dbeta[gi] = kc;
            dg[gi] = al[tid] * (dp_ - kb);
        }
    }
    if (d_S0) {
        float *o = d_S0 + ((size_t)n * H + h) * D * D;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int m = 0; m < CPT; ++m) o[(warp + 8 * r) * D + CPT * lane + m] = Dg[r][m];
    }
    // the norm-weight partial of this (sequence, head): sum of the 8 warps
    __syncthreads();
#pragma unroll
    for (int m = 0; m < CPT; ++m) red[warp * D + CPT * lane + m] = dwacc[m];
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w * D + tid];
        dnorm_part[((size_t)n * H + h) * D + tid] = s;
    }
}

// ------------------------------------------------------------ K4c: prelude backward
// One thread owns 8 consecutive conv channels (of q, k or v of one head) and a
// 64-token tile.  It walks tokens t0 .. t1 + 2 (the conv looks 3 tokens back, so
// its transpose looks 3 ahead), recomputing x = conv(raw), u = SiLU(x) and, for q
// and k, the L2Norm factor (a sum over the head's D / 8 lanes), and turns the
// gradient of the prelude output into the gradient of x; that gradient is
// spread over the raw rows t - 3 .. t (inside t's sequence) through a 4-row
// ring, and row t - 3 is final once t is done.
template <int D>
__global__ void __launch_bounds__(bwd::NT)
bwd_prelude_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                   const float *__restrict__ conv_w, const float *__restrict__ dqn, const float *__restrict__ dkn,
                   const float *__restrict__ dvn, const int32_t *__restrict__ cu, int n_seq, int n_tok, int H,
                   float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                   float *__restrict__ dw_part) {
    constexpr int G = D / 8;   // lanes of one head's channels
    const int C = 3 * H * D;
    const int octets = C / 8;
    const int co = blockIdx.x * bwd::NT + threadIdx.x;
    const bool active = co < octets;
    const int c = active ? co * 8 : 0;
    const int kind = c < H * D ? 0 : (c < 2 * H * D ? 1 : 2);
    const int col = c - kind * H * D;
    const float *src = kind == 0 ? q : (kind == 1 ? k : v);
    const float *gsrc = kind == 0 ? dqn : (kind == 1 ? dkn : dvn);
    float *dst = kind == 0 ? dq : (kind == 1 ? dk : dv);
    const size_t row = (size_t)H * D;
    float w[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 t4 = active ? __ldg(reinterpret_cast<const float4 *>(conv_w) + (c + i))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        w[i][0] = t4.x; w[i][1] = t4.y; w[i][2] = t4.z; w[i][3] = t4.w;
    }
    const int t0 = blockIdx.y * bwd::PT, t1 = min(t0 + bwd::PT, n_tok);
    const int L = cu ? 0 : n_tok / n_seq;
    int n = cu ? seq_of_token(cu, n_seq, t0) : t0 / L;
    int s_start, s_end;
    bwd_seq_bounds(cu, n_seq, n_tok, n, s_start, s_end);
    // raw rows t - 3, t - 2, t - 1 (zero before the sequence start)
    float hr[3][8];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int tt = t0 - 3 + j;
#pragma unroll
        for (int i = 0; i < 8; ++i) hr[j][i] = 0.f;
        if (active && tt >= s_start && tt < n_tok)
#pragma unroll
            for (int i = 0; i < 8; ++i) hr[j][i] = src[(size_t)tt * row + col + i];
    }
    float ring[4][8];   // gradient of raw rows t - 3 .. t
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) ring[j][i] = 0.f;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int t = t0; t < t1 + 3; ++t) {
        const bool live = t < n_tok;
        if (live && t >= s_end) {   // a new sequence: its history starts empty
            while (t >= s_end) {
                ++n;
                bwd_seq_bounds(cu, n_seq, n_tok, n, s_start, s_end);
            }
#pragma unroll
            for (int j = 0; j < 3; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) hr[j][i] = 0.f;
        }
        float cur[8], dx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = dx[i] = 0.f;
        if (live) {
            float x[8], u[8], g[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cur[i] = active ? src[(size_t)t * row + col + i] : 0.f;
                g[i] = active ? gsrc[(size_t)t * row + col + i] : 0.f;
                float a = w[i][0] * hr[0][i];
                a = fmaf(w[i][1], hr[1][i], a);
                a = fmaf(w[i][2], hr[2][i], a);
                a = fmaf(w[i][3], cur[i], a);
                x[i] = a;
                u[i] = a * sigmoid_acc(a);
            }
            // L2Norm backward over the head's D channels (q, k).  The group sums run
            // in every lane: a warp may hold channels of two tensors, and the
            // shuffles need the whole warp; v lanes ignore the result.
            float ss = 0.f, ug = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ss = fmaf(u[i], u[i], ss);
                ug = fmaf(u[i], g[i], ug);
            }
            ss = group_sum<G>(ss);
            ug = group_sum<G>(ug);
            if (kind < 2) {
                const float rho = 1.0f / sqrtf(ss + kNormEps);
#pragma unroll
                for (int i = 0; i < 8; ++i) g[i] = rho * g[i] - rho * rho * rho * u[i] * ug;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float s = sigmoid_acc(x[i]);
                dx[i] = g[i] * s * (1.0f + x[i] * (1.0f - s));
            }
            if (t < t1) {   // conv-weight gradient: this tile's tokens only
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    acc[i][0] = fmaf(dx[i], hr[0][i], acc[i][0]);
                    acc[i][1] = fmaf(dx[i], hr[1][i], acc[i][1]);
                    acc[i][2] = fmaf(dx[i], hr[2][i], acc[i][2]);
                    acc[i][3] = fmaf(dx[i], cur[i], acc[i][3]);
                }
            }
            // raw row t - 3 + j receives w_j dx (rows of t's sequence only)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (t - 3 + j >= s_start) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) ring[j][i] = fmaf(w[i][j], dx[i], ring[j][i]);
                }
            }
        }
        // row t - 3 is complete
        if (active && t - 3 >= t0 && t - 3 < t1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[(size_t)(t - 3) * row + col + i] = ring[0][i];
        }
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) ring[j][i] = ring[j + 1][i];
#pragma unroll
        for (int i = 0; i < 8; ++i) ring[3][i] = 0.f;
        if (live) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                hr[0][i] = hr[1][i];
                hr[1][i] = hr[2][i];
                hr[2][i] = cur[i];
            }
        }
    }
    if (active) {
        float *o = dw_part + ((size_t)blockIdx.y * C + c) * 4;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4 *>(o + i * 4) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

// --------------------------------------------------------------- K4d: gates
__global__ void __launch_bounds__(bwd::NT)
bwd_gates_kernel(const float *__restrict__ a_logit, const float *__restrict__ b_logit,
                 const float *__restrict__ A, const float *__restrict__ b_alpha, const float *__restrict__ dg,
                 const float *__restrict__ dbeta, int n_tok, int H, float *__restrict__ d_a,
                 float *__restrict__ d_b, float *__restrict__ d_A, float *__restrict__ d_b_alpha) {
    __shared__ float part[2][bwd::NT / 32];
    const int h = blockIdx.x, tid = threadIdx.x;
    const float eA = expf(__ldg(A + h)), ba = __ldg(b_alpha + h);
    float sA = 0.f, sba = 0.f;
    for (int t = tid; t < n_tok; t += bwd::NT) {
        const size_t gi = (size_t)t * H + h;
        const float ain = a_logit[gi] + ba;
        const float g = -eA * softplus_acc(ain);
        const float dgv = dg[gi];
        const float da = dgv * (-eA) * sigmoid_acc(ain);
        d_a[gi] = da;
        sA = fmaf(dgv, g, sA);
        sba += da;
        const float be = sigmoid_acc(b_logit[gi]);
        d_b[gi] = dbeta[gi] * be * (1.0f - be);
    }
    sA = group_sum<32>(sA);
    sba = group_sum<32>(sba);
    if ((tid & 31) == 0) {
        part[0][tid >> 5] = sA;
        part[1][tid >> 5] = sba;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < bwd::NT / 32; ++w) {
            a += part[0][w];
            b += part[1][w];
        }
        d_A[h] = a;
        d_b_alpha[h] = b;
    }
}

// --------------------------------------------------------------- K4e: reductions
__global__ void __launch_bounds__(bwd::NT)
bwd_reduce_kernel(const float *__restrict__ dw_part, int n_tiles, int C4, const float *__restrict__ dnorm_part,
                  int n_pairs, int D, float *__restrict__ d_conv_w, float *__restrict__ d_norm_w) {
    const int e = blockIdx.x * bwd::NT + threadIdx.x;
    if (e < C4) {
        float s = 0.f;
        for (int i = 0; i < n_tiles; ++i) s += dw_part[(size_t)i * C4 + e];
        d_conv_w[e] = s;
    } else if (e < C4 + D) {
        const int j = e - C4;
        float s = 0.f;
        for (int i = 0; i < n_pairs; ++i) s += dnorm_part[(size_t)i * D + j];
        d_norm_w[j] = s;
    }
}

// ---------------------------------------------------------------------- host
size_t backward_workspace_bytes(int n_seq, int n_tok, int H, int D) {
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nt = (size_t)n_tok * H;
    const size_t n_ckpt = (size_t)n_tok / bwd::IV + n_seq;
    const size_t n_tiles = ((size_t)n_tok + bwd::PT - 1) / bwd::PT;
    return 6 * ru(nt * D * 4) + 2 * ru(nt * 4) + ru(n_ckpt * H * D * D * 4) +
           ru((size_t)n_seq * H * bwd::IV * D * D * 4) + ru(n_tiles * 3 * H * D * 4 * 4) +
           ru((size_t)n_seq * H * D * 4);
}

cudaError_t launch_backward(const BackwardArgs &b, void *ws) {
    const int D = b.f.dk, n_seq = b.f.n_seq, n_tok = b.f.n_tok, H = b.f.H;
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nt = (size_t)n_tok * H;
    char *p = static_cast<char *>(ws);
    auto take = [&](size_t bytes) { char *r = p; p += ru(bytes); return reinterpret_cast<float *>(r); };
    float *qn = take(nt * D * 4), *kn = take(nt * D * 4), *vn = take(nt * D * 4);
    float *dqn = take(nt * D * 4), *dkn = take(nt * D * 4), *dvn = take(nt * D * 4);
    float *dgw = take(nt * 4), *dbw = take(nt * 4);
    const size_t n_ckpt = (size_t)n_tok / bwd::IV + n_seq;
    float *ckpt = take(n_ckpt * H * D * D * 4);
    float *scratch = take((size_t)n_seq * H * bwd::IV * D * D * 4);
    const int n_tiles = (n_tok + bwd::PT - 1) / bwd::PT;
    float *dw_part = take((size_t)n_tiles * 3 * H * D * 4 * 4);
    float *dnorm_part = take((size_t)n_seq * H * D * 4);
    cudaStream_t s = b.f.stream;
    const float *fq = static_cast<const float *>(b.f.q), *fk = static_cast<const float *>(b.f.k);
    const float *fv = static_cast<const float *>(b.f.v), *fz = static_cast<const float *>(b.f.z);
    const float *fa = static_cast<const float *>(b.f.a_logit), *fb = static_cast<const float *>(b.f.b_logit);
    cudaError_t e;
    if (n_tok > 0) {
        if ((e = launch_prelude_f32(b.f, qn, kn, vn)) != cudaSuccess) return e;
    }
    const dim3 pairs(H, n_seq);
#define GDN_BWD(D_)                                                                                          \
    do {                                                                                                     \
        if (n_tok > 0) {                                                                                     \
            bwd_ckpt_kernel<D_><<<pairs, bwd::NT, 0, s>>>(kn, vn, fa, fb, b.f.A, b.f.b_alpha, b.f.S0,        \
                                                          b.f.cu_seqlens, n_seq, n_tok, H, ckpt);           \
            if ((e = launched()) != cudaSuccess) return e;                                                   \
        }                                                                                                    \
        constexpr int SM_ = bwd::RecLayout<D_>::BYTES;                                                       \
        if ((e = cudaFuncSetAttribute(bwd_recurrence_kernel<D_>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                      SM_)) != cudaSuccess)                                                  \
            return e;                                                                                        \
        bwd_recurrence_kernel<D_><<<pairs, bwd::NT, SM_, s>>>(                                               \
            qn, kn, vn, fa, fb, b.f.A, b.f.b_alpha, fz, b.f.norm_w, static_cast<const float *>(b.d_out),     \
            b.d_S_final, b.f.cu_seqlens, n_seq, n_tok, H, ckpt, scratch, dqn, dkn, dvn, dgw, dbw,            \
            static_cast<float *>(b.d_z), dnorm_part, b.d_S0);                                                \
        if ((e = launched()) != cudaSuccess) return e;                                                       \
        if (n_tok > 0) {                                                                                     \
            const dim3 g((3 * H * D_ / 8 + bwd::NT - 1) / bwd::NT, n_tiles);                                 \
            bwd_prelude_kernel<D_><<<g, bwd::NT, 0, s>>>(fq, fk, fv, b.f.conv_w, dqn, dkn, dvn,              \
                                                         b.f.cu_seqlens, n_seq, n_tok, H,                    \
                                                         static_cast<float *>(b.dq), static_cast<float *>(b.dk), \
                                                         static_cast<float *>(b.dv), dw_part);               \
            if ((e = launched()) != cudaSuccess) return e;                                                   \
        }                                                                                                    \
    } while (0)
    if (D == 128) GDN_BWD(128); else GDN_BWD(64);
#undef GDN_BWD
    bwd_gates_kernel<<<H, bwd::NT, 0, s>>>(fa, fb, b.f.A, b.f.b_alpha, dgw, dbw, n_tok, H,
                                           static_cast<float *>(b.d_a_logit), static_cast<float *>(b.d_b_logit),
                                           b.d_A, b.d_b_alpha);
    if ((e = launched()) != cudaSuccess) return e;
    const int C4 = 3 * H * D * 4;
    bwd_reduce_kernel<<<(C4 + D + bwd::NT - 1) / bwd::NT, bwd::NT, 0, s>>>(dw_part, n_tiles, C4, dnorm_part,
                                                                           n_seq * H, D, b.d_conv_w,
                                                                           b.d_norm_w);
    return launched();
}

}  // namespace gdn

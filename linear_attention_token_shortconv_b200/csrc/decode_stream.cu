// K3s -- the decode step as a streaming kernel (bf16 inputs, dk = dv = 128),
// for one token per sequence (gdn_decode_step) or up to four consecutive tokens
// per sequence, as when a speculative (multi-token-prediction) draft is verified
// (gdn_decode_multi).
//
// Same arithmetic as K3, token after token (slinene.github.io write-up of "On
// the Design of Qwen3.8-Next Architecture", 模块 A; decode time is set by the
// bytes moved, as the digest's 前置知识 notes): conv over [history, tokens],
// SiLU, L2Norm, gates, and per token
//     S' = alpha S + beta k e^T,  e = v - alpha S^T k,
//     y  = alpha S^T q + beta (k.q) e,   out = sigmoid(z) RMSNorm(y) (1 + w).
// With T tokens the state is read and written once for all of them.  The state
// and history advance by n_keep[b] of the T tokens (all T when n_keep is NULL):
// a verifier can compute the outputs of a draft without committing it
// (n_keep = 0: the state is not written at all) and commit the accepted prefix.
//
// Persistent CTAs walk the (sequence, head) items.  Each item's inputs -- the
// 64 KB fp32 state, the tokens' q, k, v, z rows and the three history rows --
// arrive by bulk copies (TMA, cp.async.bulk) into one of the CTA's shared-memory
// stages, completing on the stage's mbarrier.  The CTA moves the stage into
// registers at once and refills it with a later item, so loads stay in flight
// while it computes; S' leaves from registers with coalesced streaming stores.
// One token: one CTA per SM with three stages.  Several tokens: the step is
// latency-bound in its barrier phases (a prelude, the state products, a small
// solve, the update), so two CTAs share each SM with one stage each and one
// CTA's phases fill the other's waits.  Every wait is bounded.
#include <cuda_bf16.h>

#include <cstring>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

__device__ unsigned int g_decode_err;

namespace dstream {
constexpr int D = 128;                      // dk = dv
constexpr int NT = 256;
constexpr int STATE = D * D * 4;            // 64 KB
constexpr uint32_t kMaxPolls = 1u << 24;
// Layout for up to TMAX tokens per item: one token (one CTA per SM, three
// stages in flight) or four (two CTAs per SM, one stage each: the state is read
// once for four tokens).
template <int TMAX> struct Layout {
    static constexpr int CTAS_PER_SM = TMAX == 1 ? 1 : 2;
    static constexpr int NSTAGE = TMAX == 1 ? 3 : 1;
    static constexpr int OFF_TOK = STATE;                      // q, k, v, z rows: [4][TMAX] x 256 B
    static constexpr int OFF_HIST = OFF_TOK + 4 * TMAX * 256;  // 3 slots x (q, k, v) x 256 B
    static constexpr int STAGE = OFF_HIST + 2304;
    static constexpr int OFF_MISC = NSTAGE * STAGE;            // barriers, reductions, prelude values
    // misc: barriers / flag [0, 64), gates [TMAX][2], Gram products [4][TMAX][TMAX],
    // then xs [TMAX][384] (conv + SiLU values), red [2][TMAX][8][128] (per-warp
    // partial state products; e and y later take slot w = 0 of each token's k and
    // q partials), kb [TMAX][128] (the update's scaled keys), zb [TMAX][128] bf16
    static constexpr int OFF_GATE = 64;
    static constexpr int OFF_GRAM = OFF_GATE + 8 * TMAX;
    static constexpr int OFF_XS = (OFF_GRAM + 16 * TMAX * TMAX + 15) / 16 * 16;
    static constexpr int SMEM = OFF_MISC + OFF_XS + (TMAX * 384 + 2 * TMAX * 8 * 128 + TMAX * 128) * 4 +
                                TMAX * 128 * 2 + 128;
    static_assert(STAGE % 128 == 0, "stage alignment");
    static_assert(SMEM * CTAS_PER_SM + 1024 * CTAS_PER_SM <= 233472, "shared memory per SM");
};
}  // namespace dstream

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            umma::smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(umma::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool dwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                      uint32_t max_polls = dstream::kMaxPolls) {
    for (uint32_t i = 0; i < max_polls; ++i) {
        if (umma::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicOr(&g_decode_err, 1u);
    return false;
}

// The token rows and history rows arrive by tensor copies (one per tensor instead
// of one per row).
struct DecodeMaps {
    CUtensorMap tok[4];   // q, k, v, z [B T][H][128] bf16, box {128, 1, TMAX}
    CUtensorMap hist;     // conv_hist as [3B][3][H][128] bf16, box {128, 1, 3, 3}
};

template <typename Tout, int TMAX>
__global__ void __launch_bounds__(dstream::NT, dstream::Layout<TMAX>::CTAS_PER_SM)
decode_stream_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k,
                     const bf16 *__restrict__ v, const float *__restrict__ conv_w,
                     bf16 *__restrict__ hist, const bf16 *__restrict__ a_logit,
                     const bf16 *__restrict__ b_logit, const float *__restrict__ A,
                     const float *__restrict__ b_alpha, const bf16 *__restrict__ z,
                     const float *__restrict__ norm_w, float *__restrict__ S,
                     Tout *__restrict__ out, const int32_t *__restrict__ n_keep, int B, int H, int T_rt,
                     const __grid_constant__ DecodeMaps maps) {
    using namespace dstream;
    using Lo = Layout<TMAX>;
    constexpr int NSTAGE = Lo::NSTAGE, STAGE = Lo::STAGE, OFF_TOK = Lo::OFF_TOK, OFF_HIST = Lo::OFF_HIST;
    const int T = TMAX == 1 ? 1 : T_rt;     // tokens per sequence in this call (<= TMAX)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<128>(smem_raw);
    uint8_t *misc = sm + Lo::OFF_MISC;
    uint64_t *full = reinterpret_cast<uint64_t *>(misc);                          // [NSTAGE]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 32);
    float *gate = reinterpret_cast<float *>(misc + Lo::OFF_GATE);                 // [TMAX][2]: alpha, beta
    float *gram = reinterpret_cast<float *>(misc + Lo::OFF_GRAM);                 // [4][TMAX][TMAX]
    float *xs = reinterpret_cast<float *>(misc + Lo::OFF_XS);                     // [TMAX][384] conv+SiLU values
    float *red = xs + TMAX * 384;                                                  // [2][TMAX][8][128]
    constexpr int ES = 8 * D;                                                      // e_t, y_t: stride between tokens
    float *e_s = red;                                                              // e_t at e_s + t ES
    float *y_s = red + TMAX * 8 * D;                                               // y_t at y_s + t ES
    float *kb = red + 2 * TMAX * 8 * D;                                            // [TMAX][128]
    bf16 *zb = reinterpret_cast<bf16 *>(kb + TMAX * D);                            // [TMAX][128], warp 7 only

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = B * H;
    // row of the state held in this thread's register r
    auto row_of = [&](int r) { return TMAX == 1 ? 16 * warp + r : warp + 8 * r; };
    const size_t C = (size_t)H * 3 * D;   // conv channels per token

    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) umma::mbar_init(full + i, 1);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    __syncthreads();

    // Stage s's loads for `item`, issued by lane 0 of warp 0: the state in one bulk
    // copy, each token tensor's rows by one tensor copy and the history rows by one
    // (per-row copies cost about 150 cycles of issue each, on the critical path).
    auto issue = [&](int item, int s) {   // warp 0
        const int b = item / H, h = item % H;
        uint8_t *st = sm + s * STAGE;
        uint64_t *bar = full + s;
        // the token box is TMAX rows (for several tokens, rows past T are not read)
        if (lane == 0) umma::mbar_expect_tx(bar, STATE + (TMAX == 1 ? T : TMAX) * 1024 + 2304);
        if (lane == 0) {   // the state in one copy, then one tensor copy per token tensor and the history
            bulk_load(st, S + ((size_t)b * H + h) * D * D, STATE, bar);
#pragma unroll
            for (int part = 0; part < 4; ++part)
                umma::tma_load_3d(st + OFF_TOK + part * TMAX * 256, &maps.tok[part], 0, h, b * T, bar);
            umma::tma_load_4d(st + OFF_HIST, &maps.hist, 0, h, 0, 3 * b, bar);
        }
    };
    const int first = blockIdx.x, stride = gridDim.x;
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < NSTAGE; ++i)
            if (first + i * stride < n_items) issue(first + i * stride, i);
    }

    int j = 0;
    for (int item = first; item < n_items; item += stride, ++j) {
        const int s = j % NSTAGE;
        const uint32_t parity = (uint32_t)(j / NSTAGE) & 1u;
        const uint8_t *st = sm + s * STAGE;
        const int b = item / H, h = item % H;
        const size_t gi = (size_t)b * H + h;
        // tokens of sequence b committed to the state and history
        const int nk = TMAX == 1 ? 1 : (n_keep ? min(max(__ldg(n_keep + b), 0), T) : T);
        // gate logits of this item's tokens (warp 3, lane t)
        float a_l = 0.f, b_l = 0.f;
        if (warp == 3 && lane < T) {
            const size_t gt = ((size_t)b * T + lane) * H + h;
            a_l = __bfloat162float(a_logit[gt]);
            b_l = __bfloat162float(b_logit[gt]);
        }
        // this thread's conv weights: channel tid (q or k) and v channel tid % 128
        // (one token: threads < 128 only)
        const float4 w0 = __ldg(reinterpret_cast<const float4 *>(conv_w) +
                                (tid < D ? (size_t)h * D + tid : (size_t)H * D + (size_t)h * D + (tid - D)));
        const float4 w1 = (TMAX > 1 || tid < D)
                              ? __ldg(reinterpret_cast<const float4 *>(conv_w) + (size_t)2 * H * D + (size_t)h * D + tid % D)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        dwait(full + s, parity, abort_flag);

        // ---- take everything out of the stage: the state into registers (lane l
        // holds columns 4 l .. 4 l + 3 of 16 rows: rows 16 w .. 16 w + 15 of warp w
        // for one token, rows w, w + 8, .. for several -- each measured faster
        // in its kernel), the
        // conv inputs through the prelude into xs, z into warp 7's registers; the
        // advanced history goes straight back to global memory.
        const float4 *Sv = reinterpret_cast<const float4 *>(st);
        float4 sreg[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) sreg[r] = Sv[row_of(r) * 32 + lane];
        const bf16 *tok = reinterpret_cast<const bf16 *>(st + OFF_TOK);
        const bf16 *hs = reinterpret_cast<const bf16 *>(st + OFF_HIST);
        bf16 *hb = hist + (size_t)b * 3 * C;
        // One channel over the window [history slots 0..2, tokens 0..T-1]: the conv +
        // SiLU values of tokens [t_lo, t_hi) into xs and, if `adv`, the history
        // advanced by the committed tokens.
        auto channel = [&](int part, int i, const float4 w, int t_lo, int t_hi, bool adv) {
            const int ch = part * D + i;   // part 0 q, 1 k, 2 v
            bf16 win[3 + TMAX];
#pragma unroll
            for (int r = 0; r < 3; ++r) win[r] = hs[r * 384 + part * 128 + i];
#pragma unroll
            for (int t = 0; t < TMAX; ++t)
                if (t < T) win[3 + t] = tok[(part * TMAX + t) * 128 + i];
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T && t >= t_lo && t < t_hi) {
                    float acc = w.x * __bfloat162float(win[t]);
                    acc = fmaf(w.y, __bfloat162float(win[t + 1]), acc);
                    acc = fmaf(w.z, __bfloat162float(win[t + 2]), acc);
                    acc = fmaf(w.w, __bfloat162float(win[t + 3]), acc);
                    xs[t * 384 + ch] = __fdividef(acc, 1.0f + __expf(-acc));
                }
            }
            if (adv && nk > 0) {
                const size_t c = (size_t)part * H * D + (size_t)h * D + i;
#pragma unroll
                for (int r = 0; r < 3; ++r) {
                    bf16 val = win[0];
#pragma unroll
                    for (int u = 1; u < 3 + TMAX; ++u)
                        if (u == nk + r) val = win[u];
                    hb[r * C + c] = val;
                }
            }
        };
        if constexpr (TMAX == 1) {
            for (int ch = tid; ch < 3 * D; ch += NT) channel(ch / D, ch % D, ch < NT ? w0 : w1, 0, 1, true);
        } else {
            // q or k channel tid over all tokens, and half of v channel tid % 128:
            // the first half of the tokens (threads < 128, which also advance its
            // history) or the second
            channel(tid / D, tid % D, w0, 0, TMAX, true);
            const int half = tid / D;
            channel(2, tid % D, w1, half * (TMAX / 2), half ? TMAX : TMAX / 2, half == 0);
        }
        if (warp == NT / 32 - 1) {   // z rows out of the stage; warp 7 alone reads them back
            const uint2 *zsrc = reinterpret_cast<const uint2 *>(tok + 3 * TMAX * 128);
#pragma unroll
            for (int t = 0; t < TMAX; ++t)
                if (t < T) reinterpret_cast<uint2 *>(zb)[t * 32 + lane] = zsrc[t * 32 + lane];
        }
        __syncthreads();   // stage s is consumed and xs is complete
        if (warp == 0 && item + NSTAGE * stride < n_items) issue(item + NSTAGE * stride, s);

        // ---- the Gram products of the raw conv outputs, alongside pass 1.  Token t
        // owns entries t (t + 2) .. (t + 1)(t + 3) - 1: q_t.q_t (type 0), k_t.k_t
        // (type 1), k_s.k_t for s < t (type 2), k_s.q_t for s <= t (type 3); warp w
        // takes entries w, w + 8, ..  Warp 3, lane t, also computes token t's gates.
        for (int d = warp; d < 2 * TMAX + TMAX * TMAX; d += NT / 32) {
            int t = 0;
            while ((t + 1) * (t + 3) <= d) ++t;
            const int r = d - t * (t + 2);
            const int type = r < 2 ? r : (r < 2 + t ? 2 : 3);
            const int sx = r < 2 ? t : (type == 2 ? r - 2 : r - 2 - t);
            if (t < T) {
                const float *xa = xs + (type == 0 ? t * 384 : sx * 384 + D);
                const float *xb = xs + t * 384 + (type == 1 || type == 2 ? D : 0);
                float acc = 0.f;
#pragma unroll
                for (int i = lane; i < D; i += 32) acc = fmaf(xa[i], xb[i], acc);
                acc = group_sum<32>(acc);
                if (lane == 0) gram[(type * TMAX + t) * TMAX + sx] = acc;
            }
        }
        if (warp == 3 && lane < T) {
            gate[lane * 2 + 0] = expf(log_decay(a_l, __ldg(A + h), __ldg(b_alpha + h)));
            gate[lane * 2 + 1] = sigmoid_acc(b_l);
        }
        // ---- pass 1: partial S0^T k_t and S0^T q_t over this thread's 16 rows, two
        // tokens per sweep over the register state (fewer live accumulators)
        constexpr int TG = TMAX < 2 ? TMAX : 2;
#pragma unroll
        for (int t0 = 0; t0 < TMAX; t0 += TG) {
            if (t0 < T) {
                float4 pk[TG], pq[TG];
#pragma unroll
                for (int u = 0; u < TG; ++u) { pk[u] = make_float4(0.f, 0.f, 0.f, 0.f); pq[u] = pk[u]; }
                // row r of the state against token t0 + u's key and query entries kk, qq
                auto acc_row = [&](int r, int u, float kk, float qq) {
                    const float2 s01 = make_float2(sreg[r].x, sreg[r].y), s23 = make_float2(sreg[r].z, sreg[r].w);
                    const float2 k2 = make_float2(kk, kk), q2 = make_float2(qq, qq);
                    float2 lo = ffma2(s01, k2, make_float2(pk[u].x, pk[u].y));
                    float2 hi = ffma2(s23, k2, make_float2(pk[u].z, pk[u].w));
                    pk[u] = make_float4(lo.x, lo.y, hi.x, hi.y);
                    lo = ffma2(s01, q2, make_float2(pq[u].x, pq[u].y));
                    hi = ffma2(s23, q2, make_float2(pq[u].z, pq[u].w));
                    pq[u] = make_float4(lo.x, lo.y, hi.x, hi.y);
                };
                if constexpr (TMAX == 1) {   // consecutive rows: one 16-byte load per four
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const float4 kv = *reinterpret_cast<const float4 *>(xs + D + 16 * warp + 4 * g);
                        const float4 qv = *reinterpret_cast<const float4 *>(xs + 16 * warp + 4 * g);
                        acc_row(4 * g + 0, 0, kv.x, qv.x);
                        acc_row(4 * g + 1, 0, kv.y, qv.y);
                        acc_row(4 * g + 2, 0, kv.z, qv.z);
                        acc_row(4 * g + 3, 0, kv.w, qv.w);
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const int i = row_of(r);
#pragma unroll
                        for (int u = 0; u < TG; ++u) {
                            const int t = t0 + u;
                            if (t < T) acc_row(r, u, xs[t * 384 + D + i], xs[t * 384 + i]);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < TG; ++u) {
                    const int t = t0 + u;
                    if (t < T) {
                        reinterpret_cast<float4 *>(red + (t * 8 + warp) * D)[lane] = pk[u];
                        reinterpret_cast<float4 *>(red + ((TMAX + t) * 8 + warp) * D)[lane] = pq[u];
                    }
                }
            }
        }
        __syncthreads();   // gram, gate and red are complete

        // Per-token scalars, the same in every thread: rq, rk normalise q_t, k_t;
        // cum[t] = alpha_0 .. alpha_{t-1} (the decay from the item's start to token t).
        float rq[TMAX], rk[TMAX], al[TMAX], be[TMAX], cum[TMAX + 1];
        cum[0] = 1.f;
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
            if (t < T) {
                rq[t] = rsqrtf(gram[(0 * TMAX + t) * TMAX + t] + kNormEps);
                rk[t] = rsqrtf(gram[(1 * TMAX + t) * TMAX + t] + kNormEps);
                al[t] = gate[t * 2 + 0];
                be[t] = gate[t * 2 + 1];
            } else {
                rq[t] = rk[t] = be[t] = 0.f;
                al[t] = 1.f;
            }
            cum[t + 1] = cum[t] * al[t];
        }
        // ---- column solve (thread j < 128 owns column j), from S0 alone:
        //   e_t = v_t - cum_{t+1} S0^T k_t - sum_{s<t} (cum_{t+1}/cum_{s+1}) beta_s (k_s.k_t) e_s
        //   y_t = cum_{t+1} S0^T q_t + sum_{s<=t} (cum_{t+1}/cum_{s+1}) beta_s (k_s.q_t) e_s
        // with unit-norm k, q; the ratio is the product alpha_{s+1} .. alpha_t.
        if (tid < D) {
            float e[TMAX];
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    float sk = 0.f, sq = 0.f;
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        sk += red[(t * 8 + w) * D + tid];
                        sq += red[((TMAX + t) * 8 + w) * D + tid];
                    }
                    float ev = xs[t * 384 + 2 * D + tid] - cum[t + 1] * rk[t] * sk;
                    float yv = cum[t + 1] * rq[t] * sq;
                    float ratio = 1.f;   // alpha_{s+1} .. alpha_t, built downwards from s = t
#pragma unroll
                    for (int s2 = TMAX - 1; s2 >= 0; --s2) {
                        if (s2 <= t) {
                            if (s2 < t) {
                                ratio *= al[s2 + 1];
                                ev -= ratio * be[s2] * rk[s2] * rk[t] * gram[(2 * TMAX + t) * TMAX + s2] * e[s2];
                            }
                        }
                    }
                    e[t] = ev;
                    ratio = 1.f;
#pragma unroll
                    for (int s2 = TMAX - 1; s2 >= 0; --s2) {
                        if (s2 <= t) {
                            if (s2 < t) ratio *= al[s2 + 1];
                            yv = fmaf(ratio * be[s2] * rk[s2] * rq[t] * gram[(3 * TMAX + t) * TMAX + s2], e[s2], yv);
                        }
                    }
                    e_s[t * ES + tid] = ev;   // over slot w = 0, which this thread alone read
                    y_s[t * ES + tid] = yv;
                }
            }
            // the update's keys, (cum_nk / cum_{s+1}) beta_s k_s with unit-norm k_s
            float ratio = 1.f;
#pragma unroll
            for (int s2 = TMAX - 1; s2 >= 0; --s2) {
                if (s2 < nk) {
                    kb[s2 * D + tid] = ratio * be[s2] * rk[s2] * xs[s2 * 384 + D + tid];
                    ratio *= al[s2];
                }
            }
        }
        __syncthreads();   // e, y and kb are complete
        // ---- pass 2: the committed state
        //   S_nk = cum_nk S0 + sum_{s<nk} (cum_nk/cum_{s+1}) beta_s k_s e_s^T
        // from registers straight to HBM (nothing is written when nk = 0)
        if (nk > 0) {
            float decay = 1.f;   // cum_nk
#pragma unroll
            for (int s2 = 0; s2 < TMAX; ++s2)
                if (s2 < nk) decay *= al[s2];
            float2 e01[TMAX], e23[TMAX];
#pragma unroll
            for (int s2 = 0; s2 < TMAX; ++s2) {
                const float4 e4 = s2 < nk ? reinterpret_cast<const float4 *>(e_s + s2 * ES)[lane]
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                e01[s2] = make_float2(e4.x, e4.y);
                e23[s2] = make_float2(e4.z, e4.w);
            }
            const float2 dec2 = make_float2(decay, decay);
            float4 *Sg = reinterpret_cast<float4 *>(S + gi * D * D);
            // row r of S' from the register state and the keys' entries bk[s2] at row r
            auto store_row = [&](int r, const float (&bk)[TMAX]) {
                float2 lo = fmul2(dec2, make_float2(sreg[r].x, sreg[r].y));
                float2 hi = fmul2(dec2, make_float2(sreg[r].z, sreg[r].w));
#pragma unroll
                for (int s2 = 0; s2 < TMAX; ++s2) {
                    if (s2 < nk) {
                        const float2 b2 = make_float2(bk[s2], bk[s2]);
                        lo = ffma2(b2, e01[s2], lo);
                        hi = ffma2(b2, e23[s2], hi);
                    }
                }
                __stcs(Sg + row_of(r) * 32 + lane, make_float4(lo.x, lo.y, hi.x, hi.y));
            };
            if constexpr (TMAX == 1) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float4 kv = *reinterpret_cast<const float4 *>(kb + 16 * warp + 4 * g);
                    store_row(4 * g + 0, {kv.x});
                    store_row(4 * g + 1, {kv.y});
                    store_row(4 * g + 2, {kv.z});
                    store_row(4 * g + 3, {kv.w});
                }
            } else {
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float bk[TMAX];
#pragma unroll
                    for (int s2 = 0; s2 < TMAX; ++s2) bk[s2] = s2 < nk ? kb[s2 * D + row_of(r)] : 0.f;
                    store_row(r, bk);
                }
            }
        }
        // ---- outputs (warp 7)
        if (warp == NT / 32 - 1) {
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    float yv[4], ss = 0.f;
#pragma unroll
                    for (int m = 0; m < 4; ++m) { yv[m] = y_s[t * ES + lane + 32 * m]; ss = fmaf(yv[m], yv[m], ss); }
                    ss = group_sum<32>(ss);
                    const float rr = rsqrtf(ss / D + kNormEps);
                    const size_t go = (((size_t)b * T + t) * H + h) * D;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int col = lane + 32 * m;
                        const float zv = __bfloat162float(zb[t * D + col]);
                        out[go + col] = from_f32<Tout>(sigmoid_fast(zv) * yv[m] * rr * (1.0f + __ldg(norm_w + col)));
                    }
                }
            }
        }
        // No barrier here: after the third barrier nothing reads xs, so the next
        // item's prelude may overwrite it; red (with e and y), kb, gram and gate
        // are written only after the next item's first barrier, which every
        // thread reaches after its own reads here; zb is warp 7's alone.
    }
}

bool decode_stream_supported(const DecodeArgs &a) {
    return a.in_bf16 && a.dk == 128 && a.dv == 128;
}

cudaError_t launch_decode_stream(const DecodeArgs &a, int T, const int32_t *n_keep) {
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (T < 1 || T > 4) return cudaErrorInvalidValue;
    const int items = a.B * a.H;
    if (items == 0) return cudaSuccess;
    const int per_sm = T == 1 && !n_keep ? dstream::Layout<1>::CTAS_PER_SM : dstream::Layout<4>::CTAS_PER_SM;
    const int grid = items < sms * per_sm ? items : sms * per_sm;
    DecodeMaps maps;
    std::memset(&maps, 0, sizeof maps);
    {   // tensor maps of the token rows and the history
        const long long C = 3LL * a.H * 128;
        const void *tok[4] = {a.q, a.k, a.v, a.z};
        const long long td[3] = {128, a.H, (long long)a.B * T}, ts[2] = {256, (long long)a.H * 256};
        const int tb[3] = {128, 1, T == 1 && !n_keep ? 1 : 4};
        for (int p = 0; p < 4; ++p)
            if ((e = make_tma_plain_bf16(reinterpret_cast<TmaMap *>(&maps.tok[p]), tok[p], 3, td, ts, tb)) != cudaSuccess)
                return e;
        const long long hd[4] = {128, a.H, 3, 3LL * a.B}, hs[3] = {256, (long long)a.H * 256, C * 2};
        const int hbx[4] = {128, 1, 3, 3};
        if ((e = make_tma_plain_bf16(reinterpret_cast<TmaMap *>(&maps.hist), a.conv_hist, 4, hd, hs, hbx)) != cudaSuccess)
            return e;
    }
#define GDN_DSTREAM(TOUT, TM)                                                                      \
    e = cudaFuncSetAttribute(decode_stream_kernel<TOUT, TM>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             dstream::Layout<TM>::SMEM);                                          \
    if (e != cudaSuccess) return e;                                                                \
    decode_stream_kernel<TOUT, TM><<<grid, dstream::NT, dstream::Layout<TM>::SMEM, a.stream>>>(    \
        (const bf16 *)a.q, (const bf16 *)a.k, (const bf16 *)a.v, a.conv_w, (bf16 *)a.conv_hist,   \
        (const bf16 *)a.a_logit, (const bf16 *)a.b_logit, a.A, a.b_alpha, (const bf16 *)a.z,      \
        a.norm_w, a.S, (TOUT *)a.out, n_keep, a.B, a.H, T, maps)
    if (T == 1 && !n_keep) {
        if (a.out_bf16) { GDN_DSTREAM(bf16, 1); } else { GDN_DSTREAM(float, 1); }
    } else {
        if (a.out_bf16) { GDN_DSTREAM(bf16, 4); } else { GDN_DSTREAM(float, 4); }
    }
#undef GDN_DSTREAM
    return launched();
}

cudaError_t launch_decode_stream(const DecodeArgs &a) { return launch_decode_stream(a, 1, nullptr); }

// One CTA waits, through dwait, for a barrier phase that nothing completes.
__global__ void decode_wait_selftest_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        abort_flag = 0;
        umma::fence_mbar_init();
    }
    __syncthreads();
    dwait(&bar, 0, &abort_flag, max_polls);
}

cudaError_t decode_wait_selftest(uint32_t max_polls, cudaStream_t s) {
    decode_wait_selftest_kernel<<<1, 32, 0, s>>>(max_polls);
    return cudaGetLastError();
}

cudaError_t decode_error_word(unsigned *v, bool clear, cudaStream_t s) {
    return read_error_word(g_decode_err, v, clear, s);
}

}  // namespace gdn

/*
 * gdn_oracle.c -- plain fp64 CPU oracle of the Gated DeltaNet (GDN) token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check of the package entry
 * file and the CPU-baseline leg of bench.py load this library; the CUDA
 * product path never does, and the two share no code.
 *
 * What it follows (web write-ups of the technical report "On the Design of
 * Qwen3.8-Next Architecture: Evaluation, Efficiency, and Training Stability"):
 *   [digest]   paper.rainbus.top digest, section "方法步骤详情", step (1):
 *              S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T and
 *              alpha_t = exp[-exp(A) softplus(W_alpha x_t + b_alpha)];
 *              Figure 2 caption: short causal convolutions on q, k, v, L2-normalised
 *              q and k, sigmoid output gate on the zero-centred RMS-normalised output.
 *   [write-up] slinene.github.io write-up, section "模块 A — Gated DeltaNet 混合层":
 *              "递归状态" (per-head state S in R^{dk x dv}, transposed convention;
 *              the erase-then-write update and the readout y_t = S_t^T q_t),
 *              "参数化" (q = L2Norm(SiLU(ShortConv(.))), k likewise,
 *              v = SiLU(ShortConv(.)), beta = sigmoid(.), alpha as above,
 *              o = W_o[sigmoid(W_z x) * RMSNorm(y)]), and the list of engineering
 *              choices (sigmoid output gate, zero-centred RMSNorm).
 *
 * Readings taken where the pages are silent (all listed in the design notes):
 *   - ShortConv: causal depthwise cross-correlation of width K, tap K-1 on the
 *     current token, zero history before each sequence start, no bias.
 *     Conv channels are ordered [q heads | k heads | v heads]:
 *     c = h*dk + i (q), H*dk + h*dk + i (k), 2*H*dk + h*dv + i (v).
 *   - L2Norm: x / sqrt(sum x^2 + eps); RMSNorm: y / sqrt(mean y^2 + eps);
 *     eps = 1e-6 for both.
 *   - zero-centred RMSNorm has gain (1 + w), w of shape [dv] shared by heads.
 *   - A and b_alpha are one scalar per head; no 1/sqrt(dk) scale on q.
 *   - The readout uses the post-update state.
 *   - Decode keeps the last K-1 raw (pre-conv) tokens of each sequence in a
 *     history buffer, oldest first (slot j holds tap j); after the step the
 *     buffer shifts by one and the current raw token enters the last slot.
 *
 * Inputs are read from the exact stored bits (fp32, or bf16 widened exactly)
 * and every operation is done in double precision, token by token.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_EPS 1e-6

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Read element i of an fp32 or bf16 array as a double (exact widening). */
static double load_elem(const void *p, int dtype, size_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static void copy_elem(void *dst, size_t di, const void *src, size_t si, int dtype)
{
    if (dtype == ORACLE_F32)
        ((float *)dst)[di] = ((const float *)src)[si];
    else
        ((uint16_t *)dst)[di] = ((const uint16_t *)src)[si];
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double silu(double u) { return u * sigmoid(u); }

/* softplus(x) = log(1 + e^x), evaluated without overflow. */
static double softplus(double x)
{
    return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x));
}

/* alpha = exp(-exp(A) * softplus(a + b_alpha))  ([digest] step (1); [write-up] 参数化). */
static double decay_gate(double a_logit, double A, double b_alpha)
{
    return exp(-exp(A) * softplus(a_logit + b_alpha));
}

/* beta = sigmoid(b)  ([write-up] 参数化, "写入强度"). */
static double write_gate(double b_logit) { return sigmoid(b_logit); }

static void l2_normalise(double *x, int n)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i)
        ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss + ORACLE_EPS);
    for (int i = 0; i < n; ++i)
        x[i] *= r;
}

/*
 * One prefill token's conv output for `n` consecutive channels of one tensor.
 * x is the raw tensor [N_tok, H, d]; the channel's column inside a token row is
 * col0 + i; the conv weight row is wrow0 + i.  Tokens before seq_start count 0.
 */
static void shortconv_prefill(const void *x, int dtype, size_t row_elems, size_t col0,
                              const float *conv_w, size_t wrow0, int K,
                              long t, long seq_start, int n, double *outv)
{
    for (int i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = 0; j < K; ++j) {
            long src = t - (K - 1) + j;
            if (src < seq_start)
                continue;
            acc += (double)conv_w[(wrow0 + i) * K + j] *
                   load_elem(x, dtype, (size_t)src * row_elems + col0 + i);
        }
        outv[i] = acc;
    }
}

/*
 * Gated delta rule, erase-then-write form ([write-up] 递归状态):
 *   S~ = alpha S;  e = v - S~^T k;  S = S~ + beta k e^T;  y = S^T q.
 * S is row-major [dk][dv].
 */
static void delta_rule_step(double *S, int dk, int dv, const double *q, const double *k,
                            const double *v, double alpha, double beta, double *e, double *y)
{
    for (int i = 0; i < dk * dv; ++i)
        S[i] *= alpha;
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i)
            s += S[(size_t)i * dv + j] * k[i];
        e[j] = v[j] - s;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] += beta * k[i] * e[j];
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i)
            s += S[(size_t)i * dv + j] * q[i];
        y[j] = s;
    }
}

/* o = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w)  ([write-up] 参数化 and the
 * zero-centred RMSNorm choice). */
static void gated_rmsnorm(int dv, const double *y, const double *z, const float *w, double *o)
{
    double ms = 0.0;
    for (int j = 0; j < dv; ++j)
        ms += y[j] * y[j];
    ms /= (double)dv;
    double r = 1.0 / sqrt(ms + ORACLE_EPS);
    for (int j = 0; j < dv; ++j)
        o[j] = sigmoid(z[j]) * y[j] * r * (1.0 + (double)w[j]);
}

/* Per-token prelude of one head: conv -> SiLU (-> L2Norm for q, k); gates. */
typedef struct {
    int H, dk, dv, K, dtype;
    const void *q, *k, *v, *a, *b;
    const float *conv_w, *A, *b_alpha;
} prelude_args;

static void prelude_prefill_token(const prelude_args *p, int h, long t, long seq_start,
                                  double *qh, double *kh, double *vh, double *alpha, double *beta)
{
    const int H = p->H, dk = p->dk, dv = p->dv;
    shortconv_prefill(p->q, p->dtype, (size_t)H * dk, (size_t)h * dk, p->conv_w,
                      (size_t)h * dk, p->K, t, seq_start, dk, qh);
    shortconv_prefill(p->k, p->dtype, (size_t)H * dk, (size_t)h * dk, p->conv_w,
                      (size_t)H * dk + (size_t)h * dk, p->K, t, seq_start, dk, kh);
    shortconv_prefill(p->v, p->dtype, (size_t)H * dv, (size_t)h * dv, p->conv_w,
                      (size_t)2 * H * dk + (size_t)h * dv, p->K, t, seq_start, dv, vh);
    for (int i = 0; i < dk; ++i) qh[i] = silu(qh[i]);
    for (int i = 0; i < dk; ++i) kh[i] = silu(kh[i]);
    for (int i = 0; i < dv; ++i) vh[i] = silu(vh[i]);
    l2_normalise(qh, dk);
    l2_normalise(kh, dk);
    size_t gi = (size_t)t * H + h;
    *alpha = decay_gate(load_elem(p->a, p->dtype, gi), (double)p->A[h], (double)p->b_alpha[h]);
    *beta = write_gate(load_elem(p->b, p->dtype, gi));
}

static int set_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
    return omp_get_max_threads();
#else
    (void)n_threads;
    return 1;
#endif
}

/* ---------------------------------------------------------------- exported */

/* Number of OpenMP threads a call with n_threads would use. */
int gdn_oracle_threads(int n_threads) { return set_threads(n_threads); }

/*
 * Whole prefill of a packed batch.  Shapes: q,k [N_tok,H,dk], v,z [N_tok,H,dv],
 * a,b [N_tok,H] (dtype in_dtype), conv_w [H(2dk+dv), K] fp32, A,b_alpha [H],
 * norm_w [dv], S0 [N_seq,H,dk,dv] fp32 or NULL (zeros), cu_seqlens [N_seq+1]
 * host int32 or NULL (equal lengths N_tok/N_seq).  Writes out [N_tok,H,dv] and,
 * when non-NULL, S_final [N_seq,H,dk,dv] in double.  Returns 0, or -1 on bad sizes.
 */
int gdn_oracle_prefill(int n_seq, int n_tok, int H, int dk, int dv, int K, int in_dtype,
                       const void *q, const void *k, const void *v, const float *conv_w,
                       const void *a_logit, const void *b_logit, const float *A,
                       const float *b_alpha, const void *z, const float *norm_w,
                       const float *S0, const int32_t *cu_seqlens, double *out,
                       double *S_final, int n_threads)
{
    if (n_seq <= 0 || n_tok < 0 || H <= 0 || dk <= 0 || dv <= 0 || K <= 0)
        return -1;
    if (!cu_seqlens && n_tok % n_seq != 0)
        return -1;
    prelude_args p = {H, dk, dv, K, in_dtype, q, k, v, a_logit, b_logit, conv_w, A, b_alpha};
    set_threads(n_threads);
    const long pairs = (long)n_seq * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long ph = 0; ph < pairs; ++ph) {
        const int n = (int)(ph / H), h = (int)(ph % H);
        const long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * (n_tok / n_seq);
        const long t1 = cu_seqlens ? cu_seqlens[n + 1] : (long)(n + 1) * (n_tok / n_seq);
        if (t0 < 0 || t1 < t0 || t1 > n_tok) {
            bad = 1;
            continue;
        }
        double *S = calloc((size_t)dk * dv, sizeof(double));
        double *buf = malloc(sizeof(double) * (size_t)(2 * dk + 4 * dv));
        double *qh = buf, *kh = qh + dk, *vh = kh + dk, *e = vh + dv, *y = e + dv, *zz = y + dv;
        if (S0)
            for (size_t i = 0; i < (size_t)dk * dv; ++i)
                S[i] = (double)S0[((size_t)n * H + h) * dk * dv + i];
        for (long t = t0; t < t1; ++t) {
            double alpha, beta;
            prelude_prefill_token(&p, h, t, t0, qh, kh, vh, &alpha, &beta);
            delta_rule_step(S, dk, dv, qh, kh, vh, alpha, beta, e, y);
            for (int j = 0; j < dv; ++j)
                zz[j] = load_elem(z, in_dtype, ((size_t)t * H + h) * dv + j);
            gated_rmsnorm(dv, y, zz, norm_w, out + ((size_t)t * H + h) * dv);
        }
        if (S_final)
            memcpy(S_final + ((size_t)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
        free(buf);
        free(S);
    }
    return bad ? -1 : 0;
}

/*
 * One decode step for B sequences of one token each.  q,k [B,H,dk], v,z [B,H,dv],
 * a,b [B,H] in in_dtype; hist [B,K-1,H(2dk+dv)] in in_dtype (raw pre-conv
 * history, oldest first, shifted in place); S [B,H,dk,dv] double (updated in
 * place); out [B,H,dv] double.
 */
int gdn_oracle_decode_step(int B, int H, int dk, int dv, int K, int in_dtype,
                           const void *q, const void *k, const void *v, const float *conv_w,
                           void *hist, const void *a_logit,
                           const void *b_logit, const float *A, const float *b_alpha,
                           const void *z, const float *norm_w, double *S, double *out,
                           int n_threads)
{
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0 || K < 2)
        return -1;
    const int R = K - 1;
    const size_t C = (size_t)H * (2 * dk + dv);
    set_threads(n_threads);
    const long pairs = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long ph = 0; ph < pairs; ++ph) {
        const int bq = (int)(ph / H), h = (int)(ph % H);
        double *buf = malloc(sizeof(double) * (size_t)(2 * dk + 4 * dv));
        double *qh = buf, *kh = qh + dk, *vh = kh + dk, *e = vh + dv, *y = e + dv, *zz = y + dv;
        /* the three tensors of this head: (source, width, column in its tensor row, conv channel) */
        const void *src[3] = {q, k, v};
        const int width[3] = {dk, dk, dv};
        const size_t row_elems[3] = {(size_t)H * dk, (size_t)H * dk, (size_t)H * dv};
        const size_t col[3] = {(size_t)h * dk, (size_t)h * dk, (size_t)h * dv};
        const size_t chan[3] = {(size_t)h * dk, (size_t)H * dk + (size_t)h * dk,
                                (size_t)2 * H * dk + (size_t)h * dv};
        double *dst[3] = {qh, kh, vh};
        for (int s = 0; s < 3; ++s) {
            for (int i = 0; i < width[s]; ++i) {
                const size_t c = chan[s] + i;
                double acc = 0.0;
                for (int j = 0; j < R; ++j)
                    acc += (double)conv_w[c * K + j] *
                           load_elem(hist, in_dtype, ((size_t)bq * R + j) * C + c);
                acc += (double)conv_w[c * K + (K - 1)] *
                       load_elem(src[s], in_dtype, (size_t)bq * row_elems[s] + col[s] + i);
                dst[s][i] = silu(acc);
            }
        }
        l2_normalise(qh, dk);
        l2_normalise(kh, dk);
        const size_t gi = (size_t)bq * H + h;
        const double alpha = decay_gate(load_elem(a_logit, in_dtype, gi), (double)A[h],
                                        (double)b_alpha[h]);
        const double beta = write_gate(load_elem(b_logit, in_dtype, gi));
        delta_rule_step(S + gi * dk * dv, dk, dv, qh, kh, vh, alpha, beta, e, y);
        for (int j = 0; j < dv; ++j)
            zz[j] = load_elem(z, in_dtype, gi * dv + j);
        gated_rmsnorm(dv, y, zz, norm_w, out + gi * dv);
        /* shift the history of this head's channels by one; the raw token enters last */
        for (int s = 0; s < 3; ++s)
            for (int i = 0; i < width[s]; ++i) {
                const size_t c = chan[s] + i;
                for (int j = 0; j + 1 < R; ++j)
                    copy_elem(hist, ((size_t)bq * R + j) * C + c, hist,
                              ((size_t)bq * R + j + 1) * C + c, in_dtype);
                copy_elem(hist, ((size_t)bq * R + R - 1) * C + c, src[s],
                          (size_t)bq * row_elems[s] + col[s] + i, in_dtype);
            }
        free(buf);
    }
    return 0;
}

/* The recurrence alone, on prepared vectors: q,k [T,dk], v [T,dv], alpha,beta [T];
 * S [dk,dv] in/out; y [T,dv] out. */
int gdn_oracle_delta_rule(int T, int dk, int dv, const double *q, const double *k,
                          const double *v, const double *alpha, const double *beta, double *S,
                          double *y)
{
    if (T < 0 || dk <= 0 || dv <= 0)
        return -1;
    double *e = malloc(sizeof(double) * (size_t)dv);
    for (int t = 0; t < T; ++t)
        delta_rule_step(S, dk, dv, q + (size_t)t * dk, k + (size_t)t * dk, v + (size_t)t * dv,
                        alpha[t], beta[t], e, y + (size_t)t * dv);
    free(e);
    return 0;
}

/* The prelude alone for head h of one sequence made of tokens 0..T-1 of the given
 * arrays (same layouts as the prefill).  Writes q,k [T,dk], v [T,dv], alpha, beta [T]. */
int gdn_oracle_prelude(int T, int H, int dk, int dv, int K, int in_dtype, const void *q,
                       const void *k, const void *v, const float *conv_w, const void *a_logit,
                       const void *b_logit, const float *A, const float *b_alpha, int h,
                       double *qh, double *kh, double *vh, double *alpha, double *beta)
{
    if (T < 0 || H <= 0 || h < 0 || h >= H || dk <= 0 || dv <= 0 || K <= 0)
        return -1;
    prelude_args p = {H, dk, dv, K, in_dtype, q, k, v, a_logit, b_logit, conv_w, A, b_alpha};
    for (long t = 0; t < T; ++t)
        prelude_prefill_token(&p, h, t, 0, qh + (size_t)t * dk, kh + (size_t)t * dk,
                              vh + (size_t)t * dv, alpha + t, beta + t);
    return 0;
}

/* The output stage alone: o = sigmoid(z) * RMSNorm(y) * (1 + w) on n rows of dv. */
int gdn_oracle_gated_rmsnorm(int n, int dv, const double *y, const double *z, const float *w,
                             double *o)
{
    if (n < 0 || dv <= 0)
        return -1;
    for (int r = 0; r < n; ++r)
        gated_rmsnorm(dv, y + (size_t)r * dv, z + (size_t)r * dv, w, o + (size_t)r * dv);
    return 0;
}

/* ------------------------------------------------------------------ backward */

static double dsilu(double x)   /* d/dx [x sigmoid(x)] */
{
    const double s = sigmoid(x);
    return s * (1.0 + x * (1.0 - s));
}

/*
 * Gradients of L = <d_out, out> + <d_S_final, S_final> for the prefill above, with
 * respect to every input: the reverse-mode derivative of each forward step, taken
 * in the reverse order of the tokens.  Per token t of a sequence (one head), with
 * P = S_{t-1} (the state before the token), e = v - alpha P^T k, S_t = alpha P +
 * beta k e^T, y = S_t^T q, n = y r, r = (mean y^2 + eps)^{-1/2},
 * o = sigmoid(z) n (1 + w), and D the gradient of S_t:
 *   dz = do n (1 + w) s'(z);  dw += do sigmoid(z) n;  dn = do sigmoid(z) (1 + w);
 *   dy = r dn - r^3 y mean(dn y);           D += q dy^T;  dq = S_t dy;
 *   de = beta D^T k;  dv = de;  dbeta = k^T D e;
 *   dk = beta D e - alpha P de;  dalpha = <D, P> - k^T P de;
 *   gradient of P = alpha D - alpha k de^T.
 * Gates: alpha = exp(g), g = -e^A softplus(a + b_alpha): dg = alpha dalpha,
 * da = dg (-e^A) sigmoid(a + b_alpha), dA += dg g, db_alpha += da; beta =
 * sigmoid(b): db = dbeta beta (1 - beta).  L2Norm x -> x rho, rho = (|x|^2 +
 * eps)^{-1/2}: dx = rho dxh - rho^3 x (x . dxh).  SiLU: du/dx = sigmoid(x)(1 + x
 * (1 - sigmoid(x))).  ShortConv (tap j of K on token t - (K-1) + j): d_raw[t - (K-1)
 * + j] += w_j dx_t and dw_j += dx_t raw[t - (K-1) + j], inside the sequence.
 *
 * Shapes as gdn_oracle_prefill; d_out [N_tok,H,dv] and d_S_final [N_seq,H,dk,dv]
 * (or NULL = 0) in double.  Outputs in double: dq, dk [N_tok,H,dk], dv, dz
 * [N_tok,H,dv], d_a, d_b [N_tok,H], d_conv_w [H(2dk+dv),K], d_A, d_b_alpha [H],
 * d_norm_w [dv], d_S0 [N_seq,H,dk,dv].  Every state of a sequence is kept, so this
 * is for small inputs.  Returns 0, or -1 on bad sizes.
 */
int gdn_oracle_backward(int n_seq, int n_tok, int H, int dk, int dv, int K, int in_dtype,
                        const void *q, const void *k, const void *v, const float *conv_w,
                        const void *a_logit, const void *b_logit, const float *A,
                        const float *b_alpha, const void *z, const float *norm_w,
                        const float *S0, const int32_t *cu_seqlens, const double *d_out,
                        const double *d_S_final, double *dq, double *dk_out, double *dv_out,
                        double *d_conv_w, double *d_a, double *d_b, double *d_A,
                        double *d_b_alpha, double *d_z, double *d_norm_w, double *d_S0,
                        int n_threads)
{
    if (n_seq <= 0 || n_tok < 0 || H <= 0 || dk <= 0 || dv <= 0 || K <= 0)
        return -1;
    if (!cu_seqlens && n_tok % n_seq != 0)
        return -1;
    set_threads(n_threads);
    const size_t C = (size_t)H * (2 * dk + dv);
    const long pairs = (long)n_seq * H;
    /* per (sequence, head) partial sums of the parameter gradients */
    double *part_w = calloc((size_t)pairs * (2 * dk + dv) * K, sizeof(double));
    double *part_norm = calloc((size_t)pairs * dv, sizeof(double));
    double *part_A = calloc((size_t)pairs, sizeof(double));
    double *part_ba = calloc((size_t)pairs, sizeof(double));
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long ph = 0; ph < pairs; ++ph) {
        const int n = (int)(ph / H), h = (int)(ph % H);
        const long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * (n_tok / n_seq);
        const long t1 = cu_seqlens ? cu_seqlens[n + 1] : (long)(n + 1) * (n_tok / n_seq);
        if (t0 < 0 || t1 < t0 || t1 > n_tok) {
            bad = 1;
            continue;
        }
        const long T = t1 - t0;
        const int wd[3] = {dk, dk, dv};
        const void *src[3] = {q, k, v};
        const size_t row_elems[3] = {(size_t)H * dk, (size_t)H * dk, (size_t)H * dv};
        const size_t col[3] = {(size_t)h * dk, (size_t)h * dk, (size_t)h * dv};
        const size_t chan[3] = {(size_t)h * dk, (size_t)H * dk + (size_t)h * dk,
                                (size_t)2 * H * dk + (size_t)h * dv};
        /* forward, keeping what the reverse sweep needs */
        double *x[3], *u[3], *dx[3];
        for (int s = 0; s < 3; ++s) {
            x[s] = malloc(sizeof(double) * (size_t)(T ? T : 1) * wd[s]);    /* conv outputs */
            u[s] = malloc(sizeof(double) * (size_t)(T ? T : 1) * wd[s]);    /* SiLU(x), normalised for q, k */
            dx[s] = calloc((size_t)(T ? T : 1) * wd[s], sizeof(double));     /* gradient of x */
        }
        double *rho = malloc(sizeof(double) * (size_t)(T ? T : 1) * 2);     /* L2Norm factors of q, k */
        double *al = malloc(sizeof(double) * (size_t)(T ? T : 1)), *be = malloc(sizeof(double) * (size_t)(T ? T : 1));
        double *gl = malloc(sizeof(double) * (size_t)(T ? T : 1)), *ain = malloc(sizeof(double) * (size_t)(T ? T : 1));
        double *P = malloc(sizeof(double) * (size_t)(T ? T : 1) * dk * dv);  /* state before each token */
        double *E = malloc(sizeof(double) * (size_t)(T ? T : 1) * dv);       /* e of each token */
        double *Y = malloc(sizeof(double) * (size_t)(T ? T : 1) * dv);       /* y of each token */
        double *S = calloc((size_t)dk * dv, sizeof(double));
        if (S0)
            for (size_t i = 0; i < (size_t)dk * dv; ++i)
                S[i] = (double)S0[((size_t)n * H + h) * dk * dv + i];
        const double eA = exp((double)A[h]);
        for (long t = 0; t < T; ++t) {
            const long tt = t0 + t;
            for (int s = 0; s < 3; ++s) {
                shortconv_prefill(src[s], in_dtype, row_elems[s], col[s], conv_w, chan[s], K, tt,
                                  t0, wd[s], x[s] + (size_t)t * wd[s]);
                for (int i = 0; i < wd[s]; ++i)
                    u[s][(size_t)t * wd[s] + i] = silu(x[s][(size_t)t * wd[s] + i]);
            }
            for (int s = 0; s < 2; ++s) {
                double ss = 0.0;
                for (int i = 0; i < dk; ++i)
                    ss += u[s][(size_t)t * dk + i] * u[s][(size_t)t * dk + i];
                rho[t * 2 + s] = 1.0 / sqrt(ss + ORACLE_EPS);
            }
            const size_t gi = (size_t)tt * H + h;
            ain[t] = load_elem(a_logit, in_dtype, gi) + (double)b_alpha[h];
            gl[t] = -eA * softplus(ain[t]);
            al[t] = exp(gl[t]);
            be[t] = write_gate(load_elem(b_logit, in_dtype, gi));
            double qh[dk], kh[dk];
            for (int i = 0; i < dk; ++i) {
                qh[i] = u[0][(size_t)t * dk + i] * rho[t * 2];
                kh[i] = u[1][(size_t)t * dk + i] * rho[t * 2 + 1];
            }
            memcpy(P + (size_t)t * dk * dv, S, sizeof(double) * dk * dv);
            delta_rule_step(S, dk, dv, qh, kh, u[2] + (size_t)t * dv, al[t], be[t],
                            E + (size_t)t * dv, Y + (size_t)t * dv);
        }
        /* reverse sweep */
        double *D = calloc((size_t)dk * dv, sizeof(double));
        double *St = malloc(sizeof(double) * (size_t)dk * dv);
        if (d_S_final)
            memcpy(D, d_S_final + ((size_t)n * H + h) * dk * dv, sizeof(double) * dk * dv);
        for (long t = T - 1; t >= 0; --t) {
            const long tt = t0 + t;
            const size_t gi = (size_t)tt * H + h;
            const double *Pt = P + (size_t)t * dk * dv, *e = E + (size_t)t * dv, *y = Y + (size_t)t * dv;
            const double alpha = al[t], beta = be[t];
            double qh[dk], kh[dk], dy[dv], dqh[dk], dkh[dk], de[dv], De[dk];
            for (int i = 0; i < dk; ++i) {
                qh[i] = u[0][(size_t)t * dk + i] * rho[t * 2];
                kh[i] = u[1][(size_t)t * dk + i] * rho[t * 2 + 1];
            }
            /* output stage */
            double ms = 0.0, dny = 0.0;
            for (int j = 0; j < dv; ++j)
                ms += y[j] * y[j];
            const double r = 1.0 / sqrt(ms / dv + ORACLE_EPS);
            double dn[dv];
            for (int j = 0; j < dv; ++j) {
                const double zj = load_elem(z, in_dtype, gi * dv + j), sz = sigmoid(zj);
                const double doj = d_out[gi * dv + j], nj = y[j] * r, gain = 1.0 + (double)norm_w[j];
                d_z[gi * dv + j] = doj * nj * gain * sz * (1.0 - sz);
                part_norm[(size_t)ph * dv + j] += doj * sz * nj;
                dn[j] = doj * sz * gain;
                dny += dn[j] * y[j];
            }
            for (int j = 0; j < dv; ++j)
                dy[j] = r * dn[j] - r * r * r * y[j] * dny / dv;
            /* the update */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    St[(size_t)i * dv + j] = alpha * Pt[(size_t)i * dv + j] + beta * kh[i] * e[j];
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    D[(size_t)i * dv + j] += qh[i] * dy[j];
            for (int i = 0; i < dk; ++i) {
                double s = 0.0;
                for (int j = 0; j < dv; ++j)
                    s += St[(size_t)i * dv + j] * dy[j];
                dqh[i] = s;
            }
            for (int j = 0; j < dv; ++j) {
                double s = 0.0;
                for (int i = 0; i < dk; ++i)
                    s += D[(size_t)i * dv + j] * kh[i];
                de[j] = beta * s;
            }
            double dbeta = 0.0, dalpha = 0.0;
            for (int i = 0; i < dk; ++i) {
                double s = 0.0, pde = 0.0;
                for (int j = 0; j < dv; ++j) {
                    s += D[(size_t)i * dv + j] * e[j];
                    pde += Pt[(size_t)i * dv + j] * de[j];
                }
                De[i] = s;
                dbeta += kh[i] * s;
                dkh[i] = beta * s - alpha * pde;
                dalpha -= kh[i] * pde;
            }
            for (size_t i = 0; i < (size_t)dk * dv; ++i)
                dalpha += D[i] * Pt[i];
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    D[(size_t)i * dv + j] = alpha * D[(size_t)i * dv + j] - alpha * kh[i] * de[j];
            /* gates */
            const double dg = alpha * dalpha;
            const double da = dg * (-eA) * sigmoid(ain[t]);
            d_a[gi] = da;
            part_A[ph] += dg * gl[t];
            part_ba[ph] += da;
            d_b[gi] = dbeta * beta * (1.0 - beta);
            /* L2Norm and SiLU of q, k; SiLU of v */
            const double *dxh[2] = {dqh, dkh};
            for (int s = 0; s < 2; ++s) {
                const double *uu = u[s] + (size_t)t * dk, rh = rho[t * 2 + s];
                double dot = 0.0;
                for (int i = 0; i < dk; ++i)
                    dot += uu[i] * dxh[s][i];
                for (int i = 0; i < dk; ++i) {
                    const double du = rh * dxh[s][i] - rh * rh * rh * uu[i] * dot;
                    dx[s][(size_t)t * dk + i] = du * dsilu(x[s][(size_t)t * dk + i]);
                }
            }
            for (int j = 0; j < dv; ++j)
                dx[2][(size_t)t * dv + j] = de[j] * dsilu(x[2][(size_t)t * dv + j]);
        }
        if (d_S0)
            memcpy(d_S0 + ((size_t)n * H + h) * dk * dv, D, sizeof(double) * dk * dv);
        /* ShortConv */
        double *outs[3] = {dq, dk_out, dv_out};
        for (int s = 0; s < 3; ++s) {
            for (long t = 0; t < T; ++t)
                for (int i = 0; i < wd[s]; ++i)
                    outs[s][((size_t)(t0 + t)) * row_elems[s] + col[s] + i] = 0.0;
            for (long t = 0; t < T; ++t)
                for (int i = 0; i < wd[s]; ++i) {
                    const double g = dx[s][(size_t)t * wd[s] + i];
                    const size_t c = chan[s] + i;
                    for (int j = 0; j < K; ++j) {
                        const long srct = t - (K - 1) + j;
                        if (srct < 0)
                            continue;
                        const size_t si = (size_t)(t0 + srct) * row_elems[s] + col[s] + i;
                        outs[s][si] += (double)conv_w[c * K + j] * g;
                        const size_t li = (s == 0 ? 0 : s == 1 ? (size_t)dk : (size_t)2 * dk) + i;
                        part_w[((size_t)ph * (2 * dk + dv) + li) * K + j] += g * load_elem(src[s], in_dtype, si);
                    }
                }
        }
        for (int s = 0; s < 3; ++s) {
            free(x[s]);
            free(u[s]);
            free(dx[s]);
        }
        free(rho); free(al); free(be); free(gl); free(ain);
        free(P); free(E); free(Y); free(S); free(D); free(St);
    }
    if (!bad) {
        memset(d_conv_w, 0, sizeof(double) * C * K);
        memset(d_norm_w, 0, sizeof(double) * dv);
        memset(d_A, 0, sizeof(double) * H);
        memset(d_b_alpha, 0, sizeof(double) * H);
        for (long ph = 0; ph < pairs; ++ph) {
            const int h = (int)(ph % H);
            const size_t chan[3] = {(size_t)h * dk, (size_t)H * dk + (size_t)h * dk,
                                    (size_t)2 * H * dk + (size_t)h * dv};
            for (int li = 0; li < 2 * dk + dv; ++li) {
                const size_t c = li < dk ? chan[0] + li : li < 2 * dk ? chan[1] + (li - dk) : chan[2] + (li - 2 * dk);
                for (int j = 0; j < K; ++j)
                    d_conv_w[c * K + j] += part_w[((size_t)ph * (2 * dk + dv) + li) * K + j];
            }
            for (int j = 0; j < dv; ++j)
                d_norm_w[j] += part_norm[(size_t)ph * dv + j];
            d_A[h] += part_A[ph];
            d_b_alpha[h] += part_ba[ph];
        }
    }
    free(part_w);
    free(part_norm);
    free(part_A);
    free(part_ba);
    return bad ? -1 : 0;
}

/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet (GDN) token mixer.
 *
 * The operation (web write-ups of "On the Design of Qwen3.8-Next Architecture"):
 *   paper.rainbus.top digest, 方法步骤详情 step (1), and the slinene.github.io
 *   write-up, 模块 A — Gated DeltaNet 混合层 (递归状态, 参数化):
 *
 *   q_t = L2Norm(SiLU(ShortConv(q_raw)))    k_t = L2Norm(SiLU(ShortConv(k_raw)))
 *   v_t = SiLU(ShortConv(v_raw))
 *   beta_t  = sigmoid(b_logit_t)
 *   alpha_t = exp(-exp(A_h) * softplus(a_logit_t + b_alpha_h))
 *   S_t = alpha_t S_{t-1};  e_t = v_t - S_t^T k_t;  S_t += beta_t k_t e_t^T
 *         (= alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T)
 *   y_t = S_t^T q_t
 *   out_t = sigmoid(z_t) * y_t / sqrt(mean(y_t^2) + eps) * (1 + norm_w)
 *
 * per head h, with the state S in R^{dk x dv} (the transposed convention of the
 * write-up), stored row-major [dk][dv] in fp32.  Readings where the pages are
 * silent: ShortConv is a causal depthwise cross-correlation of width conv_k
 * (tap conv_k-1 multiplies the current token), no bias, zero history at each
 * sequence start; eps = 1e-6 in both L2Norm (x / sqrt(sum x^2 + eps)) and
 * RMSNorm; the zero-centred RMSNorm gain is (1 + norm_w); no scale on q.
 *
 * Conventions shared by every call:
 *   - Every pointer is a DEVICE pointer unless stated otherwise; the caller
 *     allocates and frees all buffers it passes.
 *   - Token tensors are packed [N_tok, H, d] row-major (d fastest); gate
 *     logits are [N_tok, H]; conv weights are [H*(2*dk+dv), conv_k] fp32 with
 *     channels ordered [q heads | k heads | v heads]: channel h*dk+i of q,
 *     H*dk + h*dk+i of k, 2*H*dk + h*dv+i of v.
 *   - in_dtype applies to q, k, v, z, a_logit, b_logit (and the decode conv
 *     history); out_dtype to out.  Parameters and states are fp32.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     Arguments are validated on the host before anything is launched; an
 *     invalid call returns an error and launches nothing.  Faults of a kernel
 *     surface at the caller's next synchronisation, as with any CUDA launch.
 *   - Tensors read or written in vectors (q, k, v, z, conv_w, S0, S_final, S,
 *     conv_hist, out) must be 16-byte aligned (GDN_ERR_ALIGNMENT otherwise);
 *     the per-token gate logits, A, b_alpha, norm_w and cu_seqlens need only
 *     the alignment of their element type.
 *   - Supported sizes: dk, dv in {64, 128}; conv_k = 4 (GDN_ERR_UNSUPPORTED
 *     otherwise).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* NULL where a buffer is required, bad sizes */
    GDN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head dim, conv width, dtype) */
    GDN_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    GDN_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 5       /* a bounded device-side wait expired */
} gdn_status_t;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype_t;

typedef struct {
    int32_t num_seqs;      /* sequences in the batch (decode: batch size B) */
    int32_t total_tokens;  /* packed tokens N_tok (decode: must equal num_seqs) */
    int32_t H;             /* heads */
    int32_t dk, dv;        /* key / value head dims */
    int32_t conv_k;        /* ShortConv width */
    gdn_dtype_t in_dtype;  /* q, k, v, z, gate logits */
    gdn_dtype_t out_dtype; /* out */
} gdn_dims_t;

/*
 * gdn_prefill -- the whole mixer over a packed batch of sequences.
 *
 *   q, k       [N_tok, H, dk]   raw (pre-conv) projections, in_dtype
 *   v, z       [N_tok, H, dv]   raw value projection and output-gate logits
 *   conv_w     [H(2dk+dv), conv_k] fp32
 *   a_logit    [N_tok, H]       decay-gate logits (W_alpha x), in_dtype
 *   b_logit    [N_tok, H]       write-gate logits (W_beta x), in_dtype
 *   A, b_alpha [H] fp32         per-head decay parameters
 *   norm_w     [dv] fp32        zero-centred RMSNorm weight (gain 1 + w)
 *   S0         [N_seq, H, dk, dv] fp32 initial states, or NULL for zeros
 *   cu_seqlens [N_seq + 1] int32 DEVICE prefix offsets (cu[0] = 0, non-
 *              decreasing, cu[N_seq] = N_tok; empty sequences allowed), or
 *              NULL for N_seq equal lengths N_tok / N_seq.  Not checked on the
 *              device: a malformed array is undefined behaviour.
 *   out        [N_tok, H, dv]   out_dtype, written
 *   S_final    [N_seq, H, dk, dv] fp32 final states, written (may alias S0;
 *              may be NULL when not wanted)
 *
 * Each sequence starts with an empty conv history.  `out` must not alias any
 * input.  Any finite decay logit is accepted: on the tensor-core path the
 * log-decay -exp(A) softplus(a_logit + b_alpha) is clamped below at -128, where
 * exp() of it is already exactly 0 in fp32, so a logit that makes it overflow to
 * -inf (near 3e38 / exp(A)) gives alpha = 0 as in exact arithmetic instead of
 * NaN.  On the tensor-core path (bf16 inputs, dk = 128) a call with
 * dk = dv = 128 and at most as many (sequence, head) pairs as the device has
 * SMs (and at most 256) runs as one cooperative persistent kernel on `stream`
 * (one CTA per SM; with cu_seqlens after a one-CTA kernel that builds its task
 * list on the device); other long inputs
 * run in chunk segments whose kernels overlap on `stream` and on two
 * library-owned streams of the same device, forked from and joined back into
 * `stream` with events, so work queued on `stream` afterwards sees the results.  When
 * total_tokens is 0 the token tensors (q, k, v, z, a_logit, b_logit, out) may
 * be NULL and the call only writes S_final = S0 (or zeros).  The call takes a
 * stream-ordered workspace of
 * gdn_prefill_workspace_size() bytes from a private CUDA memory pool of the
 * current device and returns it to the pool on the same stream.
 */
GDN_API gdn_status_t gdn_prefill(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                         const float *conv_w, const void *a_logit, const void *b_logit,
                         const float *A, const float *b_alpha, const void *z,
                         const float *norm_w, const float *S0, const int32_t *cu_seqlens,
                         void *out, float *S_final, gdn_stream_t stream);

/* Bytes of device workspace one gdn_prefill call with these dims uses (host call). */
GDN_API gdn_status_t gdn_prefill_workspace_size(const gdn_dims_t *dims, size_t *bytes);

/*
 * gdn_prefill_ws -- gdn_prefill with the workspace supplied by the caller, so
 * that the call allocates no memory at all.  Same arguments and results as
 * gdn_prefill (the same kernels run; the results are bit-identical), plus
 *   workspace        device buffer of at least gdn_prefill_workspace_size()
 *                    bytes, 256-byte aligned (may be NULL when that size is 0)
 *   workspace_bytes  its size
 * The call reads and writes the workspace on `stream`; the caller must not use
 * it for anything else until that work is done.  Its contents need no
 * initialisation and are meaningless afterwards.  A workspace that is NULL or
 * too small returns GDN_ERR_INVALID_ARG, a misaligned one GDN_ERR_ALIGNMENT,
 * both before any launch.
 */
GDN_API gdn_status_t gdn_prefill_ws(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                                    const float *conv_w, const void *a_logit, const void *b_logit,
                                    const float *A, const float *b_alpha, const void *z,
                                    const float *norm_w, const float *S0, const int32_t *cu_seqlens,
                                    void *out, float *S_final, void *workspace, size_t workspace_bytes,
                                    gdn_stream_t stream);

/*
 * gdn_prefill_conv_tail -- the ShortConv history that continues each prefilled
 * sequence in decode: the causal depthwise convolution (slinene.github.io
 * write-up of "On the Design of Qwen3.8-Next Architecture", 模块 A, 参数化) looks
 * back conv_k - 1 = 3 raw tokens, and gdn_decode_step reads them from its
 * history buffer.
 *   q, k, v, cu_seqlens  as for gdn_prefill (raw, pre-conv projections)
 *   conv_hist  [N_seq, 3, H(2dk + dv)] in_dtype, written: row j of sequence n is
 *              the raw token cu[n+1] - 3 + j as [q heads | k heads | v heads],
 *              or zeros where that token lies before the sequence's start.
 * With this history and S_final of gdn_prefill as the state, gdn_decode_step on
 * the following tokens continues every sequence exactly as a longer prefill
 * would.  One kernel on `stream`; no workspace.
 */
GDN_API gdn_status_t gdn_prefill_conv_tail(const gdn_dims_t *dims, const void *q, const void *k,
                                           const void *v, const int32_t *cu_seqlens, void *conv_hist,
                                           gdn_stream_t stream);

/*
 * gdn_prefill_backward -- gradients of L = <d_out, out> + <d_S_final, S_final>
 * for the gdn_prefill call with the same arguments, with respect to every
 * input: the reverse-mode derivative of the forward the two web write-ups
 * define (slinene.github.io write-up of "On the Design of Qwen3.8-Next
 * Architecture", 模块 A: 递归状态, 参数化; paper.rainbus.top digest, 方法步骤详情
 * step (1)).  Per token, with P the state before it, e = v - alpha P^T k and D
 * the gradient of the state after it: D += q dy^T, dv = beta D^T k,
 * dk = beta D e - alpha P dv, dq = S dy, dbeta = k^T D e,
 * dalpha = <D, P> - k^T P dv, and the state before receives alpha (D - k dv^T);
 * then the gates, L2Norm, SiLU and the short convolution in reverse.
 *
 * Forward inputs as gdn_prefill (q, k, v, z, a_logit, b_logit in fp32 here:
 * dims->in_dtype and dims->out_dtype must be GDN_F32; dk = dv in {64, 128}).
 *   d_out      [N_tok, H, dv] fp32 gradient of out
 *   d_S_final  [N_seq, H, dk, dv] fp32 gradient of S_final, or NULL for zeros
 * Written, fp32, same shapes as the inputs they belong to:
 *   dq, dk [N_tok, H, dk]; dv, d_z [N_tok, H, dv]; d_a_logit, d_b_logit
 *   [N_tok, H]; d_conv_w [H(2dk+dv), 4]; d_A, d_b_alpha [H]; d_norm_w [dv];
 *   d_S0 [N_seq, H, dk, dv], or NULL when not wanted.
 * Token tensors may be NULL only when total_tokens is 0; every pointer 16-byte
 * aligned except the [H] and [N_tok, H] arrays (4-byte).  No output may alias an
 * input.  The results do not depend on scheduling (every sum has a fixed order).
 * The call recomputes the forward (states checkpointed every 16 tokens) and takes
 * a stream-ordered workspace of gdn_prefill_backward_workspace_size() bytes from
 * the library's private pool of the current device, returned on `stream`.
 * GDN_ERR_UNSUPPORTED for bf16 tensors or dk != dv.
 */
GDN_API gdn_status_t gdn_prefill_backward(
    const gdn_dims_t *dims, const void *q, const void *k, const void *v, const float *conv_w,
    const void *a_logit, const void *b_logit, const float *A, const float *b_alpha, const void *z,
    const float *norm_w, const float *S0, const int32_t *cu_seqlens, const void *d_out,
    const float *d_S_final, void *dq, void *dk, void *dv, float *d_conv_w, void *d_a_logit,
    void *d_b_logit, float *d_A, float *d_b_alpha, void *d_z, float *d_norm_w, float *d_S0,
    gdn_stream_t stream);

/* Bytes of device workspace one gdn_prefill_backward call with these dims uses (host call). */
GDN_API gdn_status_t gdn_prefill_backward_workspace_size(const gdn_dims_t *dims, size_t *bytes);

/*
 * gdn_qsa_indexer -- the compressed lightweight indexer of Qwen Sparse Attention
 * (slinene.github.io write-up of "On the Design of Qwen3.8-Next Architecture",
 * 模块 B: "压缩轻量 indexer" and the block selection paragraph), for `batch`
 * independent sequences of n tokens:
 *   q_i^h   = PRoPE(RMSNorm(q[i, h]) * w_q, i)          (h < heads = 4)
 *   k_bar_b = PRoPE(RMSNorm(mean(k[4b .. 4b+3])) * w_k, 4b)   (b < n / 4)
 *   I_ib    = sum_h ReLU(<q_i^h, k_bar_b>) for complete blocks (4b + 3 <= i)
 *   sel[i]  = the budget / 4 highest-scoring complete blocks, ties to the smaller
 *             block index, in ascending order, padded with -1.
 * RMSNorm: x / sqrt(mean x^2 + 1e-6) times the weight; PRoPE rotates dims [0, 64)
 * in pairs (j, j + 32) by p * 10000^(-j / 32), dims [64, 128) unchanged.  The
 * token set of query i is the selected blocks expanded to tokens plus the tail
 * 4 floor((i + 1) / 4) .. i.
 *
 *   q       [batch, n, 4, 128] bf16 (the per-head projections W_Q^h x_i)
 *   k       [batch, n, 128] bf16    (the shared key projection W_K x_i)
 *   w_q, w_k [128] fp32             RMSNorm weights
 *   sel     [batch, n, budget / 4] int32, written
 *   scores  [batch, n, n / 4] fp32: if non-NULL the block scores are written
 *           there (entries of incomplete blocks are left untouched); NULL keeps
 *           them in the workspace.
 * Supported: heads = 4, d = 128, block = 4, budget a multiple of 4.  The scores
 * are tcgen05 products of fp16-rounded rotated rows with fp32 accumulation.  The
 * call takes a stream-ordered workspace of gdn_qsa_indexer_workspace_size()
 * bytes (the fp16 rows and, unless `scores` is given, the score matrix) from the
 * library's pool.  n = 0 writes nothing.
 */
GDN_API gdn_status_t gdn_qsa_indexer(int batch, int n, int heads, int d, int block, int budget, const void *q,
                                     const void *k, const float *w_q, const float *w_k, int32_t *sel,
                                     float *scores, gdn_stream_t stream);

/* Bytes of device workspace one gdn_qsa_indexer call uses (host call). */
GDN_API gdn_status_t gdn_qsa_indexer_workspace_size(int batch, int n, size_t *bytes);

/*
 * gdn_layer_forward -- the GDN layer from the hidden states to the output
 * projection (slinene.github.io write-up of "On the Design of Qwen3.8-Next
 * Architecture", 模块 A, 参数化: q, k, v, z and the two gate logits are linear
 * projections of x, and o = W_o[sigmoid(z) RMSNorm(y)]):
 *   [q | k | v | z | a | b] = x W_in,  out = gdn_prefill(...),  y = out W_o.
 *   x      [N_tok, d_model] bf16
 *   w_in   [d_model, H(2dk + 2dv) + 2H] bf16, row-major; column blocks q [H dk],
 *          k [H dk], v [H dv], z [H dv], a [H], b [H]
 *   w_o    [H dv, d_model] bf16, row-major
 *   y      [N_tok, d_model] bf16, written
 * and the mixer's parameters as gdn_prefill (dims->in_dtype and out_dtype must be
 * GDN_BF16; d_model a multiple of 8, else GDN_ERR_UNSUPPORTED).  The projections
 * are stored in bf16 between the steps.
 * The GEMM steps are bf16 products with fp32 accumulation on the library's own
 * tcgen05 GEMM kernel; they are not fused with the mixer's prelude.  Stateless
 * apart from the workspace, so threads may run layers at the same time.
 * Stream-ordered workspace from the library's pool: gdn_layer_workspace_size()
 * bytes.  An expired wait inside a GEMM raises GDN_ERRF_GEMM.
 */
GDN_API gdn_status_t gdn_layer_forward(const gdn_dims_t *dims, int d_model, const void *x, const void *w_in,
                                       const float *conv_w, const float *A, const float *b_alpha,
                                       const float *norm_w, const void *w_o, const float *S0,
                                       const int32_t *cu_seqlens, void *y, float *S_final, gdn_stream_t stream);

/* Bytes of device workspace one gdn_layer_forward call uses, the mixer's included (host call). */
GDN_API gdn_status_t gdn_layer_workspace_size(const gdn_dims_t *dims, int d_model, size_t *bytes);

/*
 * gdn_gemm_bf16 -- C [M, N] = A [M, K] B [K, N], the product the layer's
 * projections use (slinene.github.io write-up of "On the Design of Qwen3.8-Next
 * Architecture", 模块 A, 参数化: q, k, v, z and the gate logits are linear maps of
 * the hidden state), on the library's tcgen05 GEMM: bf16 row-major operands with
 * leading dimensions lda, ldb, ldc (elements), fp32 accumulation, C rounded to
 * bf16 (round to nearest even).  K, lda and ldc multiples of 8; for N >= 64 also
 * ldb; A, B and C 16-byte aligned (else GDN_ERR_ALIGNMENT; other violations
 * GDN_ERR_INVALID_ARG).  N < 64 takes a stream-ordered workspace from the
 * library's pool (B transposed).  M = 0 or N = 0 writes nothing.  An expired
 * wait raises GDN_ERRF_GEMM.  Asynchronous on `stream`.
 */
GDN_API gdn_status_t gdn_gemm_bf16(int M, int N, int K, const void *A, int lda, const void *B, int ldb, void *C,
                                   int ldc, gdn_stream_t stream);

/*
 * gdn_decode_step -- one token for each of B = dims->num_seqs sequences,
 * reading and updating the per-head state in place.
 *
 *   q, k       [B, H, dk]; v, z [B, H, dv]; a_logit, b_logit [B, H]  (in_dtype)
 *   conv_w, A, b_alpha, norm_w   as for gdn_prefill
 *   conv_hist  [B, conv_k-1, H(2dk+dv)] in_dtype, in/out: the raw (pre-conv)
 *              q|k|v channels of the previous conv_k-1 tokens, oldest first.
 *              The step convolves [hist, current], then shifts the history by
 *              one so the current raw token becomes the newest entry.  Zeros
 *              mean "no history" (a fresh sequence).
 *   S          [B, H, dk, dv] fp32, in/out (updated in place)
 *   out        [B, H, dv] out_dtype, written
 *
 * dims->total_tokens must equal dims->num_seqs.  No workspace is used.
 */
GDN_API gdn_status_t gdn_decode_step(const gdn_dims_t *dims, const void *q, const void *k,
                             const void *v, const float *conv_w, void *conv_hist,
                             const void *a_logit, const void *b_logit, const float *A,
                             const float *b_alpha, const void *z, const float *norm_w, float *S,
                             void *out, gdn_stream_t stream);

/*
 * gdn_decode_multi -- T consecutive tokens (1 <= T <= 4) for each of
 * B = dims->num_seqs sequences in one step: the verification step of
 * speculative decoding, where a draft of several tokens is checked by the
 * backbone in parallel (the digest's 前置知识, on multi-token prediction).  The
 * state is read once and written at most once for all T tokens.
 *
 *   q, k       [B, T, H, dk]; v, z [B, T, H, dv]; a_logit, b_logit [B, T, H] (bf16)
 *   conv_w, A, b_alpha, norm_w   as for gdn_prefill
 *   conv_hist  [B, 3, H(2dk+dv)] bf16, in/out, as for gdn_decode_step
 *   S          [B, H, dk, dv] fp32, in/out
 *   out        [B, T, H, dv] out_dtype, written for all T tokens
 *   n_keep     [B] int32 device array or NULL (NULL = T for every sequence):
 *              the number of leading tokens of sequence b committed to S and
 *              conv_hist (values outside [0, T] are clamped).  n_keep[b] = 0
 *              leaves both untouched (the state is not written at all).
 *
 * out is exactly what T successive gdn_decode_step calls would produce; S and
 * conv_hist end as after the first n_keep[b] of those calls.  A verifier can
 * run the draft with n_keep = 0 and commit the accepted prefix with a second
 * call of those tokens.  dims->total_tokens must equal B * T.  Supported:
 * in_dtype = GDN_BF16, dk = dv = 128 (GDN_ERR_UNSUPPORTED otherwise); T outside
 * [1, 4] is GDN_ERR_INVALID_ARG.  No workspace is used.
 */
GDN_API gdn_status_t gdn_decode_multi(const gdn_dims_t *dims, int T, const void *q, const void *k,
                                      const void *v, const float *conv_w, void *conv_hist,
                                      const void *a_logit, const void *b_logit, const float *A,
                                      const float *b_alpha, const void *z, const float *norm_w,
                                      float *S, void *out, const int32_t *n_keep, gdn_stream_t stream);

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is an interface choice of the
 * library.  Callers that may not call cudaMalloc or any allocator while they
 * run the layer (code inside host callbacks or allocation-free regions,
 * embedders whose device memory is partitioned up-front by another runtime,
 * real-time paths that must not take an allocator lock or fail with
 * out-of-memory mid-request) cannot use gdn_prefill, which takes its workspace
 * from a memory pool.  This call takes the same arguments and runs the same
 * tensor-core kernels, with the workspace in a fixed array of
 * GDN_NOALLOC_SCRATCH_BYTES inside the library's device memory; it allocates
 * nothing.  The caller still allocates every input and output.
 *
 *   - Supported: in_dtype = GDN_BF16, dk = 128, dv in {64, 128}, conv_k = 4
 *     (GDN_ERR_UNSUPPORTED otherwise).
 *   - Size limit: the workspace of 3*dk*2 + dv*2 + 64*2 + 4 bytes per token
 *     and head (each of its six arrays rounded up to 256 bytes) must fit in
 *     GDN_NOALLOC_SCRATCH_BYTES, about 29,000 token-heads at dk = dv = 128;
 *     larger calls return GDN_ERR_INVALID_ARG and launch nothing.
 *   - The array exists once per GPU that loads the library, until exit.  The
 *     first call on a device looks up its device address and keeps it; make
 *     that first call before any stream capture, and do not use the library
 *     across a cudaDeviceReset() of that device (the kept address would be
 *     stale).
 *   - The profiling hooks gdn_set_timing_events and gdn_set_kernel_events
 *     record nothing for this call.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents (nothing in it must start at zero).  Calls whose GPU work
 *     overlaps, e.g. on two streams at once, race on it: serialise them.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (32u << 20)
GDN_API gdn_status_t gdn_prefill_noalloc(const gdn_dims_t *dims, const void *q, const void *k,
                                         const void *v, const float *conv_w, const void *a_logit,
                                         const void *b_logit, const float *A, const float *b_alpha,
                                         const void *z, const float *norm_w, const float *S0,
                                         const int32_t *cu_seqlens, void *out, float *S_final,
                                         gdn_stream_t stream);

/*
 * gdn_set_timing_events -- optional profiling hook (host call, not thread-safe).
 * When both handles are non-NULL (cudaEvent_t values), each following call
 * records `begin` and `end` on its stream: gdn_prefill around all of its GPU
 * work on the tensor-core path (whose kernels overlap on two streams) and around
 * the state recurrence on the fp32 path; gdn_decode_step around its kernel.
 * The hook stays until cleared with (NULL, NULL).  Recording adds no work to
 * the kernels; it lets a caller time the library's GPU work with CUDA events.
 */
GDN_API gdn_status_t gdn_set_timing_events(void *begin, void *end);

/*
 * gdn_set_kernel_events -- optional per-launch profiling hook (host call, not
 * thread-safe).  begin[i] / end[i] (cudaEvent_t values, created and owned by
 * the caller; the library copies the n handles) are recorded around launch
 * slot i of every following gdn_prefill / gdn_decode_step call, on the stream
 * that slot's kernel runs on.  Slots in launch order:
 *   gdn_prefill, tensor-core path with dk = dv = 128 and at most as many
 *     (sequence, head) pairs as the device has SMs (and at most 256): one slot,
 *     the fused persistent kernel, on the caller's stream; with cu_seqlens the
 *     slot also holds the one-CTA kernel that builds its task list, launched
 *     just before it (two launches, one slot);
 *   gdn_prefill, other tensor-core shapes, n segments: chunk_prep(0),
 *     chunk_chain(0), chunk_prep(1), chunk_chain(1), ... -- chunk_prep of even
 *     segments on the caller's stream, of odd segments on a second library
 *     stream, chunk_chain on the library's highest-priority stream;
 *   gdn_prefill, fp32 path: prelude, recurrent;
 *   gdn_decode_step: the decode kernel.
 * Slots beyond n are not recorded.  n = 0 clears the hook.  Returns
 * GDN_ERR_INVALID_ARG for n < 0 or a NULL handle among the first n.
 */
GDN_API gdn_status_t gdn_set_kernel_events(void *const *begin, void *const *end, int n);

/*
 * Number of kernels the calling thread's most recent gdn_prefill,
 * gdn_prefill_noalloc or gdn_decode_step call launched (0 after a call that
 * returned before its first launch).  Host-side count, no synchronisation.
 */
GDN_API int gdn_last_call_launches(void);

/*
 * Number of launch slots of the same call: the kernels, or groups of kernels,
 * that gdn_set_kernel_events brackets with one (begin, end) pair each.  Equal
 * to gdn_last_call_launches() except where a slot holds more than one kernel
 * (the fused prefill of a packed batch of unequal lengths: its task-list
 * builder and the fused kernel share one slot).  Host-side count.
 */
GDN_API int gdn_last_call_slots(void);

/*
 * Device error flags.  Every wait inside the kernels (on an mbarrier fed by TMA
 * or by the tensor cores) is bounded; when one expires the kernel raises its
 * family's device error word, gives up its remaining waits promptly and
 * returns, so a stuck transfer shows up as an error status instead of a hang.
 */
#define GDN_ERRF_PREP 1u    /* chunk_prep (gdn_prefill, tensor-core path) */
#define GDN_ERRF_CHAIN 2u   /* chunk_chain (gdn_prefill, tensor-core path) */
#define GDN_ERRF_DECODE 4u  /* streaming decode kernel (gdn_decode_step) */
#define GDN_ERRF_QSA 8u     /* QSA indexer score kernel (gdn_qsa_indexer) */
#define GDN_ERRF_GEMM 16u   /* projection GEMMs (gdn_layer_forward) */

/*
 * gdn_device_error_status -- reads the current device's error words into
 * *flags (a GDN_ERRF_* mask; may be NULL) and, when `clear` is non-zero, resets
 * them.  Synchronises `stream` (the reads are ordered after the work queued on
 * it).  Returns GDN_ERR_TIMEOUT when any flag is set, GDN_OK when none is,
 * GDN_ERR_CUDA if the reads fail.
 */
GDN_API gdn_status_t gdn_device_error_status(unsigned *flags, int clear, gdn_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
GDN_API const char *gdn_status_string(gdn_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */

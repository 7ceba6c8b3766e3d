// Internal launch interface between the host ABI layer and the kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

struct PrefillArgs {
    int n_seq, n_tok, H, dk, dv;
    bool in_bf16, out_bf16;
    const void *q, *k, *v, *z, *a_logit, *b_logit;
    const float *conv_w, *A, *b_alpha, *norm_w, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    cudaStream_t stream;
};

struct DecodeArgs {
    int B, H, dk, dv;
    bool in_bf16, out_bf16;
    const void *q, *k, *v, *z, *a_logit, *b_logit;
    const float *conv_w, *A, *b_alpha, *norm_w;
    void *conv_hist;
    float *S;
    void *out;
    cudaStream_t stream;
};

// K1: conv + SiLU + L2Norm into a workspace (fp32 for the SIMT chain, fp16 for
// the tensor-core chain).
cudaError_t launch_prelude_f32(const PrefillArgs &a, float *qn, float *kn, float *vn);
cudaError_t launch_prelude_f16(const PrefillArgs &a, __half *qn, __half *kn, __half *vn);

// Workspace of the tensor-core prefill (all token-indexed, [N_tok, H, *]).
struct TcWorkspace {
    __half *Qt, *Kt, *Wn;   // e^G q, e^{G_C - G} k, -W  [dk]
    __half *Up, *Aqk;       // U' [dv], decayed masked q.k [64]
    float *decay;           // e^{G_C} at the first token row of each chunk
};

// K2a (prelude fused) / K2b: chunked prefill on tcgen05 (dk = 128, dv in {64, 128}).
// The two-argument forms cover every chunk on a.stream, from a.S0 to a.S_final.
// The ranged forms cover chunks [c_lo, c_hi) of every sequence on `stream`; the
// chain carries the state from state_in (NULL: zeros) to state_out (NULL: dropped).
cudaError_t launch_chunk_prep(const PrefillArgs &a, const TcWorkspace &w);
// The fused persistent prefill (dk = dv = 128, few (sequence, head) pairs): chain
// CTAs and prep workers in one cooperative launch of one CTA per SM, ordered by
// per-chunk ready flags.  fused_chain_ctas returns its chain CTA count, or 0 when
// the shape does not suit it.  `ready` holds n_seq * H * ceil(n_tok / 64) + 1
// ints (flags and the task counter), zeroed by the launcher on `stream`.
int fused_chain_ctas(const PrefillArgs &a, int sms);
size_t fused_task_capacity(int n_tok, int n_seq, int H);
cudaError_t launch_prefill_fused(const PrefillArgs &a, const TcWorkspace &w, int *ready, int sms,
                                 cudaStream_t stream);
cudaError_t launch_chunk_chain(const PrefillArgs &a, const TcWorkspace &w);
cudaError_t launch_chunk_prep(const PrefillArgs &a, const TcWorkspace &w, int c_lo, int c_hi,
                              cudaStream_t stream);
cudaError_t launch_chunk_chain(const PrefillArgs &a, const TcWorkspace &w, int c_lo, int c_hi,
                               const float *state_in, float *state_out, cudaStream_t stream);

// Host side of TMA: a 3-D tiled tensor map over a token-indexed [N_tok][H][inner]
// tensor (16-bit elements), box {box_inner, 1, box_rows}.
struct TmaMap { alignas(64) unsigned char bytes[128]; };
cudaError_t make_tma_3d(TmaMap *out, const void *base, bool bf16, int inner, int H, int n_tok,
                        int box_inner, int box_rows, bool swizzle128);
cudaError_t make_tma_rows_f32(TmaMap *out, const void *base, int cols, int rows, int box_cols, int box_rows);
cudaError_t make_tma_mat_bf16(TmaMap *out, const void *base, int inner, int rows, int ld, int box_inner,
                              int box_rows);
cudaError_t make_tma_plain_bf16(TmaMap *out, const void *base, int rank, const long long *dims,
                                const long long *strides, const int *box);
// K7: C [M, N] = A [M, K] B [K, N], bf16 row-major with leading dimensions lda,
// ldb, ldc (elements; lda and K multiples of 8, A 16-byte aligned; for N >= 64
// also ldb a multiple of 8 and B 16-byte aligned), fp32 accumulation.  N < 64
// takes gemm_workspace_bytes(N, K) of 16-byte-aligned workspace (B transposed);
// N >= 64 none.
size_t gemm_workspace_bytes(int N, int K);
cudaError_t launch_gemm_bf16(int M, int N, int K, const void *A, int lda, const void *B, int ldb, void *C, int ldc,
                             void *ws, cudaStream_t stream);
cudaError_t gemm_error_word(unsigned *v, bool clear, cudaStream_t s);
cudaError_t gemm_wait_selftest(uint32_t max_polls, cudaStream_t s);

// K4: prefill backward (fp32 inputs, dk = dv in {64, 128}); `f` holds the forward's
// inputs (f.out and f.S_final are unused), the rest the incoming and outgoing
// gradients, all fp32.
struct BackwardArgs {
    PrefillArgs f;
    const void *d_out;
    const float *d_S_final;
    void *dq, *dk, *dv, *d_a_logit, *d_b_logit, *d_z;
    float *d_conv_w, *d_A, *d_b_alpha, *d_norm_w, *d_S0;
};
size_t backward_workspace_bytes(int n_seq, int n_tok, int H, int D);
cudaError_t launch_backward(const BackwardArgs &b, void *ws);

// K5: QSA compressed indexer (H = 4 heads of d = 128, blocks of 4 tokens): q
// [B, n, 4, 128] and k [B, n, 128] bf16, weights [128] fp32; sel [B, n, KB] int32;
// scores [B, n, n / 4] fp32 (NULL: kept in the workspace).
struct QsaArgs {
    int B, n, KB;
    const void *q, *k;
    const float *w_q, *w_k;
    int32_t *sel;
    float *scores;
    cudaStream_t stream;
};
size_t qsa_workspace_bytes(int B, int n);
size_t qsa_scores_bytes(int B, int n);
cudaError_t launch_qsa_indexer(const QsaArgs &a, void *ws);
cudaError_t qsa_error_word(unsigned *v, bool clear, cudaStream_t s);
cudaError_t qsa_wait_selftest(uint32_t max_polls, cudaStream_t s);

// K6: the layer from the hidden states (in-projection GEMMs, the mixer, W_o).
// x [N, d_model], w_in [d_model, H(2dk + 2dv) + 2H], w_o [H dv, d_model], y
// [N, d_model], all bf16; f carries the mixer's parameters (its token pointers
// are set by launch_layer).
struct LayerArgs {
    PrefillArgs f;
    int d_model;
    const void *x, *w_in, *w_o;
    void *y;
};
size_t layer_workspace_bytes(int n_tok, int H, int dk, int dv, int d_model);
cudaError_t launch_layer(const LayerArgs &L, void *ws, cudaError_t (*run_prefill)(const PrefillArgs &));

// K2f: token-by-token recurrence with the fused gates and output stage (SIMT fp32).
cudaError_t launch_recurrent(const PrefillArgs &a, const float *qn, const float *kn,
                             const float *vn);

// K3: one decode step (any supported dims / dtypes).
cudaError_t launch_decode(const DecodeArgs &a);
// K3s: the streaming decode step for bf16 inputs with dk = dv = 128.
bool decode_stream_supported(const DecodeArgs &a);
cudaError_t launch_decode_stream(const DecodeArgs &a);
// T (1..4) consecutive tokens per sequence: q, k, v, z, out [B, T, H, d], gate
// logits [B, T, H]; the state and history advance by n_keep[b] tokens (NULL: T).
cudaError_t launch_decode_stream(const DecodeArgs &a, int T, const int32_t *n_keep);

// SM count of the current device (queried once per device, then cached).
cudaError_t sm_count(int *out);

// Kernel-launch accounting for gdn_last_call_launches(): every launcher returns
// launched() right after its <<<...>>>, which counts the launch on this thread.
void note_launch();
void reset_launch_count();   // at the entry of every public call that launches
inline cudaError_t launched() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launch();
    return e;
}

// Device error words: a kernel family raises its word when one of its bounded
// waits expires.  *_error_word copies the word to *v (zeroing it when `clear`)
// and synchronises `s`; *_wait_selftest runs one CTA whose wait -- the family's
// own wait routine -- targets a barrier phase that nothing completes.
template <class Sym>
cudaError_t read_error_word(Sym &sym, unsigned *v, bool clear, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(v, sym, sizeof(unsigned), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && clear) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, sym);
        if (e == cudaSuccess) e = cudaMemsetAsync(p, 0, sizeof(unsigned), s);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e;
}
cudaError_t prep_error_word(unsigned *v, bool clear, cudaStream_t s);
cudaError_t chain_error_word(unsigned *v, bool clear, cudaStream_t s);
cudaError_t decode_error_word(unsigned *v, bool clear, cudaStream_t s);
cudaError_t prep_wait_selftest(uint32_t max_polls, cudaStream_t s);
cudaError_t chain_wait_selftest(uint32_t max_polls, cudaStream_t s);
cudaError_t decode_wait_selftest(uint32_t max_polls, cudaStream_t s);

}  // namespace gdn

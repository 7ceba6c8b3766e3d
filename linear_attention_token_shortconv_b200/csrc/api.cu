// Host side of the C ABI declared in include/gdn.h: argument validation,
// workspace management and kernel dispatch.  No kernel launches before every
// argument has been checked.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

using std::max;

#include "../../include/gdn.h"
#include "gdn_internal.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

gdn_status_t check_dims(const gdn_dims_t *d, bool decode) {
    if (!d) return GDN_ERR_INVALID_ARG;
    if (d->num_seqs <= 0 || d->total_tokens < 0 || d->H <= 0 || d->dk <= 0 || d->dv <= 0 ||
        d->conv_k <= 0)
        return GDN_ERR_INVALID_ARG;
    if ((d->in_dtype != GDN_F32 && d->in_dtype != GDN_BF16) ||
        (d->out_dtype != GDN_F32 && d->out_dtype != GDN_BF16))
        return GDN_ERR_INVALID_ARG;
    if (decode && d->total_tokens != d->num_seqs) return GDN_ERR_INVALID_ARG;
    if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128) || d->conv_k != 4)
        return GDN_ERR_UNSUPPORTED;
    // packed index arithmetic stays in 64 bits inside the kernels; keep the
    // per-tensor element counts within int64 and the token count within int32
    if ((int64_t)d->H * (2 * d->dk + d->dv) > (int64_t)1 << 30) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

size_t round_up(size_t x) { return (x + 255) & ~(size_t)255; }

// The chunked tensor-core path serves bf16 inputs with dk = 128; everything
// else (the fp32 workload, dk = 64) runs the fp32 token-by-token recurrence.
bool use_tensor_cores(const gdn_dims_t *d) { return d->in_dtype == GDN_BF16 && d->dk == 128; }

// Chunk segments of the tensor-core path.  Prep segments are independent of one
// another (each writes its own token rows of the workspace): they alternate
// between the caller's stream and a second stream, so segment s + 1 fills the
// SMs that segment s's last CTAs leave idle.  The chain kernel of segment s runs
// on a third, highest-priority stream after prep s and chain s - 1 (events);
// the state passes from one chain launch to the next through a state buffer.
// Segments cut the chunks of the longest sequence: N_tok / N_seq of them for
// equal lengths; with cu_seqlens the host does not know the longest, and the
// bound N_tok / 64 is used (launches past a sequence's end exit at once).  The
// workspace size takes the bound, so it covers both.
struct Segments {
    int seg, n;
};
Segments segments(const gdn_dims_t *d, bool equal_lengths = false) {
    const int longest = equal_lengths && d->num_seqs > 0 ? d->total_tokens / d->num_seqs : d->total_tokens;
    const int max_chunks = (longest + 63) / 64;
    Segments g;
    g.seg = max(8, (max_chunks + 15) / 16);
    g.n = max(1, (max_chunks + g.seg - 1) / g.seg);
    return g;
}

// Workspace: tensor-core path: Qt, Kt, -W [dk], U' [dv], Aqk [64] in fp16 and
// e^{G_C} in fp32 per token-head, the fused kernel's ready flags and task
// counter, plus an fp32 state buffer [N_seq, H, dk, dv]
// when the call runs in several segments; fp32 path: q_hat, k_hat, v_hat in fp32.
size_t workspace_bytes(const gdn_dims_t *d) {
    const size_t nt = (size_t)d->total_tokens * d->H;
    if (use_tensor_cores(d)) {
        // ready flags and the task counter, then the varlen task list, its count and
        // the item order
        const size_t flags = ((size_t)d->num_seqs * d->H * ((d->total_tokens + 63) / 64) + 1) * 4 +
                             (gdn::fused_task_capacity(d->total_tokens, d->num_seqs, d->H) + 1 +
                              (size_t)d->num_seqs * d->H) * 4;
        return 3 * round_up(nt * d->dk * 2) + round_up(nt * d->dv * 2) + round_up(nt * 64 * 2) +
               round_up(nt * 4) + round_up(flags) +
               (segments(d).n > 1 ? round_up((size_t)d->num_seqs * d->H * d->dk * d->dv * 4) : 0);
    }
    return 2 * round_up(nt * d->dk * sizeof(float)) + round_up(nt * d->dv * sizeof(float));
}

// One private stream-ordered pool per device; memory stays reserved between calls.
std::mutex g_pool_mu;
cudaMemPool_t g_pools[64] = {};

cudaError_t get_pool(cudaMemPool_t *pool) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_pool_mu);
    if (!g_pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p;
        e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        g_pools[dev] = p;
    }
    *pool = g_pools[dev];
    return cudaSuccess;
}

// Per-device side streams (chain: highest priority; prep2: default priority)
// and event pool for the segments.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaStream_t prep2 = nullptr;
    std::vector<cudaEvent_t> events;
};
std::mutex g_side_mu[64];
SideStream g_side[64];

// Returns the side stream of the current device with at least n events; the
// caller holds g_side_mu[dev] while it records and waits on them.
cudaError_t side_stream(int dev, int n, SideStream **out) {
    SideStream &ss = g_side[dev];
    cudaError_t e;
    if (!ss.stream) {
        int lo = 0, hi = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&lo, &hi)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&ss.stream, cudaStreamNonBlocking, hi)) != cudaSuccess)
            return e;
    }
    if (!ss.prep2) {
        if ((e = cudaStreamCreateWithFlags(&ss.prep2, cudaStreamNonBlocking)) != cudaSuccess) return e;
    }
    while ((int)ss.events.size() < n) {
        cudaEvent_t ev;
        if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        ss.events.push_back(ev);
    }
    *out = &ss;
    return cudaSuccess;
}

// profiling hook: events recorded around the dominant kernel of each call
cudaEvent_t g_ev_begin = nullptr, g_ev_end = nullptr;

cudaError_t record(cudaEvent_t ev, cudaStream_t s) {
    return ev ? cudaEventRecord(ev, s) : cudaSuccess;
}

// Per-launch timing hook (gdn_set_kernel_events): slot i of a call is recorded
// around that call's i-th kernel launch, on the stream the kernel runs on.
std::vector<cudaEvent_t> g_kev_begin, g_kev_end;
thread_local int tl_launches = 0;
thread_local int tl_slots = 0;   // launch slots of the calling thread's last call

template <class F>
cudaError_t slot_launch(int *slot, cudaStream_t s, F &&launch) {
    const int i = (*slot)++;
    ++tl_slots;
    const bool rec = i < (int)g_kev_begin.size();
    cudaError_t e = rec ? cudaEventRecord(g_kev_begin[i], s) : cudaSuccess;
    if (e == cudaSuccess) e = launch();
    if (e == cudaSuccess && rec) e = cudaEventRecord(g_kev_end[i], s);
    return e;
}

// The prefill after validation: workspace from the pool (ext_ws NULL) or the
// caller's buffer of at least workspace_bytes(), then the kernels.
cudaError_t prefill_run(const gdn::PrefillArgs &a, char *ext_ws) {
    gdn_dims_t dd;
    dd.num_seqs = a.n_seq;
    dd.total_tokens = a.n_tok;
    dd.H = a.H;
    dd.dk = a.dk;
    dd.dv = a.dv;
    dd.conv_k = 4;
    dd.in_dtype = a.in_bf16 ? GDN_BF16 : GDN_F32;
    dd.out_dtype = a.out_bf16 ? GDN_BF16 : GDN_F32;
    const gdn_dims_t *dims = &dd;
    const size_t nt = (size_t)a.n_tok * a.H;
    const size_t ws_bytes = workspace_bytes(dims);
    char *ws = ext_ws;
    const bool own_ws = ext_ws == nullptr && ws_bytes > 0;
    if (own_ws) {
        cudaMemPool_t pool;
        cudaError_t ep = get_pool(&pool);
        if (ep != cudaSuccess) return ep;
        if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), ws_bytes, pool, a.stream) !=
            cudaSuccess)
            return cudaErrorMemoryAllocation;
    }
    cudaError_t e;
    if (use_tensor_cores(dims)) {
        gdn::TcWorkspace w;
        char *p = ws;
        auto take = [&](size_t bytes) { char *r = p; p += round_up(bytes); return r; };
        w.Qt = reinterpret_cast<__half *>(take(nt * a.dk * 2));
        w.Kt = reinterpret_cast<__half *>(take(nt * a.dk * 2));
        w.Wn = reinterpret_cast<__half *>(take(nt * a.dk * 2));
        w.Up = reinterpret_cast<__half *>(take(nt * a.dv * 2));
        w.Aqk = reinterpret_cast<__half *>(take(nt * 64 * 2));
        w.decay = reinterpret_cast<float *>(take(nt * 4));
        int *ready = reinterpret_cast<int *>(take(((size_t)a.n_seq * a.H * ((a.n_tok + 63) / 64) + 1) * 4 +
                                                  (gdn::fused_task_capacity(a.n_tok, a.n_seq, a.H) + 1 +
                                                   (size_t)a.n_seq * a.H) * 4));
        const Segments g = segments(dims, a.cu_seqlens == nullptr);
        int slot = 0, sms = 0;
        e = record(g_ev_begin, a.stream);
        if (e == cudaSuccess) e = gdn::sm_count(&sms);
        if (e == cudaSuccess && gdn::fused_chain_ctas(a, sms) > 0) {
            // few (sequence, head) chains: one persistent launch, prep and chain
            // ordered by per-chunk flags
            e = slot_launch(&slot, a.stream, [&] { return gdn::launch_prefill_fused(a, w, ready, sms, a.stream); });
        } else if (g.n == 1) {
            if (e == cudaSuccess)
                e = slot_launch(&slot, a.stream, [&] { return gdn::launch_chunk_prep(a, w); });
            if (e == cudaSuccess)
                e = slot_launch(&slot, a.stream, [&] { return gdn::launch_chunk_chain(a, w); });
        } else {
            float *state = reinterpret_cast<float *>(take((size_t)a.n_seq * a.H * a.dk * a.dv * 4));
            int dev = 0;
            if (e == cudaSuccess) e = cudaGetDevice(&dev);
            if (e == cudaSuccess && (dev < 0 || dev >= 64)) e = cudaErrorInvalidDevice;
            if (e == cudaSuccess) {
                std::lock_guard<std::mutex> lock(g_side_mu[dev]);
                SideStream *ss = nullptr;
                e = side_stream(dev, g.n + 2, &ss);
                // fork: the side streams start after the caller's prior work
                if (e == cudaSuccess) e = cudaEventRecord(ss->events[g.n], a.stream);
                if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->events[g.n], 0);
                if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->prep2, ss->events[g.n], 0);
                for (int sgi = 0; sgi < g.n && e == cudaSuccess; ++sgi) {
                    const int c_lo = sgi * g.seg, c_hi = c_lo + g.seg;
                    cudaStream_t ps = (sgi & 1) ? ss->prep2 : a.stream;
                    e = slot_launch(&slot, ps, [&] { return gdn::launch_chunk_prep(a, w, c_lo, c_hi, ps); });
                    if (e == cudaSuccess) e = cudaEventRecord(ss->events[sgi], ps);
                    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->events[sgi], 0);
                    const float *sin = sgi == 0 ? a.S0 : state;
                    float *sout = sgi == g.n - 1 ? a.S_final : state;
                    if (e == cudaSuccess)
                        e = slot_launch(&slot, ss->stream, [&] {
                            return gdn::launch_chunk_chain(a, w, c_lo, c_hi, sin, sout, ss->stream);
                        });
                }
                // every prep launch precedes a chain launch on the chain stream, so
                // joining the chain stream joins all of the call's work
                // join: the caller's stream continues after the last chain launch
                if (e == cudaSuccess) e = cudaEventRecord(ss->events[g.n + 1], ss->stream);
                if (e == cudaSuccess) e = cudaStreamWaitEvent(a.stream, ss->events[g.n + 1], 0);
            }
        }
        if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    } else {
        float *qn = reinterpret_cast<float *>(ws);
        float *kn = reinterpret_cast<float *>(ws + round_up(nt * a.dk * sizeof(float)));
        float *vn = reinterpret_cast<float *>(ws + 2 * round_up(nt * a.dk * sizeof(float)));
        int slot = 0;
        e = slot_launch(&slot, a.stream, [&] { return gdn::launch_prelude_f32(a, qn, kn, vn); });
        if (e == cudaSuccess) e = record(g_ev_begin, a.stream);
        if (e == cudaSuccess)
            e = slot_launch(&slot, a.stream, [&] { return gdn::launch_recurrent(a, qn, kn, vn); });
        if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    }
    if (own_ws) {
        cudaError_t ef = cudaFreeAsync(ws, a.stream);
        if (e == cudaSuccess) e = ef;
    }
    return e;
}

cudaError_t prefill_dispatch(const gdn::PrefillArgs &a) { return prefill_run(a, nullptr); }

}  // namespace

namespace gdn {
cudaError_t sm_count(int *out) {
    static int cache[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!cache[dev]) {
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        cache[dev] = n;
    }
    *out = cache[dev];
    return cudaSuccess;
}

void note_launch() { ++tl_launches; }
void reset_launch_count() {
    tl_launches = 0;
    tl_slots = 0;
}
}  // namespace gdn

extern "C" {

gdn_status_t gdn_set_kernel_events(void *const *begin, void *const *end, int n) {
    if (n < 0 || (n > 0 && (!begin || !end))) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!begin[i] || !end[i]) return GDN_ERR_INVALID_ARG;
    g_kev_begin.assign(reinterpret_cast<cudaEvent_t const *>(begin),
                       reinterpret_cast<cudaEvent_t const *>(begin) + n);
    g_kev_end.assign(reinterpret_cast<cudaEvent_t const *>(end),
                     reinterpret_cast<cudaEvent_t const *>(end) + n);
    return GDN_OK;
}

int gdn_last_call_launches(void) { return tl_launches; }

int gdn_last_call_slots(void) { return tl_slots; }

gdn_status_t gdn_device_error_status(unsigned *flags, int clear, gdn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned w[5] = {0, 0, 0, 0, 0};
    cudaError_t e = gdn::prep_error_word(&w[0], clear != 0, s);
    if (e == cudaSuccess) e = gdn::chain_error_word(&w[1], clear != 0, s);
    if (e == cudaSuccess) e = gdn::decode_error_word(&w[2], clear != 0, s);
    if (e == cudaSuccess) e = gdn::qsa_error_word(&w[3], clear != 0, s);
    if (e == cudaSuccess) e = gdn::gemm_error_word(&w[4], clear != 0, s);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const unsigned f = (w[0] ? GDN_ERRF_PREP : 0u) | (w[1] ? GDN_ERRF_CHAIN : 0u) |
                       (w[2] ? GDN_ERRF_DECODE : 0u) | (w[3] ? GDN_ERRF_QSA : 0u) |
                       (w[4] ? GDN_ERRF_GEMM : 0u);
    if (flags) *flags = f;
    return f ? GDN_ERR_TIMEOUT : GDN_OK;
}

gdn_status_t gdn_set_timing_events(void *begin, void *end) {
    if ((begin == nullptr) != (end == nullptr)) return GDN_ERR_INVALID_ARG;
    g_ev_begin = static_cast<cudaEvent_t>(begin);
    g_ev_end = static_cast<cudaEvent_t>(end);
    return GDN_OK;
}

const char *gdn_status_string(gdn_status_t s) {
    switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_ALIGNMENT: return "GDN_ERR_ALIGNMENT";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_ERR_UNKNOWN";
}

gdn_status_t gdn_prefill_workspace_size(const gdn_dims_t *dims, size_t *bytes) {
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (!bytes) return GDN_ERR_INVALID_ARG;
    *bytes = workspace_bytes(dims);
    return GDN_OK;
}

}  // extern "C"

namespace {
// Argument checks of gdn_prefill and gdn_prefill_ws; fills *a on success.
gdn_status_t prefill_args(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                          const float *conv_w, const void *a_logit, const void *b_logit,
                          const float *A, const float *b_alpha, const void *z,
                          const float *norm_w, const float *S0, const int32_t *cu_seqlens,
                          void *out, float *S_final, gdn_stream_t stream, gdn::PrefillArgs *ap) {
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (!cu_seqlens && dims->total_tokens % dims->num_seqs != 0) return GDN_ERR_INVALID_ARG;
    // token tensors may be NULL only when there are no tokens
    const bool no_tokens = dims->total_tokens == 0;
    const uintptr_t in_sz = dims->in_dtype == GDN_BF16 ? 2 : 4;
    const void *tok[] = {q, k, v, z, out};
    for (const void *p : tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *gates[] = {a_logit, b_logit};
    for (const void *p : gates) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !aligned_to(p, in_sz)) return GDN_ERR_ALIGNMENT;
    }
    if (!conv_w) return GDN_ERR_INVALID_ARG;
    if (!aligned16(conv_w)) return GDN_ERR_ALIGNMENT;
    const void *params[] = {A, b_alpha, norm_w};
    for (const void *p : params) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    const void *opt[] = {S0, S_final};
    for (const void *p : opt)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (cu_seqlens && !aligned_to(cu_seqlens, 4)) return GDN_ERR_ALIGNMENT;

    gdn::PrefillArgs &a = *ap;
    a.n_seq = dims->num_seqs;
    a.n_tok = dims->total_tokens;
    a.H = dims->H;
    a.dk = dims->dk;
    a.dv = dims->dv;
    a.in_bf16 = dims->in_dtype == GDN_BF16;
    a.out_bf16 = dims->out_dtype == GDN_BF16;
    a.q = q; a.k = k; a.v = v; a.z = z; a.a_logit = a_logit; a.b_logit = b_logit;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w; a.S0 = S0;
    a.cu_seqlens = cu_seqlens;
    a.out = out;
    a.S_final = S_final;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return GDN_OK;
}
}  // namespace

extern "C" {

gdn_status_t gdn_prefill(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                         const float *conv_w, const void *a_logit, const void *b_logit,
                         const float *A, const float *b_alpha, const void *z,
                         const float *norm_w, const float *S0, const int32_t *cu_seqlens,
                         void *out, float *S_final, gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    gdn::PrefillArgs a;
    const gdn_status_t st = prefill_args(dims, q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0,
                                         cu_seqlens, out, S_final, stream, &a);
    if (st != GDN_OK) return st;
    return prefill_dispatch(a) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_prefill_ws(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                            const float *conv_w, const void *a_logit, const void *b_logit,
                            const float *A, const float *b_alpha, const void *z,
                            const float *norm_w, const float *S0, const int32_t *cu_seqlens,
                            void *out, float *S_final, void *workspace, size_t workspace_bytes_given,
                            gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    gdn::PrefillArgs a;
    const gdn_status_t st = prefill_args(dims, q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0,
                                         cu_seqlens, out, S_final, stream, &a);
    if (st != GDN_OK) return st;
    const size_t need = workspace_bytes(dims);
    if (need > 0 && (!workspace || workspace_bytes_given < need)) return GDN_ERR_INVALID_ARG;
    if (workspace && !aligned_to(workspace, 256)) return GDN_ERR_ALIGNMENT;
    return prefill_run(a, static_cast<char *>(workspace)) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_prefill_backward_workspace_size(const gdn_dims_t *dims, size_t *bytes) {
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (!bytes) return GDN_ERR_INVALID_ARG;
    if (dims->in_dtype != GDN_F32 || dims->out_dtype != GDN_F32 || dims->dk != dims->dv)
        return GDN_ERR_UNSUPPORTED;
    *bytes = gdn::backward_workspace_bytes(dims->num_seqs, dims->total_tokens, dims->H, dims->dk);
    return GDN_OK;
}

gdn_status_t gdn_prefill_backward(const gdn_dims_t *dims, const void *q, const void *k, const void *v,
                                  const float *conv_w, const void *a_logit, const void *b_logit,
                                  const float *A, const float *b_alpha, const void *z, const float *norm_w,
                                  const float *S0, const int32_t *cu_seqlens, const void *d_out,
                                  const float *d_S_final, void *dq, void *dk, void *dv, float *d_conv_w,
                                  void *d_a_logit, void *d_b_logit, float *d_A, float *d_b_alpha, void *d_z,
                                  float *d_norm_w, float *d_S0, gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (dims->in_dtype != GDN_F32 || dims->out_dtype != GDN_F32 || dims->dk != dims->dv)
        return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens && dims->total_tokens % dims->num_seqs != 0) return GDN_ERR_INVALID_ARG;
    const bool no_tokens = dims->total_tokens == 0;
    const void *tok[] = {q, k, v, z, d_out, dq, dk, dv, d_z};
    for (const void *p : tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *per_tok[] = {a_logit, b_logit, d_a_logit, d_b_logit};
    for (const void *p : per_tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    const void *need16[] = {conv_w, d_conv_w, norm_w, d_norm_w};
    for (const void *p : need16) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *need4[] = {A, b_alpha, d_A, d_b_alpha};
    for (const void *p : need4) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    const void *opt[] = {S0, d_S_final, d_S0};
    for (const void *p : opt)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (cu_seqlens && !aligned_to(cu_seqlens, 4)) return GDN_ERR_ALIGNMENT;

    gdn::BackwardArgs b;
    gdn::PrefillArgs &a = b.f;
    a.n_seq = dims->num_seqs;
    a.n_tok = dims->total_tokens;
    a.H = dims->H;
    a.dk = dims->dk;
    a.dv = dims->dv;
    a.in_bf16 = false;
    a.out_bf16 = false;
    a.q = q; a.k = k; a.v = v; a.z = z; a.a_logit = a_logit; a.b_logit = b_logit;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w; a.S0 = S0;
    a.cu_seqlens = cu_seqlens;
    a.out = nullptr;
    a.S_final = nullptr;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    b.d_out = d_out;
    b.d_S_final = d_S_final;
    b.dq = dq; b.dk = dk; b.dv = dv; b.d_a_logit = d_a_logit; b.d_b_logit = d_b_logit; b.d_z = d_z;
    b.d_conv_w = d_conv_w; b.d_A = d_A; b.d_b_alpha = d_b_alpha; b.d_norm_w = d_norm_w; b.d_S0 = d_S0;

    const size_t ws_bytes = gdn::backward_workspace_bytes(a.n_seq, a.n_tok, a.H, a.dk);
    char *ws = nullptr;
    cudaMemPool_t pool;
    if (get_pool(&pool) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), ws_bytes, pool, a.stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    cudaError_t e = record(g_ev_begin, a.stream);
    if (e == cudaSuccess) e = gdn::launch_backward(b, ws);
    if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    cudaError_t ef = cudaFreeAsync(ws, a.stream);
    if (e == cudaSuccess) e = ef;
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_qsa_indexer_workspace_size(int batch, int n, size_t *bytes) {
    if (batch <= 0 || n < 0 || !bytes) return GDN_ERR_INVALID_ARG;
    *bytes = gdn::qsa_workspace_bytes(batch, n);
    return GDN_OK;
}

gdn_status_t gdn_qsa_indexer(int batch, int n, int heads, int d, int block, int budget, const void *q,
                             const void *k, const float *w_q, const float *w_k, int32_t *sel, float *scores,
                             gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    if (batch <= 0 || n < 0 || heads <= 0 || d <= 0 || block <= 0 || budget <= 0) return GDN_ERR_INVALID_ARG;
    if (heads != 4 || d != 128 || block != 4 || budget % block != 0) return GDN_ERR_UNSUPPORTED;
    // row coordinates of the score kernel's tensor maps stay within int32
    if ((int64_t)batch * n * heads >= ((int64_t)1 << 31)) return GDN_ERR_UNSUPPORTED;
    const bool empty = n == 0;
    const void *need16[] = {q, k};
    for (const void *p : need16) {
        if (!p && !empty) return GDN_ERR_INVALID_ARG;
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    if (!sel && !empty) return GDN_ERR_INVALID_ARG;
    if (sel && !aligned_to(sel, 4)) return GDN_ERR_ALIGNMENT;
    if (scores && !aligned16(scores)) return GDN_ERR_ALIGNMENT;
    const void *need4[] = {w_q, w_k};
    for (const void *p : need4) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    if (empty) return GDN_OK;
    gdn::QsaArgs a;
    a.B = batch;
    a.n = n;
    a.KB = budget / block;
    a.q = q;
    a.k = k;
    a.w_q = w_q;
    a.w_k = w_k;
    a.sel = sel;
    a.scores = scores;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    const size_t ws_bytes = gdn::qsa_workspace_bytes(batch, n);
    char *ws = nullptr;
    cudaMemPool_t pool;
    if (get_pool(&pool) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), ws_bytes, pool, a.stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    cudaError_t e = record(g_ev_begin, a.stream);
    if (e == cudaSuccess) e = gdn::launch_qsa_indexer(a, ws);
    if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    cudaError_t ef = cudaFreeAsync(ws, a.stream);
    if (e == cudaSuccess) e = ef;
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_gemm_bf16(int M, int N, int K, const void *A, int lda, const void *B, int ldb, void *C, int ldc,
                           gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    if (M < 0 || N < 0 || K <= 0 || lda < K || ldb < N || ldc < N) return GDN_ERR_INVALID_ARG;
    if (K % 8 || lda % 8 || ldc % 8 || (N >= 64 && ldb % 8)) return GDN_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return GDN_OK;
    if (!A || !B || !C) return GDN_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return GDN_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t ws_bytes = gdn::gemm_workspace_bytes(N, K);
    char *ws = nullptr;
    if (ws_bytes) {
        cudaMemPool_t pool;
        if (get_pool(&pool) != cudaSuccess) return GDN_ERR_CUDA;
        if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), ws_bytes, pool, s) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    cudaError_t e = gdn::launch_gemm_bf16(M, N, K, A, lda, B, ldb, C, ldc, ws, s);
    if (ws) {
        cudaError_t ef = cudaFreeAsync(ws, s);
        if (e == cudaSuccess) e = ef;
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_layer_workspace_size(const gdn_dims_t *dims, int d_model, size_t *bytes) {
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (!bytes || d_model <= 0) return GDN_ERR_INVALID_ARG;
    *bytes = gdn::layer_workspace_bytes(dims->total_tokens, dims->H, dims->dk, dims->dv, d_model) + workspace_bytes(dims);
    return GDN_OK;
}

gdn_status_t gdn_layer_forward(const gdn_dims_t *dims, int d_model, const void *x, const void *w_in,
                               const float *conv_w, const float *A, const float *b_alpha, const float *norm_w,
                               const void *w_o, const float *S0, const int32_t *cu_seqlens, void *y, float *S_final,
                               gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    gdn_status_t st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    if (dims->in_dtype != GDN_BF16 || dims->out_dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (d_model <= 0) return GDN_ERR_INVALID_ARG;
    if (d_model % 8 != 0) return GDN_ERR_UNSUPPORTED;   // 16-byte rows for the GEMMs
    if (!cu_seqlens && dims->total_tokens % dims->num_seqs != 0) return GDN_ERR_INVALID_ARG;
    const bool no_tokens = dims->total_tokens == 0;
    const void *tok[] = {x, y};
    for (const void *p : tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *weights[] = {w_in, w_o, conv_w};
    for (const void *p : weights) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *params[] = {A, b_alpha, norm_w};
    for (const void *p : params) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    const void *opt[] = {S0, S_final};
    for (const void *p : opt)
        if (p && !aligned16(p)) return GDN_ERR_ALIGNMENT;
    if (cu_seqlens && !aligned_to(cu_seqlens, 4)) return GDN_ERR_ALIGNMENT;

    gdn::LayerArgs L;
    gdn::PrefillArgs &a = L.f;
    a.n_seq = dims->num_seqs;
    a.n_tok = dims->total_tokens;
    a.H = dims->H;
    a.dk = dims->dk;
    a.dv = dims->dv;
    a.in_bf16 = true;
    a.out_bf16 = true;
    a.q = a.k = a.v = a.z = a.a_logit = a.b_logit = nullptr;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w; a.S0 = S0;
    a.cu_seqlens = cu_seqlens;
    a.out = nullptr;
    a.S_final = S_final;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    L.d_model = d_model;
    L.x = x;
    L.w_in = w_in;
    L.w_o = w_o;
    L.y = y;
    if (no_tokens) return prefill_dispatch(a) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    const size_t ws_bytes = gdn::layer_workspace_bytes(a.n_tok, a.H, a.dk, a.dv, d_model);
    char *ws = nullptr;
    cudaMemPool_t pool;
    if (get_pool(&pool) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), ws_bytes, pool, a.stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    cudaError_t e = gdn::launch_layer(L, ws, &prefill_dispatch);
    cudaError_t ef = cudaFreeAsync(ws, a.stream);
    if (e == cudaSuccess) e = ef;
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_decode_step(const gdn_dims_t *dims, const void *q, const void *k,
                             const void *v, const float *conv_w, void *conv_hist,
                             const void *a_logit, const void *b_logit, const float *A,
                             const float *b_alpha, const void *z, const float *norm_w, float *S,
                             void *out, gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    gdn_status_t st = check_dims(dims, true);
    if (st != GDN_OK) return st;
    const void *vec[] = {q, k, v, conv_w, conv_hist, z, S, out};
    for (const void *p : vec) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const uintptr_t in_sz = dims->in_dtype == GDN_BF16 ? 2 : 4;
    const void *gates[] = {a_logit, b_logit};
    for (const void *p : gates) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, in_sz)) return GDN_ERR_ALIGNMENT;
    }
    const void *params[] = {A, b_alpha, norm_w};
    for (const void *p : params) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    gdn::DecodeArgs a;
    a.B = dims->num_seqs;
    a.H = dims->H;
    a.dk = dims->dk;
    a.dv = dims->dv;
    a.in_bf16 = dims->in_dtype == GDN_BF16;
    a.out_bf16 = dims->out_dtype == GDN_BF16;
    a.q = q; a.k = k; a.v = v; a.z = z; a.a_logit = a_logit; a.b_logit = b_logit;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w;
    a.conv_hist = conv_hist;
    a.S = S;
    a.out = out;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = record(g_ev_begin, a.stream);
    int slot = 0;
    if (e == cudaSuccess)
        e = slot_launch(&slot, a.stream, [&] {
            return gdn::decode_stream_supported(a) ? gdn::launch_decode_stream(a) : gdn::launch_decode(a);
        });
    if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_decode_multi(const gdn_dims_t *dims, int T, const void *q, const void *k,
                              const void *v, const float *conv_w, void *conv_hist, const void *a_logit,
                              const void *b_logit, const float *A, const float *b_alpha, const void *z,
                              const float *norm_w, float *S, void *out, const int32_t *n_keep,
                              gdn_stream_t stream) {
    tl_launches = 0;
    tl_slots = 0;
    if (!dims) return GDN_ERR_INVALID_ARG;
    if (T < 1 || T > 4) return GDN_ERR_INVALID_ARG;
    gdn_dims_t one = *dims;   // validate as a single-token step of the same shape
    if ((int64_t)dims->total_tokens != (int64_t)dims->num_seqs * T) return GDN_ERR_INVALID_ARG;
    one.total_tokens = dims->num_seqs;
    gdn_status_t st = check_dims(&one, true);
    if (st != GDN_OK) return st;
    if (dims->in_dtype != GDN_BF16 || dims->dk != 128 || dims->dv != 128) return GDN_ERR_UNSUPPORTED;
    const void *vec[] = {q, k, v, conv_w, conv_hist, z, S, out};
    for (const void *p : vec) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned16(p)) return GDN_ERR_ALIGNMENT;
    }
    const void *gates[] = {a_logit, b_logit};
    for (const void *p : gates) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 2)) return GDN_ERR_ALIGNMENT;
    }
    const void *params[] = {A, b_alpha, norm_w};
    for (const void *p : params) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!aligned_to(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    if (n_keep && !aligned_to(n_keep, 4)) return GDN_ERR_ALIGNMENT;
    gdn::DecodeArgs a;
    a.B = dims->num_seqs;
    a.H = dims->H;
    a.dk = dims->dk;
    a.dv = dims->dv;
    a.in_bf16 = true;
    a.out_bf16 = dims->out_dtype == GDN_BF16;
    a.q = q; a.k = k; a.v = v; a.z = z; a.a_logit = a_logit; a.b_logit = b_logit;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w;
    a.conv_hist = conv_hist;
    a.S = S;
    a.out = out;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = record(g_ev_begin, a.stream);
    int slot = 0;
    if (e == cudaSuccess)
        e = slot_launch(&slot, a.stream, [&] { return gdn::launch_decode_stream(a, T, n_keep); });
    if (e == cudaSuccess) e = record(g_ev_end, a.stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"

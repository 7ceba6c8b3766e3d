// gdn_prefill_noalloc -- the tensor-core prefill for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocator at the time they run the
// layer: code that executes inside a host callback or a driver-managed region
// where allocation is forbidden, embedders whose device memory is carved up
// up-front by another runtime, and real-time services that must not take an
// allocator lock or risk an out-of-memory failure mid-request.  gdn_prefill
// takes its workspace from a stream-ordered memory pool, so those callers
// cannot use it.  This entry point runs the same two kernels (chunk prep, then
// the chunk chain) with their workspace placed in a fixed-size array in the
// library's own device memory instead, and allocates nothing.
//
// The array is a file-scope static __device__ object of GDN_NOALLOC_SCRATCH_BYTES:
// every GPU that loads the library holds it until the process exits.  Its
// device address is looked up once per device with cudaGetSymbolAddress (the
// host-side name of a __device__ array is only a stand-in and must never be
// handed to a kernel); the first call on each device does that lookup, so make
// that first call before any stream capture.
//
// Every call on a device shares the one array and the array keeps whatever the
// last call left in it.  Nothing in it needs to start at zero: each call writes
// every workspace element before reading it.  Calls whose work overlaps on the
// GPU (for example on two streams at once) race on the array.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/gdn.h"
#include "gdn_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {};

// Device address of the scratch array for the current device, looked up once.
cudaError_t noalloc_scratch(char **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = static_cast<char *>(g_noalloc_addr[dev]);
    return cudaSuccess;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

bool is_aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" gdn_status_t gdn_prefill_noalloc(const gdn_dims_t *dims, const void *q, const void *k,
                                            const void *v, const float *conv_w, const void *a_logit,
                                            const void *b_logit, const float *A,
                                            const float *b_alpha, const void *z,
                                            const float *norm_w, const float *S0,
                                            const int32_t *cu_seqlens, void *out, float *S_final,
                                            gdn_stream_t stream) {
    gdn::reset_launch_count();
    if (!dims) return GDN_ERR_INVALID_ARG;
    const gdn_dims_t &d = *dims;
    if (d.num_seqs <= 0 || d.total_tokens < 0 || d.H <= 0 || d.dk <= 0 || d.dv <= 0 || d.conv_k <= 0)
        return GDN_ERR_INVALID_ARG;
    if ((d.in_dtype != GDN_F32 && d.in_dtype != GDN_BF16) ||
        (d.out_dtype != GDN_F32 && d.out_dtype != GDN_BF16))
        return GDN_ERR_INVALID_ARG;
    // only the tensor-core path has a no-allocation variant
    if (d.in_dtype != GDN_BF16 || d.dk != 128 || (d.dv != 64 && d.dv != 128) || d.conv_k != 4)
        return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens && d.total_tokens % d.num_seqs != 0) return GDN_ERR_INVALID_ARG;
    const bool no_tokens = d.total_tokens == 0;
    const void *tok[] = {q, k, v, z, out};
    for (const void *p : tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !is_aligned(p, 16)) return GDN_ERR_ALIGNMENT;
    }
    const void *gates[] = {a_logit, b_logit};
    for (const void *p : gates) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && !is_aligned(p, 2)) return GDN_ERR_ALIGNMENT;
    }
    if (!conv_w) return GDN_ERR_INVALID_ARG;
    if (!is_aligned(conv_w, 16)) return GDN_ERR_ALIGNMENT;
    const void *params[] = {A, b_alpha, norm_w};
    for (const void *p : params) {
        if (!p) return GDN_ERR_INVALID_ARG;
        if (!is_aligned(p, 4)) return GDN_ERR_ALIGNMENT;
    }
    if ((S0 && !is_aligned(S0, 16)) || (S_final && !is_aligned(S_final, 16)))
        return GDN_ERR_ALIGNMENT;
    if (cu_seqlens && !is_aligned(cu_seqlens, 4)) return GDN_ERR_ALIGNMENT;

    // workspace layout of the tensor-core path: Qt, Kt, -W [dk], U' [dv], Aqk [64]
    // in fp16 and e^{G_C} in fp32 per token-head
    const size_t nt = (size_t)d.total_tokens * d.H;
    const size_t need = 3 * round256(nt * d.dk * 2) + round256(nt * d.dv * 2) +
                        round256(nt * 64 * 2) + round256(nt * 4);
    if (need > (size_t)GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_INVALID_ARG;

    char *ws = nullptr;
    if (noalloc_scratch(&ws) != cudaSuccess) return GDN_ERR_CUDA;

    gdn::PrefillArgs a;
    a.n_seq = d.num_seqs;
    a.n_tok = d.total_tokens;
    a.H = d.H;
    a.dk = d.dk;
    a.dv = d.dv;
    a.in_bf16 = true;
    a.out_bf16 = d.out_dtype == GDN_BF16;
    a.q = q; a.k = k; a.v = v; a.z = z; a.a_logit = a_logit; a.b_logit = b_logit;
    a.conv_w = conv_w; a.A = A; a.b_alpha = b_alpha; a.norm_w = norm_w; a.S0 = S0;
    a.cu_seqlens = cu_seqlens;
    a.out = out;
    a.S_final = S_final;
    a.stream = reinterpret_cast<cudaStream_t>(stream);

    gdn::TcWorkspace w;
    char *p = ws;
    auto take = [&](size_t bytes) { char *r = p; p += round256(bytes); return r; };
    w.Qt = reinterpret_cast<__half *>(take(nt * d.dk * 2));
    w.Kt = reinterpret_cast<__half *>(take(nt * d.dk * 2));
    w.Wn = reinterpret_cast<__half *>(take(nt * d.dk * 2));
    w.Up = reinterpret_cast<__half *>(take(nt * d.dv * 2));
    w.Aqk = reinterpret_cast<__half *>(take(nt * 64 * 2));
    w.decay = reinterpret_cast<float *>(take(nt * 4));
    cudaError_t e = gdn::launch_chunk_prep(a, w);
    if (e == cudaSuccess) e = gdn::launch_chunk_chain(a, w);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

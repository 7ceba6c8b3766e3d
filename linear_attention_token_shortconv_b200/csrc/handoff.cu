// gdn_prefill_conv_tail -- the ShortConv history a decode step needs to continue
// a prefilled sequence.
//
// The causal depthwise convolution (slinene.github.io write-up of "On the Design
// of Qwen3.8-Next Architecture", 模块 A, 参数化: q, k, v each pass through a short
// convolution before SiLU) looks back conv_k - 1 = 3 raw tokens.  After a prefill
// those are the last three raw q | k | v rows of each sequence; decode reads them
// from its history buffer [B, 3, H (2 dk + dv)], oldest row first.  This kernel
// gathers them: history row j of sequence n is raw token s_end - 3 + j when that
// token belongs to the sequence, else a row of zeros (the sequence is shorter
// than three tokens, and the convolution's left padding is zero).
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

// One block per (sequence, history row); 16-byte vectors over the row's
// q, k and v channels.
__global__ void conv_tail_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ k,
                                 const uint4 *__restrict__ v, const int32_t *__restrict__ cu, int n_tok,
                                 int n_seq, int q_vec, int v_vec, uint4 *__restrict__ hist) {
    const int n = blockIdx.x, j = blockIdx.y;
    int s_begin, s_end;
    if (cu) { s_begin = cu[n]; s_end = cu[n + 1]; }
    else { const int L = n_tok / n_seq; s_begin = n * L; s_end = s_begin + L; }
    const int t = s_end - 3 + j;
    const bool in = t >= s_begin;
    const int row_vec = 2 * q_vec + v_vec;
    uint4 *dst = hist + ((size_t)n * 3 + j) * row_vec;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int e = threadIdx.x; e < row_vec; e += blockDim.x) {
        uint4 x = zero;
        if (in) {
            if (e < q_vec) x = q[(size_t)t * q_vec + e];
            else if (e < 2 * q_vec) x = k[(size_t)t * q_vec + e - q_vec];
            else x = v[(size_t)t * v_vec + e - 2 * q_vec];
        }
        dst[e] = x;
    }
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status_t gdn_prefill_conv_tail(const gdn_dims_t *dims, const void *q, const void *k,
                                              const void *v, const int32_t *cu_seqlens, void *conv_hist,
                                              gdn_stream_t stream) {
    gdn::reset_launch_count();
    if (!dims) return GDN_ERR_INVALID_ARG;
    const gdn_dims_t &d = *dims;
    if (d.num_seqs <= 0 || d.total_tokens < 0 || d.H <= 0 || d.dk <= 0 || d.dv <= 0 || d.conv_k <= 0)
        return GDN_ERR_INVALID_ARG;
    if (d.in_dtype != GDN_F32 && d.in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((d.dk != 64 && d.dk != 128) || (d.dv != 64 && d.dv != 128) || d.conv_k != 4) return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens && d.total_tokens % d.num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (!conv_hist) return GDN_ERR_INVALID_ARG;
    const bool no_tokens = d.total_tokens == 0;
    const void *tok[] = {q, k, v};
    for (const void *p : tok) {
        if (!p && !no_tokens) return GDN_ERR_INVALID_ARG;
        if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return GDN_ERR_ALIGNMENT;
    }
    if (reinterpret_cast<uintptr_t>(conv_hist) & 15u) return GDN_ERR_ALIGNMENT;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN_ERR_ALIGNMENT;
    const int esz = d.in_dtype == GDN_BF16 ? 2 : 4;
    const int q_vec = d.H * d.dk * esz / 16, v_vec = d.H * d.dv * esz / 16;
    const dim3 grid(d.num_seqs, 3);
    gdn::conv_tail_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(q), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), cu_seqlens,
        d.total_tokens, d.num_seqs, q_vec, v_vec, static_cast<uint4 *>(conv_hist));
    return gdn::launched() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

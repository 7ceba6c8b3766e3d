// K6 -- the GDN layer from the hidden states to the output projection: the steps
// on either side of the mixer (slinene.github.io write-up of "On the Design of
// Qwen3.8-Next Architecture", 模块 A, 参数化: q, k, v, z, the decay and write
// logits are linear projections of x; o = W_o [sigmoid(z) RMSNorm(y)]).
//
//   [q | k | v | z | a | b] = x W_in      (bf16 GEMMs, fp32 accumulation, bf16 out)
//   o = gdn_prefill(q, k, v, ..., z, ...) (the mixer, bf16 out)
//   y = o W_o                              (bf16 GEMM)
//
// The projections run on the library's own tcgen05 GEMM (K7, gemm.cu); each
// column block of the packed W_in is its own GEMM, writing the contiguous
// [N, H, d] tensor the mixer reads.  Not fused: the GEMM epilogues do not run
// the conv / SiLU / norm prelude.
#include <cuda_bf16.h>

#include "gdn_internal.h"

namespace gdn {

namespace {
// dst [rows][cols] (contiguous) = the column block [rows][c0, c0 + cols) of src
// (leading dimension ld): a W_in block whose rows do not start on 16-byte
// boundaries, made readable by TMA.
__global__ void copy_cols_kernel(const __nv_bfloat16 *__restrict__ src, int ld, int c0, int rows, int cols,
                                 __nv_bfloat16 *__restrict__ dst) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)rows * cols) return;
    const int r = (int)(i / cols), c = (int)(i % cols);
    dst[i] = src[(size_t)r * ld + c0 + c];
}

// The gate logits [rows][a_0 .. a_{H-1} b_0 .. b_{H-1}] of one GEMM into the
// mixer's a [rows][H] and b [rows][H].
__global__ void split_gates_kernel(const __nv_bfloat16 *__restrict__ ab, int rows, int H,
                                   __nv_bfloat16 *__restrict__ a, __nv_bfloat16 *__restrict__ b) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)rows * 2 * H) return;
    const long long r = i / (2 * H);
    const int j = (int)(i % (2 * H));
    if (j < H) a[r * H + j] = ab[i];
    else b[r * H + j - H] = ab[i];
}
}  // namespace

size_t layer_workspace_bytes(int n_tok, int H, int dk, int dv, int d_model) {
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t n = (size_t)n_tok;
    const int wide = dk > dv ? dk : dv;
    return 2 * ru(n * H * dk * 2) + 3 * ru(n * H * dv * 2) + 2 * ru(n * H * 2) + ru(n * 2 * H * 2) +
           ru(gemm_workspace_bytes(2 * H, d_model)) + ru((size_t)d_model * H * wide * 2);
}

cudaError_t launch_layer(const LayerArgs &L, void *ws, cudaError_t (*run_prefill)(const PrefillArgs &)) {
    const PrefillArgs &a = L.f;
    const int N = a.n_tok, H = a.H, dk = a.dk, dv = a.dv, D = L.d_model;
    const int c_in = H * (2 * dk + 2 * dv) + 2 * H;
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    char *p = static_cast<char *>(ws);
    auto take = [&](size_t bytes) { char *r = p; p += ru(bytes); return r; };
    char *q = take((size_t)N * H * dk * 2), *k = take((size_t)N * H * dk * 2);
    char *v = take((size_t)N * H * dv * 2), *z = take((size_t)N * H * dv * 2);
    char *al = take((size_t)N * H * 2), *bl = take((size_t)N * H * 2);
    char *o = take((size_t)N * H * dv * 2);
    char *ab = take((size_t)N * 2 * H * 2);                   // both gate logits, one GEMM
    char *gw = take(gemm_workspace_bytes(2 * H, D));
    char *wcopy = take((size_t)D * H * (dk > dv ? dk : dv) * 2);
    // W_in rows start on 16-byte boundaries only when its width is a multiple of 8
    const bool w_aligned = c_in % 8 == 0;
    const char *w_in = static_cast<const char *>(L.w_in);
    // column blocks of W_in: q, k [H dk], v, z [H dv], then a and b [H] side by
    // side, one GEMM of 2H columns (x is read once for both)
    struct Part { char *dst; int cols; } parts[5] = {
        {q, H * dk}, {k, H * dk}, {v, H * dv}, {z, H * dv}, {ab, 2 * H}};
    cudaError_t e;
    int c0 = 0;
    for (const Part &pt : parts) {
        const void *B = w_in + (size_t)c0 * 2;
        int ldb = c_in;
        if (!w_aligned && pt.cols >= 64) {   // a block read by TMA: copy it out, contiguous
            const long long n_el = (long long)D * pt.cols;
            copy_cols_kernel<<<(unsigned)((n_el + 255) / 256), 256, 0, a.stream>>>(
                static_cast<const __nv_bfloat16 *>(L.w_in), c_in, c0, D, pt.cols, reinterpret_cast<__nv_bfloat16 *>(wcopy));
            if ((e = launched()) != cudaSuccess) return e;
            B = wcopy;
            ldb = pt.cols;
        }
        if ((e = launch_gemm_bf16(N, pt.cols, D, L.x, D, B, ldb, pt.dst, pt.cols, gw, a.stream)) != cudaSuccess)
            return e;
        c0 += pt.cols;
    }
    {
        const long long n_el = (long long)N * 2 * H;
        split_gates_kernel<<<(unsigned)((n_el + 255) / 256), 256, 0, a.stream>>>(
            reinterpret_cast<const __nv_bfloat16 *>(ab), N, H, reinterpret_cast<__nv_bfloat16 *>(al),
            reinterpret_cast<__nv_bfloat16 *>(bl));
        if ((e = launched()) != cudaSuccess) return e;
    }
    PrefillArgs m = a;
    m.q = q; m.k = k; m.v = v; m.z = z; m.a_logit = al; m.b_logit = bl;
    m.out = o;
    m.in_bf16 = true;
    m.out_bf16 = true;
    if ((e = run_prefill(m)) != cudaSuccess) return e;
    return launch_gemm_bf16(N, D, H * dv, o, H * dv, L.w_o, D, L.y, D, nullptr, a.stream);
}

}  // namespace gdn

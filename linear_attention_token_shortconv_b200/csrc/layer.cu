// K6 -- the GDN layer from the hidden states to the output projection: the steps
// on either side of the mixer (slinene.github.io write-up of "On the Design of
// Qwen3.8-Next Architecture", 模块 A, 参数化: q, k, v, z, the decay and write
// logits are linear projections of x; o = W_o [sigmoid(z) RMSNorm(y)]).
//
//   [q | k | v | z | a | b] = x W_in      (bf16 GEMMs, fp32 accumulation, bf16 out)
//   o = gdn_prefill(q, k, v, ..., z, ...) (the mixer, bf16 out)
//   y = o W_o                              (bf16 GEMM)
//
// The projections are plain GEMMs and run on cuBLAS (loaded with dlopen at first
// use, so the library itself loads without it); each column block of the packed
// W_in is its own GEMM, writing the contiguous [N, H, d] tensor the mixer reads.
// Not fused: the GEMM epilogues do not run the conv / SiLU / norm prelude.
#include <cublas_v2.h>
#include <dlfcn.h>

#include <mutex>

#include "gdn_internal.h"

namespace gdn {

namespace {

typedef cublasStatus_t (*CreateFn)(cublasHandle_t *);
typedef cublasStatus_t (*SetStreamFn)(cublasHandle_t, cudaStream_t);
typedef cublasStatus_t (*GemmExFn)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                   const void *, const void *, cudaDataType, int, const void *, cudaDataType, int,
                                   const void *, void *, cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t);

struct Blas {
    bool tried = false, ok = false;
    CreateFn create = nullptr;
    SetStreamFn set_stream = nullptr;
    GemmExFn gemm = nullptr;
};
std::mutex g_blas_mu;
Blas g_blas;

// The cuBLAS entry points (resolved once) and the calling thread's handle for this
// device.  A handle carries the stream of the call in progress, so threads that
// run layers at the same time must not share one: each (host thread, device)
// gets its own, created at its first use and kept for the thread's lifetime.
bool blas_handle(int dev, cublasHandle_t *h) {
    {
        std::lock_guard<std::mutex> lock(g_blas_mu);
        if (!g_blas.tried) {
            g_blas.tried = true;
            void *lib = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
            if (lib) {
                g_blas.create = reinterpret_cast<CreateFn>(dlsym(lib, "cublasCreate_v2"));
                g_blas.set_stream = reinterpret_cast<SetStreamFn>(dlsym(lib, "cublasSetStream_v2"));
                g_blas.gemm = reinterpret_cast<GemmExFn>(dlsym(lib, "cublasGemmEx"));
                g_blas.ok = g_blas.create && g_blas.set_stream && g_blas.gemm;
            }
        }
    }
    if (!g_blas.ok || dev < 0 || dev >= 64) return false;
    thread_local cublasHandle_t tl_handle[64] = {};
    if (!tl_handle[dev] && g_blas.create(&tl_handle[dev]) != CUBLAS_STATUS_SUCCESS) return false;
    *h = tl_handle[dev];
    return true;
}

// Row-major C [M, Nc] = A [M, K] (lda) x B [K, Nc] (ldb), bf16 in and out, fp32
// accumulation: cuBLAS's column-major C^T = B^T A^T.
cudaError_t gemm_bf16(cublasHandle_t h, int M, int Nc, int K, const void *A, int lda, const void *B, int ldb,
                      void *C, int ldc) {
    if (M == 0 || Nc == 0) return cudaSuccess;
    const float one = 1.0f, zero = 0.0f;
    const cublasStatus_t st = g_blas.gemm(h, CUBLAS_OP_N, CUBLAS_OP_N, Nc, M, K, &one, B, CUDA_R_16BF, ldb, A,
                                          CUDA_R_16BF, lda, &zero, C, CUDA_R_16BF, ldc, CUBLAS_COMPUTE_32F,
                                          CUBLAS_GEMM_DEFAULT);
    return st == CUBLAS_STATUS_SUCCESS ? cudaSuccess : cudaErrorUnknown;
}

}  // namespace

size_t layer_workspace_bytes(int n_tok, int H, int dk, int dv) {
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t n = (size_t)n_tok;
    return 2 * ru(n * H * dk * 2) + 3 * ru(n * H * dv * 2) + 2 * ru(n * H * 2);
}

bool layer_blas_available() {
    int dev = 0;
    cublasHandle_t h;
    return cudaGetDevice(&dev) == cudaSuccess && blas_handle(dev, &h);
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
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cublasHandle_t h;
    if (!blas_handle(dev, &h)) return cudaErrorNotSupported;
    if (g_blas.set_stream(h, a.stream) != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
    const char *w_in = static_cast<const char *>(L.w_in);
    // column blocks of W_in: q, k [H dk], v, z [H dv], a, b [H]
    struct Part { char *dst; int cols; } parts[6] = {{q, H * dk}, {k, H * dk}, {v, H * dv}, {z, H * dv}, {al, H}, {bl, H}};
    int c0 = 0;
    for (const Part &pt : parts) {
        if ((e = gemm_bf16(h, N, pt.cols, D, L.x, D, w_in + (size_t)c0 * 2, c_in, pt.dst, pt.cols)) != cudaSuccess)
            return e;
        c0 += pt.cols;
    }
    PrefillArgs m = a;
    m.q = q; m.k = k; m.v = v; m.z = z; m.a_logit = al; m.b_logit = bl;
    m.out = o;
    m.in_bf16 = true;
    m.out_bf16 = true;
    if ((e = run_prefill(m)) != cudaSuccess) return e;
    if (g_blas.set_stream(h, a.stream) != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
    return gemm_bf16(h, N, D, H * dv, o, H * dv, L.w_o, D, L.y, D);
}

}  // namespace gdn

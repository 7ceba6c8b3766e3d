// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled, reached through
// the runtime's driver entry point so the library does not link libcuda).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gdn_internal.h"

namespace gdn {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_enc_mu;
EncodeTiledFn g_encode = nullptr;

cudaError_t encoder(EncodeTiledFn *fn) {
    std::lock_guard<std::mutex> lock(g_enc_mu);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = g_encode;
    return cudaSuccess;
}
}  // namespace

static_assert(sizeof(TmaMap) == sizeof(CUtensorMap), "tensor map size");

cudaError_t make_tma_3d(TmaMap *out, const void *base, bool bf16, int inner, int H, int n_tok,
                        int box_inner, int box_rows, bool swizzle128) {
    EncodeTiledFn fn;
    cudaError_t e = encoder(&fn);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)n_tok};
    const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * H};
    const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(out->bytes),
                    bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                    const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Rows of fp32 values [rows][cols] (row stride cols * 4 bytes, a multiple of 16)
// as a 3-D map {cols, 1, rows} with boxes {box_cols, 1, box_rows}: box_cols = 32
// (128-byte rows, 128-byte swizzle) or 16 (64-byte rows, 64-byte swizzle).
cudaError_t make_tma_rows_f32(TmaMap *out, const void *base, int cols, int rows, int box_cols, int box_rows) {
    EncodeTiledFn fn;
    cudaError_t e = encoder(&fn);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, 1, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)cols * 4};
    const cuuint32_t box[3] = {(cuuint32_t)box_cols, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(out->bytes), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// A bf16 tensor of rank 3 or 4 without swizzle: dims[0] contiguous, strides[i]
// the byte stride of dimension i + 1 (multiples of 16), box[] the copied tile.
cudaError_t make_tma_plain_bf16(TmaMap *out, const void *base, int rank, const long long *dims,
                                const long long *strides, const int *box) {
    EncodeTiledFn fn;
    cudaError_t e = encoder(&fn);
    if (e != cudaSuccess) return e;
    if (rank < 3 || rank > 4) return cudaErrorInvalidValue;
    cuuint64_t d[4], st[3];
    cuuint32_t bx[4], estr[4] = {1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = (cuuint64_t)dims[i];
        bx[i] = (cuuint32_t)box[i];
        if (i + 1 < rank) st[i] = (cuuint64_t)strides[i];
    }
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(out->bytes), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                    const_cast<void *>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// A row-major bf16 matrix [rows][inner] with leading dimension ld (elements; ld * 2
// a multiple of 16) as a 3-D map {inner, 1, rows}, boxes {box_inner, 1, box_rows},
// 128-byte swizzle (box_inner * 2 = 128).
cudaError_t make_tma_mat_bf16(TmaMap *out, const void *base, int inner, int rows, int ld, int box_inner,
                              int box_rows) {
    EncodeTiledFn fn;
    cudaError_t e = encoder(&fn);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, 1, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2};
    const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(out->bytes), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace gdn

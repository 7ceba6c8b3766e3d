// K7 -- the layer's projections as bf16 GEMMs on tcgen05 (slinene.github.io
// write-up of "On the Design of Qwen3.8-Next Architecture", 模块 A, 参数化: q, k, v,
// z and the two gate logits are linear projections of the hidden state x, and
// the mixer's output goes through W_o):
//
//   C [M, N] = A [M, K] B [K, N],   bf16 row-major, fp32 accumulation, bf16 out.
//
// One persistent CTA per SM walks 128 x 256 output tiles (the M tiles of one
// column of tiles in turn, so the CTAs running at once share their B panel in
// L2).  K advances in blocks of 64 through four shared-memory stages filled by
// TMA: an A block is K-major (128 rows x 128 bytes), a B block MN-major (four
// 64-column blocks of 64 K rows, the row-major B as it lies in memory), both
// 128-byte swizzled.  Per K block, four M = 128, N = 256, K = 16 MMAs accumulate
// into one of two 256-column TMEM buffers, so a tile's epilogue drains while the
// next tile accumulates.  Fewer than 64 columns (the gate logits: one per head)
// take 128 x 32 tiles with B transposed once into the caller's workspace
// (K-major), since an MN-major block needs 64 columns.  Roles: warp 0 lane 0
// loads, warp 1 lane 0 issues the MMAs (and owns the TMEM allocation), warps 2-9
// are the epilogue (TMEM lane quadrant w % 4, 128 of the 256 columns each):
// fp32 -> bf16, 16-byte stores of whole 64-byte row pieces.  Every wait is bounded; a timeout raises the GEMM
// error word and an abort flag that the other roles check.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

__device__ unsigned int g_gemm_err;

namespace gemm {
constexpr int BM = 128, BK = 64, NS = 4;
constexpr int A_ST = BM * BK * 2;                  // 16 KB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t MAX_POLLS = 1u << 24;
// Two shapes: wide (N tiles of 256, B MN-major: the row-major B as it lies in
// memory, four 64-column blocks per stage) and narrow (N tiles of 32, B given
// transposed, K-major: the gate-logit projections, a handful of columns).
template <int BN> struct Shape {
    static constexpr bool B_MN = BN >= 64;
    static constexpr int B_ST = BN * BK * 2;                 // 32 KB or 4 KB
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + NS * A_ST;          // 65536
    static constexpr int OFF_BAR = OFF_B + NS * B_ST;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;        // barriers, TMEM slot, abort flag; alignment slack
    static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulators
    static constexpr int EPI_COLS = BN >= 64 ? BN / 2 : BN;  // columns per epilogue warp
};
}  // namespace gemm

struct GemmMaps {
    CUtensorMap a;   // A [M][K] bf16, box {64, 1, 128}
    CUtensorMap b;   // wide: B [K][N], box {64, 1, 64}; narrow: B^T [N][K], box {64, 1, BN}
};

namespace {
__device__ __forceinline__ void gemm_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(umma::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    uint32_t w;
    std::memcpy(&w, &p, 4);
    return w;
}
}  // namespace

template <int BN>
__global__ void __launch_bounds__(gemm::THREADS, 1)
gemm_bf16_kernel(const __grid_constant__ GemmMaps maps, int M, int N, int K, __nv_bfloat16 *__restrict__ C,
                 int ldc) {
    using namespace gemm;
    using Sh = Shape<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Sh::OFF_BAR);
    uint64_t *full = bars, *empty = bars + NS;
    uint64_t *tfull = bars + 2 * NS, *tempty = bars + 2 * NS + 2;
    uint64_t *mma_done = bars + 2 * NS + 4;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2 * NS + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int n_tiles = tiles_m * tiles_n, kbs = (K + BK - 1) / BK;

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            umma::mbar_init(full + i, 1);
            umma::mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            umma::mbar_init(tfull + i, 1);
            umma::mbar_init(tempty + i, EPI_WARPS);
        }
        umma::mbar_init(mma_done, 1);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    if (warp == 1) umma::tmem_alloc(tslot, Sh::TMEM_COLS);
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = *tslot;

    auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (umma::mbar_wait_bounded(bar, parity, MAX_POLLS)) return true;
        atomicOr(&g_gemm_err, 1u);
        *abort_flag = 1;
        return false;
    };

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------------- producer
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            const int tm = t % tiles_m, tn = t / tiles_m;
            for (int kb = 0; kb < kbs; ++kb, ++it) {
                const int st = it % NS, u = it / NS;
                if (!(ok = wait(empty + st, (u + 1) & 1))) break;
                umma::mbar_expect_tx(full + st, A_ST + Sh::B_ST);
                umma::tma_load_3d(sm + Sh::OFF_A + st * A_ST, &maps.a, BK * kb, 0, BM * tm, full + st);
                uint8_t *bst = sm + Sh::OFF_B + st * Sh::B_ST;
                if constexpr (Sh::B_MN) {
                    for (int j = 0; j < BN / 64; ++j)
                        umma::tma_load_3d(bst + j * 8192, &maps.b, BN * tn + 64 * j, 0, BK * kb, full + st);
                } else {
                    umma::tma_load_3d(bst, &maps.b, BK * kb, 0, BN * tn, full + st);
                }
            }
        }
        // after an abort, loads still in flight land before the CTA leaves
        if (*abort_flag)
            for (int k = max(0, it - NS); k < it; ++k) umma::mbar_wait_bounded(full + k % NS, (k / NS) & 1, MAX_POLLS);
    } else if (warp == 1 && lane == 0) {
        // --------------------------------------------------------------- MMA issuer
        int it = 0, t_it = 0;
        bool ok = true;
        const uint32_t idesc = umma::idesc_bf16(BM, BN, false, Sh::B_MN);
        const uint32_t a0 = umma::smem_u32(sm + Sh::OFF_A), b0 = umma::smem_u32(sm + Sh::OFF_B);
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++t_it) {
            const int ts = t_it & 1, v = t_it >> 1;
            if (!(ok = wait(tempty + ts, (v + 1) & 1))) break;
            umma::tc_fence_after();
            const uint32_t d = tbase + ts * BN;
            for (int kb = 0; kb < kbs; ++kb, ++it) {
                const int st = it % NS, u = it / NS;
                if (!(ok = wait(full + st, u & 1))) break;
                umma::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < BK / 16; ++ks) {
                    const uint64_t ad = umma::sw128_desc(a0 + st * A_ST + ks * 32, 16, 1024);
                    const uint64_t bd = Sh::B_MN ? umma::sw128_desc(b0 + st * Sh::B_ST + ks * 2048, 8192, 1024)
                                                 : umma::sw128_desc(b0 + st * Sh::B_ST + ks * 32, 16, 1024);
                    umma::mma_f16(d, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
                }
                umma::mma_commit(empty + st);
            }
            if (!ok) break;
            umma::mma_commit(tfull + ts);
        }
        // after an abort the epilogue may not have waited for the last MMAs: they
        // complete before the tensor memory is released
        if (it > 0 && *abort_flag) {
            umma::mma_commit(mma_done);
            umma::mbar_wait_bounded(mma_done, 0, MAX_POLLS);
        }
    } else if (warp >= 2) {
        // ----------------------------------------------------------------- epilogue
        // warp w: TMEM lane quadrant w % 4; wide tiles: columns 128 ((w - 2) / 4) ..
        // + 127; narrow tiles: warps 2-5 take all 32 columns, warps 6-9 only release
        const int qd = warp & 3, hf = (warp - 2) >> 2;
        const int c0 = Sh::EPI_COLS * hf;
        const bool active = BN >= 64 || hf == 0;
        const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
        const bool vec = (ldc & 7) == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0;
        int t_it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++t_it) {
            const int tm = t % tiles_m, tn = t / tiles_m;
            const int ts = t_it & 1, v = t_it >> 1;
            ok = __all_sync(0xffffffffu, wait(tfull + ts, v & 1));
            if (!ok) break;
            umma::tc_fence_after();
            const int row = BM * tm + 32 * qd + lane;
            __nv_bfloat16 *crow = C + (size_t)(row < M ? row : 0) * ldc;
            if (active) {
#pragma unroll 1
                for (int c = c0; c < c0 + Sh::EPI_COLS; c += 32) {
                    float x[32];
                    umma::tmem_ld32(trow + ts * BN + c, x);
                    const int col = BN * tn + c;
                    if (row < M && col < N) {
                        if (vec && col + 32 <= N) {
                            uint4 *d4 = reinterpret_cast<uint4 *>(crow + col);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                d4[e] = make_uint4(pack_bf16(x[8 * e + 0], x[8 * e + 1]), pack_bf16(x[8 * e + 2], x[8 * e + 3]),
                                                   pack_bf16(x[8 * e + 4], x[8 * e + 5]), pack_bf16(x[8 * e + 6], x[8 * e + 7]));
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (col + e < N) crow[col + e] = __float2bfloat16_rn(x[e]);
                        }
                    }
                }
            }
            umma::tc_fence_before();
            __syncwarp();
            if (lane == 0) gemm_arrive(tempty + ts);
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 1) umma::tmem_dealloc(tbase, Sh::TMEM_COLS);
}

// B^T [Np][K] from the row-major B [K][N] (leading dimension ldb), rows N .. Np - 1
// zero: the narrow shape's K-major operand, padded to whole 32-row tiles.
__global__ void gemm_transpose_kernel(const __nv_bfloat16 *__restrict__ B, int ldb, int N, int Np, int K,
                                      __nv_bfloat16 *__restrict__ BT) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)Np * K) return;
    const int n = (int)(i / K), k = (int)(i % K);
    BT[i] = n < N ? B[(size_t)k * ldb + n] : __float2bfloat16_rn(0.f);
}

template <int BN>
cudaError_t launch_gemm_shape(const GemmMaps &m, int M, int N, int K, void *C, int ldc, cudaStream_t stream) {
    using Sh = gemm::Shape<BN>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(gemm_bf16_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::SMEM)) !=
        cudaSuccess)
        return e;
    int sms = 0;
    if ((e = sm_count(&sms)) != cudaSuccess) return e;
    const long long tiles = (long long)((M + gemm::BM - 1) / gemm::BM) * ((N + BN - 1) / BN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    gemm_bf16_kernel<BN><<<grid, gemm::THREADS, Sh::SMEM, stream>>>(m, M, N, K, static_cast<__nv_bfloat16 *>(C), ldc);
    return launched();
}

size_t gemm_workspace_bytes(int N, int K) {
    return N >= 64 ? 0 : ((size_t)((N + 31) / 32 * 32) * K * 2 + 255) & ~(size_t)255;
}

cudaError_t launch_gemm_bf16(int M, int N, int K, const void *A, int lda, const void *B, int ldb, void *C, int ldc,
                             void *ws, cudaStream_t stream) {
    using namespace gemm;
    if (M == 0 || N == 0) return cudaSuccess;
    if (M < 0 || N < 0 || K <= 0 || lda < K || ldb < N || ldc < N || (lda & 7) || (K & 7))
        return cudaErrorInvalidValue;
    if (reinterpret_cast<uintptr_t>(A) & 15) return cudaErrorInvalidValue;
    // the wide shape reads B by TMA: 16-byte rows
    if (N >= 64 && ((ldb & 7) || (reinterpret_cast<uintptr_t>(B) & 15))) return cudaErrorInvalidValue;
    GemmMaps m;
    std::memset(&m, 0, sizeof m);
    cudaError_t e;
    if ((e = make_tma_mat_bf16(reinterpret_cast<TmaMap *>(&m.a), A, K, M, lda, 64, BM)) != cudaSuccess) return e;
    if (N >= 64) {
        if ((e = make_tma_mat_bf16(reinterpret_cast<TmaMap *>(&m.b), B, N, K, ldb, 64, 64)) != cudaSuccess) return e;
        return launch_gemm_shape<256>(m, M, N, K, C, ldc, stream);
    }
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15)) return cudaErrorInvalidValue;
    __nv_bfloat16 *bt = static_cast<__nv_bfloat16 *>(ws);
    const int Np = (N + 31) / 32 * 32;
    const long long n_el = (long long)Np * K;
    gemm_transpose_kernel<<<(unsigned)((n_el + 255) / 256), 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(B),
                                                                             ldb, N, Np, K, bt);
    if ((e = launched()) != cudaSuccess) return e;
    if ((e = make_tma_mat_bf16(reinterpret_cast<TmaMap *>(&m.b), bt, K, Np, K, 64, 32)) != cudaSuccess) return e;
    return launch_gemm_shape<32>(m, M, N, K, C, ldc, stream);
}

// One CTA waits, through the GEMM's bounded wait, for a barrier phase that
// nothing completes.
__global__ void gemm_wait_selftest_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        umma::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !umma::mbar_wait_bounded(&bar, 0, max_polls)) atomicOr(&g_gemm_err, 1u);
}

cudaError_t gemm_wait_selftest(uint32_t max_polls, cudaStream_t s) {
    gemm_wait_selftest_kernel<<<1, 32, 0, s>>>(max_polls);
    return cudaGetLastError();
}

cudaError_t gemm_error_word(unsigned *v, bool clear, cudaStream_t s) {
    return read_error_word(g_gemm_err, v, clear, s);
}

}  // namespace gdn

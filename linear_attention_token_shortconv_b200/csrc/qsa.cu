// K5 -- the QSA compressed indexer (slinene.github.io write-up of "On the Design
// of Qwen3.8-Next Architecture", 模块 B — Qwen Sparse Attention: "压缩轻量 indexer"
// and the block selection paragraph), for H = 4 indexer heads of d = 128 and
// blocks of r = 4 tokens:
//   q_i^h = PRoPE(RMSNorm(q_raw_i^h) w_q, i),
//   k_bar_b = PRoPE(RMSNorm(mean(k_raw_{4b .. 4b+3})) w_k, 4b),
//   I_ib = sum_h ReLU(<q_i^h, k_bar_b>) for complete blocks (4b + 3 <= i),
//   B_i = the ceil(K / 4) highest-scoring complete blocks (ties to the smaller
//   block), ascending, padded with -1.  The tokens the sparse attention reads are
//   the blocks expanded plus the tail 4 floor((i + 1) / 4) .. i (implied).
// RMSNorm is x / sqrt(mean x^2 + 1e-6) times its weight; PRoPE rotates dims
// [0, 64) as pairs (j, j + 32) by p 10000^(-j / 32) and keeps dims [64, 128).
//
// Kernels:
//  K5a qsa_prep_kernel: one warp per query row (all 4 heads) or key block:
//      RMSNorm, rotation (the angle reduced in double precision: positions reach
//      1e5 and more), fp16 rows [(i, h)][128] and [b][128].
//  K5b qsa_score_kernel: tcgen05, persistent (one CTA per SM): a tile of 128
//      queries x 4 heads stays in shared memory while 64-block tiles stream
//      through three stages by TMA (128-byte swizzled, K-major); per block tile
//      one M = 128, N = 64 product per head into its own TMEM columns, two TMEM
//      stages; warp-specialised producer, MMA issuer and eight epilogue warps
//      (ReLU, head sum, 128-byte row segments of the complete blocks' scores).
//      Only block tiles that hold a complete block of the query tile are visited.
//  K5c qsa_topk_kernel: one warp per query row, no block barriers: the row's
//      scores counted into 2048 value buckets over [0, row max] (the score kernel
//      leaves each row's largest score) in the warp's own shared histogram; the
//      bucket holding the K_B-th largest score is the threshold, and one walk over
//      the row in index order takes the keys above it and ranks the few inside
//      it, equal scores taken from the smallest index.  A threshold bucket of
//      more than 64 keys (many equal scores) falls back to a radix select on the
//      score bits (scores are >= 0, so their bit patterns order like the values;
//      digits of 11, 11 and 9 bits).  The selected blocks come out ascending.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {

__device__ unsigned int g_qsa_err;

namespace qsa {
constexpr int D = 128, HI = 4, R = 4;
constexpr double ROPE_BASE = 10000.0;
}  // namespace qsa

// ------------------------------------------------------------------ K5a: prep
// cos and sin of the rotation of the pair (lane, lane + 32) at position pos:
// the angle pos * base^(-lane / 32) (inv_freq) formed and reduced in double
// precision, since positions reach 1e5 and more
__device__ __forceinline__ void qsa_rope_cs(long long pos, double inv_freq, float &c, float &s) {
    double sd, cd;
    sincos((double)pos * inv_freq, &sd, &cd);
    c = (float)cd;
    s = (float)sd;
}

__device__ __forceinline__ void qsa_norm_rope(float (&x)[4], const float *__restrict__ w, float c, float s,
                                              int lane) {
    // lane holds dims lane, lane + 32, lane + 64, lane + 96
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) ss = fmaf(x[u], x[u], ss);
    ss = group_sum<32>(ss);
    const float rn = 1.0f / sqrtf(ss / qsa::D + kNormEps);
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] *= rn * __ldg(w + lane + 32 * u);
    // rotate the pair (lane, lane + 32)
    const float a = x[0], b = x[1];
    x[0] = a * c - b * s;
    x[1] = a * s + b * c;
}

__global__ void __launch_bounds__(256)
qsa_prep_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k, const float *__restrict__ w_q,
                const float *__restrict__ w_k, int B, int n, __half *__restrict__ qr, __half *__restrict__ kb) {
    using namespace qsa;
    const int nb = n / R;
    const long long n_q = (long long)B * n, n_items = n_q + (long long)B * nb;
    const int lane = threadIdx.x & 31;
    const double inv_freq = pow(ROPE_BASE, -(double)lane / 32.0);   // base^(-lane / 32), once per thread
    for (long long it = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); it < n_items; it += (long long)gridDim.x * 8) {
        if (it < n_q) {   // query row (sequence it / n, token it % n), all heads: one rotation
            float c, s;
            qsa_rope_cs(it % n, inv_freq, c, s);
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                const bf16 *src = q + (it * HI + h) * D;
                float x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) x[u] = __bfloat162float(src[lane + 32 * u]);
                qsa_norm_rope(x, w_q, c, s, lane);
                __half *dst = qr + (it * HI + h) * D;
#pragma unroll
                for (int u = 0; u < 4; ++u) dst[lane + 32 * u] = __float2half_rn(x[u]);
            }
        } else {          // key block: mean of 4 raw keys
            const long long jb = it - n_q, s = jb / nb, b = jb % nb;
            const bf16 *src = k + (s * n + b * R) * D;
            float x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < R; ++t) acc += __bfloat162float(src[t * D + lane + 32 * u]);
                x[u] = acc * (1.0f / R);
            }
            float c, sn;
            qsa_rope_cs(b * R, inv_freq, c, sn);
            qsa_norm_rope(x, w_k, c, sn, lane);
            __half *dst = kb + jb * D;
#pragma unroll
            for (int u = 0; u < 4; ++u) dst[lane + 32 * u] = __float2half_rn(x[u]);
        }
    }
}

// ------------------------------------------------------------------ K5b: scores
// Bounded wait of the indexer kernels: false (and the device error word raised)
// when the phase does not complete within max_polls polls.
__device__ __forceinline__ bool qsa_wait(uint64_t *bar, uint32_t parity, uint32_t max_polls) {
    const bool ok = umma::mbar_wait_bounded(bar, parity, max_polls);
    if (!ok) atomicOr(&g_qsa_err, 1u);
    return ok;
}

namespace qsa {
// Persistent score kernel.  A work item is (sequence s, query tile qt of QT
// queries, a run of at most CH block tiles of BN blocks); items enumerate the
// (s, qt) pairs in order and cut each query tile's block tiles into runs of CH.
constexpr int QT = 128;                  // queries per tile (TMEM lanes)
constexpr int BN = 64;                   // blocks per block tile (MMA N, per head)
constexpr int CH = 8;                    // block tiles per work item at most
constexpr int NSB = 3;                   // block-tile stages in shared memory
constexpr int A_HEAD = 2 * 16384;        // one head's query tile: 2 k-blocks x [128 rows x 128 B]
constexpr int B_STAGE = 2 * 8192;        // one block tile: 2 k-blocks x [64 rows x 128 B]
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + HI * A_HEAD;             // 131072
constexpr int EPI_WARPS = 8;             // two per TMEM lane quadrant (16, four per quadrant, measured slower)
constexpr int EC = 4 * BN / EPI_WARPS;   // block columns per epilogue warp: 32 (or 16)
constexpr int OFF_STG = OFF_B + NSB * B_STAGE;         // 180224: per epilogue warp, a 32 x EC fp32 store tile
constexpr int STG_TILE = 32 * EC * 4;
constexpr int OFF_BAR = OFF_STG + EPI_WARPS * STG_TILE;   // 212992
constexpr int SMEM = OFF_BAR + 256 + 1024;             // barriers, TMEM slot, abort flag; alignment slack
constexpr uint32_t TMEM_COLS = 512;                    // 2 stages x 4 heads x 64 columns
constexpr uint32_t MAX_POLLS = 1u << 24;
}  // namespace qsa

namespace {

// N (32 or 16) consecutive TMEM columns of the warp's lane quadrant, no wait
template <int N>
__device__ __forceinline__ void qsa_tmem_ld(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 32 || N == 16, "32 or 16 columns");
    if constexpr (N == 32) umma::tmem_ld32_nowait(taddr, r);
    else umma::tmem_ld16_nowait(taddr, r);
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(umma::smem_u32(bar)) : "memory");
}

struct QsaItem {
    int s, qt, bt0, nbt;
};

// block tiles of query tile qt: those holding a block complete for its last query
__host__ __device__ __forceinline__ int qsa_tiles_of(int n, int qt) {
    const int last = min(qsa::QT * qt + qsa::QT - 1, n - 1);
    return ((last + 1) / qsa::R + qsa::BN - 1) / qsa::BN;
}

// Item `it` of the enumeration; every role walks the same increasing item
// indices, so the cursor (first item of the current (s, qt)) only moves forward.
struct QsaCursor {
    int s = 0, qt = 0, first = 0;
};

__device__ __forceinline__ bool qsa_find_item(int it, int B, int n, QsaCursor &c, QsaItem &out) {
    const int n_qt = (n + qsa::QT - 1) / qsa::QT;
    while (c.s < B) {
        const int nbt = qsa_tiles_of(n, c.qt);
        const int k = (nbt + qsa::CH - 1) / qsa::CH;
        if (it < c.first + k) {
            const int j = it - c.first;
            out.s = c.s;
            out.qt = c.qt;
            out.bt0 = j * qsa::CH;
            out.nbt = min(qsa::CH, nbt - out.bt0);
            return true;
        }
        c.first += k;
        if (++c.qt == n_qt) {
            c.qt = 0;
            ++c.s;
        }
    }
    return false;
}

}  // namespace

struct QsaMaps {
    CUtensorMap q;   // [B n][4][128] fp16, box {64, 1, 128}, 128-byte swizzle
    CUtensorMap k;   // [B nb][1][128] fp16, box {64, 1, 64}
    CUtensorMap sc;  // scores [B n][1][nb] fp32, box {32, 1, 32}, 128-byte swizzle (when nb % 4 == 0)
};

// One CTA per SM walks the work items.  The four heads' query rows of the tile
// (4 x 128 rows x 128 dims fp16 = 128 KB) stay in shared memory for the item;
// block tiles (64 x 128 fp16 = 16 KB) stream through NSB stages.  Each head's
// product (M = 128 queries, N = 64 blocks, K = 128) goes to its own 64 TMEM
// columns, so the epilogue sums ReLU over the heads per (query lane, block
// column) with no shuffles; two TMEM stages let the MMAs of block tile j + 1 run
// while tile j's epilogue drains.
// Roles: warp 0 lane 0 issues the TMA loads, warp 1 lane 0 the MMAs (warp 1 owns
// the TMEM allocation), warps 2-9 are the epilogue (TMEM lane quadrant w % 4, one
// query per lane; warps 2-5 take block columns 0-31 of each tile, warps 6-9
// columns 32-63).  A 32-query x 32-block piece whose blocks are all complete for
// its 32 queries leaves by one TMA store from the warp's swizzled tile; pieces on
// the causal edge or past the sequence's end are stored lane by lane, complete
// blocks only.  Barriers: full_a /
// empty_a (query tile), full_b / empty_b (block stages), tfull / tempty (TMEM
// stages; tempty takes one arrival per epilogue warp).  Every wait is bounded;
// a timeout raises the error word and an abort flag the other roles check.
__global__ void __launch_bounds__(64 + 32 * qsa::EPI_WARPS, 1)
qsa_score_kernel(const __grid_constant__ QsaMaps maps, int B, int n, int n_items, bool tma_out,
                 float *__restrict__ scores, float *__restrict__ rowmax) {
    using namespace qsa;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *full_a = bars, *empty_a = bars + 1;
    uint64_t *full_b = bars + 2, *empty_b = bars + 2 + NSB;
    uint64_t *tfull = bars + 2 + 2 * NSB, *tempty = bars + 4 + 2 * NSB;
    uint64_t *mma_done = bars + 6 + 2 * NSB;   // teardown after an abort: issued MMAs completed
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 7 + 2 * NSB);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = n / R;

    if (tid == 0) {
        umma::mbar_init(full_a, 1);
        umma::mbar_init(empty_a, 1);
        for (int i = 0; i < NSB; ++i) {
            umma::mbar_init(full_b + i, 1);
            umma::mbar_init(empty_b + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            umma::mbar_init(tfull + i, 1);
            umma::mbar_init(tempty + i, EPI_WARPS);
        }
        umma::mbar_init(mma_done, 1);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    if (warp == 1) umma::tmem_alloc(tslot, TMEM_COLS);
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = *tslot;

    auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (qsa_wait(bar, parity, MAX_POLLS)) return true;
        *abort_flag = 1;
        return false;
    };

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------------- producer
        QsaCursor cur;
        QsaItem item;
        int a_it = 0, b_it = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            if (!qsa_find_item(it, B, n, cur, item)) break;
            if (!(ok = wait(empty_a, (a_it + 1) & 1))) break;
            umma::mbar_expect_tx(full_a, HI * A_HEAD);
            for (int h = 0; h < HI; ++h)
                for (int kb = 0; kb < 2; ++kb)
                    umma::tma_load_3d(sm + OFF_A + h * A_HEAD + kb * 16384, &maps.q, 64 * kb, h,
                                      item.s * n + QT * item.qt, full_a);
            ++a_it;
            for (int j = 0; j < item.nbt; ++j, ++b_it) {
                const int st = b_it % NSB, u = b_it / NSB;
                if (!(ok = wait(empty_b + st, (u + 1) & 1))) break;
                umma::mbar_expect_tx(full_b + st, B_STAGE);
                for (int kb = 0; kb < 2; ++kb)
                    umma::tma_load_3d(sm + OFF_B + st * B_STAGE + kb * 8192, &maps.k, 64 * kb, 0,
                                      item.s * nb + BN * (item.bt0 + j), full_b + st);
            }
        }
        // after an abort, loads still in flight land before the CTA leaves
        if (*abort_flag) {
            if (a_it > 0) umma::mbar_wait_bounded(full_a, (a_it - 1) & 1, MAX_POLLS);
            for (int k = max(0, b_it - NSB); k < b_it; ++k)
                umma::mbar_wait_bounded(full_b + k % NSB, (k / NSB) & 1, MAX_POLLS);
        }
    } else if (warp == 1 && lane == 0) {
        // --------------------------------------------------------------- MMA issuer
        QsaCursor cur;
        QsaItem item;
        int a_it = 0, t_it = 0;
        bool ok = true;
        const uint32_t idesc = umma::idesc_f16(128, BN, false, false);
        const uint32_t a0 = umma::smem_u32(sm + OFF_A), b0 = umma::smem_u32(sm + OFF_B);
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            if (!qsa_find_item(it, B, n, cur, item)) break;
            if (!(ok = wait(full_a, a_it & 1))) break;
            for (int j = 0; j < item.nbt; ++j, ++t_it) {
                const int st = t_it % NSB, u = t_it / NSB;
                const int ts = t_it & 1, v = t_it >> 1;
                if (!(ok = wait(full_b + st, u & 1))) break;
                if (!(ok = wait(tempty + ts, (v + 1) & 1))) break;
                umma::tc_fence_after();
                for (int h = 0; h < HI; ++h) {
                    const uint32_t d = tbase + ts * (HI * BN) + h * BN;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t ad = umma::sw128_desc(a0 + h * A_HEAD + (k / 4) * 16384 + (k % 4) * 32, 16, 1024);
                        const uint64_t bd = umma::sw128_desc(b0 + st * B_STAGE + (k / 4) * 8192 + (k % 4) * 32, 16, 1024);
                        umma::mma_f16(d, ad, bd, idesc, k > 0);
                    }
                }
                umma::mma_commit(empty_b + st);
                umma::mma_commit(tfull + ts);
            }
            if (!ok) break;
            umma::mma_commit(empty_a);
            ++a_it;
        }
        // after an abort the epilogue may not have waited for the last MMAs: they
        // complete before the tensor memory is released
        if (t_it > 0 && *abort_flag) {
            umma::mma_commit(mma_done);
            umma::mbar_wait_bounded(mma_done, 0, MAX_POLLS);
        }
    } else if (warp >= 2) {
        // ----------------------------------------------------------------- epilogue
        const int qd = warp & 3, c = EC * ((warp - 2) >> 2);   // lane quadrant, first column
        const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
        const bool vec = (nb & 3) == 0;   // rows start on 16-byte boundaries
        float *tile = reinterpret_cast<float *>(sm + OFF_STG + (warp - 2) * STG_TILE);
        QsaCursor cur;
        QsaItem item;
        int t_it = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            if (!qsa_find_item(it, B, n, cur, item)) break;
            const int i0 = QT * item.qt + 32 * qd;            // this warp's first query
            const int i = i0 + lane;                          // this lane's query
            const int n_valid = i < n ? (i + 1) / R : 0;      // its complete blocks
            const int n_full = i0 + 31 < n ? (i0 + 1) / R : 0;   // blocks complete for all 32 queries
            float *dst = scores + ((size_t)item.s * n + (i < n ? i : 0)) * nb;
            float lmax = 0.f;   // this lane's largest score in the item (for the top-k's buckets)
            for (int j = 0; j < item.nbt; ++j, ++t_it) {
                const int ts = t_it & 1, v = t_it >> 1;
                ok = __all_sync(0xffffffffu, wait(tfull + ts, v & 1));
                if (!ok) break;
                umma::tc_fence_after();
                {
                    // the four heads' columns in flight together, one wait; the TMEM
                    // stage is free for the MMAs as soon as they are in registers
                    uint32_t x[HI][EC];
#pragma unroll
                    for (int h = 0; h < HI; ++h) {
                        qsa_tmem_ld(trow + ts * (HI * BN) + h * BN + c, x[h]);
                    }
                    umma::tmem_ld_wait();
                    umma::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_local(tempty + ts);
                    float acc[EC];
#pragma unroll
                    for (int e = 0; e < EC; ++e) {
                        float a = fmaxf(__uint_as_float(x[0][e]), 0.f);
#pragma unroll
                        for (int h = 1; h < HI; ++h) a += fmaxf(__uint_as_float(x[h][e]), 0.f);
                        acc[e] = a;
                    }
                    const int bs = BN * (item.bt0 + j) + c;
#pragma unroll
                    for (int e = 0; e < EC; ++e)
                        if (bs + e < n_valid) lmax = fmaxf(lmax, acc[e]);
                    if (tma_out && bs + EC <= n_full) {   // uniform across the warp
                        if (lane == 0) umma::bulk_wait_read<0>();   // the last store has read the tile
                        __syncwarp();
                        // row `lane`, 16-byte chunk e at chunk e ^ (lane % 8) (128-byte
                        // swizzle of 128-byte rows) or e ^ (lane / 2 % 4) (64-byte swizzle
                        // of 64-byte rows)
                        const int sw = EC == 32 ? (lane & 7) : ((lane >> 1) & 3);
#pragma unroll
                        for (int e = 0; e < EC / 4; ++e)
                            reinterpret_cast<float4 *>(tile + lane * EC)[e ^ sw] =
                                make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
                        umma::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            umma::tma_store_3d(&maps.sc, bs, 0, item.s * n + i0, tile);
                            umma::bulk_commit();
                        }
                    } else if (vec && bs + EC <= n_valid) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + bs);
#pragma unroll
                        for (int e = 0; e < EC / 4; ++e)
                            d4[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < EC; ++e)
                            if (bs + e < n_valid) dst[bs + e] = acc[e];
                    }
                }
            }
            // scores are >= 0, so their bit patterns order like the values
            if (ok && lmax > 0.f) atomicMax(reinterpret_cast<int *>(rowmax) + (size_t)item.s * n + i, __float_as_int(lmax));
        }
        if (lane == 0) umma::bulk_wait_all();   // the last stores have left shared memory
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 1) umma::tmem_dealloc(tbase, TMEM_COLS);
}

// Work items of the score kernel for B sequences of n tokens.
long long qsa_score_items(int B, int n) {
    const int n_qt = (n + qsa::QT - 1) / qsa::QT;
    long long total = 0;
    for (int qt = 0; qt < n_qt; ++qt) total += (qsa_tiles_of(n, qt) + qsa::CH - 1) / qsa::CH;
    return total * B;
}

// ------------------------------------------------------------------ K5c: top-k
namespace qsa {
constexpr int HB = 2048;                  // buckets of the 11-bit digits
constexpr int WH_SLOTS = HB;              // one warp's counters
constexpr int TOPK_WARPS = 8;             // rows (warps) per CTA
}  // namespace qsa

__device__ __forceinline__ unsigned topk_key(float v) {
    return v > 0.f ? __float_as_uint(v) : 0u;   // scores >= 0: bits order like values (-0 -> 0)
}

// Descending rank HB - 1 - b of the value bucket b = min(HB - 1, floor(v * scale))
// of a score v, taken as max(v, 0) (the same bucket as its topk_key).  One fma
// rounded toward -inf adds the exact product to 2^23: in [2^23, 2^24) the floats
// are the integers, so the sum's bits are 0x4B000000 + floor(v * scale), with no
// float-to-integer conversion; larger products (and +inf) clamp to the top
// bucket, rank 0.
__device__ __forceinline__ int topk_vrank(float v, float scale) {
    float f;
    asm("fma.rm.f32 %0, %1, %2, 0f4B000000;" : "=f"(f) : "f"(fmaxf(v, 0.f)), "f"(scale));
    return max(0, (qsa::HB - 1 + 0x4B000000) - __float_as_int(f));
}

__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// One digit of the radix select, by one warp: among the keys matching `prefix`,
// the bucket of the digit at `shift` (NB buckets, counter u for descending rank
// u = NB - 1 - digit) that holds the remaining-th largest key.  Lane l sums the
// counters PER l .. PER l + PER - 1, starting at a lane-rotated one so that the
// warp's reads fall in distinct banks; a warp scan of those sums crosses
// `remaining` at exactly one lane, which walks its counters in order; the
// extended prefix, the rank left inside the bucket and the bucket's count come
// back to every lane.
template <int NB>
__device__ __forceinline__ void topk_pick(const int *hist, int remaining, unsigned prefix, int shift, int lane,
                                          unsigned &out_prefix, int &out_rem, int &out_cnt) {
    constexpr int PER = NB / 32;
    int c = 0;
#pragma unroll 8
    for (int j = 0; j < PER; ++j) c += hist[PER * lane + ((j + lane) & (PER - 1))];
    const int incl = warp_incl_scan(c, lane);
    const bool mine = incl >= remaining && incl - c < remaining;
    const int src = max(__ffs(__ballot_sync(0xffffffffu, mine)) - 1, 0);   // one lane when the counts cover `remaining`
    unsigned p = 0u;
    int r = 0, cnt = 0;
    if (mine) {
        int run = incl - c;
        for (int j = 0; j < PER; ++j) {
            const int h = hist[PER * lane + j];
            if (run + h >= remaining) {
                p = prefix | ((unsigned)(NB - 1 - (PER * lane + j)) << shift);
                r = remaining - run;
                cnt = h;
                break;
            }
            run += h;
        }
    }
    out_prefix = __shfl_sync(0xffffffffu, p, src);
    out_rem = __shfl_sync(0xffffffffu, r, src);
    out_cnt = __shfl_sync(0xffffffffu, cnt, src);
}

// One warp per query row, no block barriers: the row's keys are read from the
// score matrix for each pass -- the first from HBM, the rest from L2 -- and
// counted into the warp's own histogram with shared atomics.  Fast path: value
// buckets over [0, row max] find the threshold bucket, and one walk places the
// keys above it and the bucket's candidates in index order (see below).
// Fallback (a crowded threshold bucket): a radix select on digits of 11, 11 and
// 9 bits of the score bits finds the threshold (stopping at the first digit
// whose bucket is taken whole); the selection then walks the row in index order,
// 128 keys per step (a 16-byte load per lane when rows are aligned): the keys
// above the threshold, and the first `remaining` equal to it, are written at
// ascending positions found by warp scans of per-lane counts.
__global__ void __launch_bounds__(32 * qsa::TOPK_WARPS)
qsa_topk_kernel(const float *__restrict__ scores, const float *__restrict__ rowmax, int n, long long n_rows, int KB,
                int32_t *__restrict__ sel) {
    using namespace qsa;
    extern __shared__ int hist_all[];   // [TOPK_WARPS][WH_SLOTS]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * TOPK_WARPS + warp;
    if (row >= n_rows) return;   // no block barriers below
    int *hist = hist_all + warp * WH_SLOTS;
    const int i = (int)(row % n);
    const int nb = n / R;
    const int n_valid = (i + 1) / R;
    const float *sc = scores + (size_t)row * nb;
    int32_t *out = sel + (size_t)row * KB;
    if (n_valid <= KB) {   // every complete block
        for (int j = lane; j < KB; j += 32) out[j] = j < n_valid ? j : -1;
        return;
    }
    // Rows start on 16-byte boundaries when nb % 4 == 0; the last quad may reach
    // past n_valid, never past the row.
    const bool vec = (nb & 3) == 0;
    const int n4 = (n_valid + 3) >> 2;
    // f(key) for every complete block's key, any order; U 16-byte loads per lane
    // are issued before their keys are counted, so several loads are in flight
    constexpr int U = 4;
    const float4 *sc4 = reinterpret_cast<const float4 *>(sc);
    auto for_keys = [&](auto &&f) {
        if (vec) {
            const int nq = n_valid >> 2;   // quads of four complete blocks
            for (int q0 = lane; q0 < nq; q0 += 32 * U) {
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    v[u] = q0 + 32 * u < nq ? __ldg(sc4 + q0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (q0 + 32 * u < nq) {
                        f(v[u].x);
                        f(v[u].y);
                        f(v[u].z);
                        f(v[u].w);
                    }
                }
            }
            if (lane == 0 && (n_valid & 3)) {   // the last quad, partly complete blocks
                const float4 t = __ldg(sc4 + nq);
                const float x[3] = {t.x, t.y, t.z};
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < (n_valid & 3)) f(x[j]);
            }
        } else {
            for (int b0 = lane; b0 < n_valid; b0 += 32 * U) {
                float v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = b0 + 32 * u < n_valid ? __ldg(sc + b0 + 32 * u) : 0.f;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (b0 + 32 * u < n_valid) f(v[u]);
            }
        }
    };
    // ---- Fast path: buckets of the value scaled by the row's largest score (from
    // the score kernel), 2048 across [0, max].  Near the threshold a bucket then
    // holds a few keys, so one more walk over the row, in index order, settles the
    // selection: keys above the threshold bucket are taken, the bucket's keys
    // (candidates, at most CAND) are ranked among themselves.  The list of both,
    // in index order, and the candidates' keys reuse the histogram's space.
    constexpr int CAND = 64;
    const float rmax = rowmax[row];
    if (!(rmax > 0.f)) {   // every complete block scores 0: ties go to the smallest blocks
        for (int j = lane; j < KB; j += 32) out[j] = j;
        return;
    }
    const float scale = (float)HB / rmax;
    for (int j = lane; j < WH_SLOTS / 4; j += 32) reinterpret_cast<int4 *>(hist)[j] = make_int4(0, 0, 0, 0);
    __syncwarp();
    for_keys([&](float v) { atomicAdd(&hist[topk_vrank(v, scale)], 1); });
    __syncwarp();
    {
        unsigned bstar;
        int rem, cnt;
        topk_pick<HB>(hist, KB, 0u, 0, lane, bstar, rem, cnt);
        __syncwarp();
        if (cnt <= CAND && KB + 3 * CAND <= WH_SLOTS) {   // uniform
            int *list = hist;                                               // [KB + CAND]
            unsigned *ckey = reinterpret_cast<unsigned *>(hist + KB + CAND);   // [CAND]
            int *cidx = hist + KB + 2 * CAND;                               // [CAND]
            const unsigned lt = (1u << lane) - 1u;
            // the threshold bucket's rank: keys of a rank below it are taken, keys of
            // its rank are the candidates (the same rank function as the histogram's)
            const int rstar = HB - 1 - (int)bstar;
            int list_run = 0, cand_run = 0;
            // keys at or above the threshold bucket, in index order: index, or
            // 0x80000000 | candidate ordinal
            auto place = [&](const bool (&keep)[4], const bool (&cnd)[4], const unsigned (&k)[4], int base, int per) {
                int pos = list_run, cpos = cand_run, mine = 0, cmine = 0;
                bool any_cnd = false;
                for (int j = 0; j < per; ++j) {
                    const unsigned m = __ballot_sync(0xffffffffu, keep[j]);
                    pos += __popc(m & lt);
                    list_run += __popc(m);
                    any_cnd |= cnd[j];
                }
                if (__any_sync(0xffffffffu, any_cnd)) {   // uniform; rare: the threshold bucket's keys
                    for (int j = 0; j < per; ++j) {
                        const unsigned cm = __ballot_sync(0xffffffffu, cnd[j]);
                        cpos += __popc(cm & lt);
                        cand_run += __popc(cm);
                    }
                }
                for (int j = 0; j < per; ++j) {
                    if (cnd[j]) {
                        const int o = cpos + cmine++;
                        ckey[o] = k[j];
                        cidx[o] = base + j;
                        list[pos + mine++] = (int)(0x80000000u | (unsigned)o);
                    } else if (keep[j]) {
                        list[pos + mine++] = base + j;
                    }
                }
            };
            if (vec) {
                // lane l walks quads q0 + U l .. + U - 1: 4 U consecutive blocks, as bit
                // masks of the kept keys and the candidates; one warp scan of the
                // per-lane counts places the step's keys
                for (int q0 = 0; q0 < n4; q0 += 32 * U) {
                    const int qa = q0 + U * lane, base = 4 * qa;
                    float4 v[U];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        v[u] = qa + u < n4 ? __ldg(sc4 + qa + u) : make_float4(0.f, 0.f, 0.f, 0.f);
                    const int lim = n_valid - base;   // this lane's complete blocks
                    const unsigned vmask = lim >= 4 * U ? (1u << (4 * U)) - 1u : lim > 0 ? (1u << lim) - 1u : 0u;
                    unsigned kb = 0u, cb = 0u;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int r = topk_vrank(x[j], scale);
                            kb |= (unsigned)(r <= rstar) << (4 * u + j);
                            cb |= (unsigned)(r == rstar) << (4 * u + j);
                        }
                    }
                    kb &= vmask;
                    cb &= vmask;
                    const int c = __popc(kb);
                    const int incl = warp_incl_scan(c, lane);
                    const int pos = list_run + incl - c;
                    list_run += __shfl_sync(0xffffffffu, incl, 31);
                    if (__any_sync(0xffffffffu, cb != 0u)) {   // uniform; rare: the threshold bucket's keys
                        const int cc = __popc(cb);
                        const int cincl = warp_incl_scan(cc, lane);
                        const int cpos = cand_run + cincl - cc;
                        cand_run += __shfl_sync(0xffffffffu, cincl, 31);
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int e = 4 * u + j;
                                if ((cb >> e) & 1u) {
                                    const unsigned below = (1u << e) - 1u;
                                    const int o = cpos + __popc(cb & below);
                                    ckey[o] = topk_key(x[j]);
                                    cidx[o] = base + e;
                                    list[pos + __popc(kb & below)] = (int)(0x80000000u | (unsigned)o);
                                }
                            }
                        }
                    }
                    for (unsigned m = kb & ~cb; m != 0u; m &= m - 1u) {
                        const int e = __ffs(m) - 1;
                        list[pos + __popc(kb & ((1u << e) - 1u))] = base + e;
                    }
                }
            } else {
                for (int b0 = 0; b0 < n_valid; b0 += 32) {
                    const int b = b0 + lane;
                    const bool in = b < n_valid;
                    const float x = in ? sc[b] : 0.f;
                    const unsigned k[4] = {topk_key(x), 0u, 0u, 0u};
                    const int r = topk_vrank(x, scale);
                    const bool keep[4] = {in && r <= rstar, false, false, false};
                    const bool cnd[4] = {in && r == rstar, false, false, false};
                    place(keep, cnd, k, b, 1);
                }
            }
            __syncwarp();
            // the candidates taken: the `rem` largest keys, equal keys by index order
            unsigned taken[CAND / 32];
#pragma unroll
            for (int h = 0; h < CAND / 32; ++h) {
                const int o = 32 * h + lane;
                bool t = false;
                if (o < cnt) {
                    const unsigned ko = ckey[o];
                    int rank = 0;
                    for (int o2 = 0; o2 < cnt; ++o2) {
                        const unsigned k2 = ckey[o2];
                        rank += k2 > ko || (k2 == ko && o2 < o);
                    }
                    t = rank < rem;
                }
                taken[h] = __ballot_sync(0xffffffffu, t);
            }
            // the list without the candidates not taken, in order: exactly KB entries
            int out_run = 0;
            for (int e0 = 0; e0 < list_run; e0 += 32) {
                const int e = e0 + lane;
                int val = 0;
                bool keep = false;
                if (e < list_run) {
                    const int x = list[e];
                    if (x < 0) {
                        const int o = x & 0x7FFFFFFF;
                        keep = (taken[o >> 5] >> (o & 31)) & 1u;
                        val = cidx[o];
                    } else {
                        keep = true;
                        val = x;
                    }
                }
                const unsigned m = __ballot_sync(0xffffffffu, keep);
                if (keep) out[out_run + __popc(m & lt)] = val;
                out_run += __popc(m);
            }
            return;
        }
    }
    // ---- Fallback (a threshold bucket of more than CAND keys, e.g. many equal
    // scores): the radix select on the key bits, then the selection walk.
    for (int j = lane; j < WH_SLOTS; j += 32) hist[j] = 0;
    __syncwarp();
    for_keys([&](float v) { atomicAdd(&hist[HB - 1 - (int)(topk_key(v) >> 20)], 1); });
    __syncwarp();
    unsigned prefix;
    int remaining, cnt;
    topk_pick<HB>(hist, KB, 0u, 20, lane, prefix, remaining, cnt);
    unsigned mask = 0xFFF00000u;
    if (cnt != remaining) {   // uniform
        __syncwarp();
        for (int j = lane; j < WH_SLOTS; j += 32) hist[j] = 0;
        __syncwarp();
        for_keys([&](float v) {
            const unsigned key = topk_key(v);
            if ((key & mask) == prefix) atomicAdd(&hist[HB - 1 - (int)((key >> 9) & (HB - 1))], 1);
        });
        __syncwarp();
        topk_pick<HB>(hist, remaining, prefix, 9, lane, prefix, remaining, cnt);
        mask = 0xFFFFFE00u;
        if (cnt != remaining) {
            __syncwarp();
            for (int j = lane; j < 512; j += 32) hist[j] = 0;
            __syncwarp();
            for_keys([&](float v) {
                const unsigned key = topk_key(v);
                if ((key & mask) == prefix) atomicAdd(&hist[511 - (int)(key & 511u)], 1);
            });
            __syncwarp();
            topk_pick<512>(hist, remaining, prefix, 0, lane, prefix, remaining, cnt);
            mask = 0xFFFFFFFFu;
        }
    }
    // Selection in index order: every key above the threshold, and the first
    // `remaining` equal to it.  Key 4 q + j of a step sits in lane q % 32, so the
    // keys taken before it are those of the lower lanes (one ballot per j) and of
    // its own lane's lower j.  Equal keys need their rank among the equal ones
    // seen so far; a step without any (the common case) skips that count.
    int eq_run = 0, out_run = 0;
    if (vec) {
        const unsigned lt = (1u << lane) - 1u;
        for (int q0 = 0; q0 < n4 && out_run < KB; q0 += 32 * U) {   // out_run is uniform
            float4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                v[u] = q0 + 32 * u + lane < n4 ? __ldg(sc4 + q0 + 32 * u + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + 32 * u + lane;
                const unsigned k[4] = {topk_key(v[u].x), topk_key(v[u].y), topk_key(v[u].z), topk_key(v[u].w)};
                bool take[4], eq[4];
                bool any_eq = false;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const bool in = 4 * q + j < n_valid;
                    const unsigned km = k[j] & mask;
                    take[j] = in && km > prefix;
                    eq[j] = in && km == prefix;
                    any_eq |= eq[j];
                }
                if (__any_sync(0xffffffffu, any_eq)) {   // uniform: rank the equal keys in index order
                    const int n_eq = eq[0] + eq[1] + eq[2] + eq[3];
                    const int incl = warp_incl_scan(n_eq, lane);
                    int eq_before = eq_run + incl - n_eq;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        take[j] = take[j] || (eq[j] && eq_before < remaining);
                        eq_before += eq[j];
                    }
                    eq_run += __shfl_sync(0xffffffffu, incl, 31);
                }
                int pos = out_run, mine = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const unsigned m = __ballot_sync(0xffffffffu, take[j]);
                    pos += __popc(m & lt);
                    out_run += __popc(m);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (take[j]) out[pos + mine++] = 4 * q + j;
            }
        }
    } else {
        const unsigned lt = (1u << lane) - 1u;
        for (int b0 = 0; b0 < n_valid; b0 += 32) {
            const int b = b0 + lane;
            const bool in = b < n_valid;
            const unsigned km = in ? (topk_key(sc[b]) & mask) : 0u;
            const bool eq = in && km == prefix;
            bool take = in && km > prefix;
            const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
            take = take || (eq && eq_run + __popc(eq_mask & lt) < remaining);
            eq_run += __popc(eq_mask);
            const unsigned take_mask = __ballot_sync(0xffffffffu, take);
            if (take) out[out_run + __popc(take_mask & lt)] = b;
            out_run += __popc(take_mask);
            if (out_run >= KB) break;   // uniform
        }
    }
}

// ------------------------------------------------------------------ host
size_t qsa_scores_bytes(int B, int n) { return (size_t)B * n * (n / qsa::R) * 4; }

size_t qsa_workspace_bytes(int B, int n) {
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return ru((size_t)B * n * qsa::HI * qsa::D * 2) + ru((size_t)B * (n / qsa::R) * qsa::D * 2) + ru((size_t)B * n * 4) +
           ru(qsa_scores_bytes(B, n));
}

cudaError_t launch_qsa_indexer(const QsaArgs &a, void *ws) {
    using namespace qsa;
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const int nb = a.n / R;
    char *p = static_cast<char *>(ws);
    __half *qr = reinterpret_cast<__half *>(p);
    p += ru((size_t)a.B * a.n * HI * D * 2);
    __half *kb = reinterpret_cast<__half *>(p);
    p += ru((size_t)a.B * nb * D * 2);
    float *rowmax = reinterpret_cast<float *>(p);   // per query row: its largest score
    p += ru((size_t)a.B * a.n * 4);
    float *scores = a.scores ? a.scores : reinterpret_cast<float *>(p);
    cudaError_t e;
    const long long items = (long long)a.B * a.n + (long long)a.B * nb;
    if (items == 0) return cudaSuccess;
    const long long want_blocks = (items + 7) / 8;
    int sms = 0;
    if ((e = sm_count(&sms)) != cudaSuccess) return e;
    const long long cap = 16LL * sms;   // 16 blocks of 256 threads per SM
    const int grid = (int)(want_blocks < cap ? want_blocks : cap);
    qsa_prep_kernel<<<grid, 256, 0, a.stream>>>((const bf16 *)a.q, (const bf16 *)a.k, a.w_q, a.w_k, a.B, a.n, qr, kb);
    if ((e = launched()) != cudaSuccess) return e;
    if (nb > 0) {
        QsaMaps m;
        std::memset(&m, 0, sizeof m);
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.q), qr, false, D, HI, a.B * a.n, 64, QT, true)) != cudaSuccess)
            return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.k), kb, false, D, 1, a.B * nb, 64, BN, true)) != cudaSuccess)
            return e;
        // score rows on 16-byte boundaries
        const bool tma_out = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
        if (tma_out && (e = make_tma_rows_f32(reinterpret_cast<TmaMap *>(&m.sc), scores, nb, a.B * a.n, EC, 32)) !=
                           cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(qsa_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM)) != cudaSuccess)
            return e;
        if ((e = cudaMemsetAsync(rowmax, 0, (size_t)a.B * a.n * 4, a.stream)) != cudaSuccess) return e;
        const long long n_items = qsa_score_items(a.B, a.n);
        const int g = (int)(n_items < sms ? n_items : sms);
        if (g > 0) {
            qsa_score_kernel<<<g, 64 + 32 * EPI_WARPS, SMEM, a.stream>>>(m, a.B, a.n, (int)n_items, tma_out, scores,
                                                                          rowmax);
            if ((e = launched()) != cudaSuccess) return e;
        }
    }
    if (a.n > 0) {
        const long long rows = (long long)a.B * a.n;
        const size_t smem = (size_t)TOPK_WARPS * WH_SLOTS * 4;
        if ((e = cudaFuncSetAttribute(qsa_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        qsa_topk_kernel<<<(unsigned)((rows + TOPK_WARPS - 1) / TOPK_WARPS), 32 * TOPK_WARPS, smem, a.stream>>>(
            scores, rowmax, a.n, rows, a.KB, a.sel);
        if ((e = launched()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// One CTA waits, through qsa_wait, for a barrier phase that nothing completes.
__global__ void qsa_wait_selftest_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        umma::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) qsa_wait(&bar, 0, max_polls);
}

cudaError_t qsa_wait_selftest(uint32_t max_polls, cudaStream_t s) {
    qsa_wait_selftest_kernel<<<1, 32, 0, s>>>(max_polls);
    return cudaGetLastError();
}

cudaError_t qsa_error_word(unsigned *v, bool clear, cudaStream_t s) {
    return read_error_word(g_qsa_err, v, clear, s);
}

}  // namespace gdn

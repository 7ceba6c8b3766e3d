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
//      stages; warp-specialised producer, MMA issuer and four epilogue warps
//      (ReLU, head sum, 128-byte row segments of the complete blocks' scores).
//      Only block tiles that hold a complete block of the query tile are visited.
//  K5c qsa_topk_kernel: one CTA per query row: a radix select on the score bits
//      (scores are >= 0, so their bit patterns order like the values; digits of
//      11, 11 and 9 bits, the first counted while the row is read into shared
//      memory, stopping at the first digit whose bucket is taken whole) finds the
//      threshold, then warp segments write the selected blocks in ascending
//      order, equal scores at the threshold taken from the smallest index.
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
__device__ __forceinline__ void qsa_norm_rope(float (&x)[4], const float *__restrict__ w, long long pos,
                                              int lane) {
    // lane holds dims lane, lane + 32, lane + 64, lane + 96
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) ss = fmaf(x[u], x[u], ss);
    ss = group_sum<32>(ss);
    const float rn = 1.0f / sqrtf(ss / qsa::D + kNormEps);
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] *= rn * __ldg(w + lane + 32 * u);
    // rotate the pair (lane, lane + 32) by pos * base^(-lane / 32)
    const double ang = (double)pos * pow(qsa::ROPE_BASE, -(double)lane / 32.0);
    double sd, cd;
    sincos(ang, &sd, &cd);
    const float c = (float)cd, s = (float)sd;
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
    for (long long it = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); it < n_items; it += (long long)gridDim.x * 8) {
        if (it < n_q) {   // query row (sequence it / n, token it % n), all heads
            const long long i = it % n;
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                const bf16 *src = q + (it * HI + h) * D;
                float x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) x[u] = __bfloat162float(src[lane + 32 * u]);
                qsa_norm_rope(x, w_q, i, lane);
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
            qsa_norm_rope(x, w_k, b * R, lane);
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
constexpr int OFF_BAR = OFF_B + NSB * B_STAGE;         // 180224
constexpr int SMEM = OFF_BAR + 256 + 1024;             // barriers, TMEM slot, abort flag; alignment slack
constexpr uint32_t TMEM_COLS = 512;                    // 2 stages x 4 heads x 64 columns
constexpr uint32_t MAX_POLLS = 1u << 24;
}  // namespace qsa

namespace {

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
};

// One CTA per SM walks the work items.  The four heads' query rows of the tile
// (4 x 128 rows x 128 dims fp16 = 128 KB) stay in shared memory for the item;
// block tiles (64 x 128 fp16 = 16 KB) stream through NSB stages.  Each head's
// product (M = 128 queries, N = 64 blocks, K = 128) goes to its own 64 TMEM
// columns, so the epilogue sums ReLU over the heads per (query lane, block
// column) with no shuffles; two TMEM stages let the MMAs of block tile j + 1 run
// while tile j's epilogue drains.
// Roles: warp 0 lane 0 issues the TMA loads, warp 1 lane 0 the MMAs (warp 1 owns
// the TMEM allocation), warps 2-5 are the epilogue (TMEM lane quadrant w % 4,
// one query per lane, 128-byte row segments of scores).  Barriers: full_a /
// empty_a (query tile), full_b / empty_b (block stages), tfull / tempty (TMEM
// stages; tempty takes one arrival per epilogue warp).  Every wait is bounded;
// a timeout raises the error word and an abort flag the other roles check.
__global__ void __launch_bounds__(192, 1)
qsa_score_kernel(const __grid_constant__ QsaMaps maps, int B, int n, int n_items, float *__restrict__ scores) {
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
            umma::mbar_init(tempty + i, 4);
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
        const int qd = warp & 3;
        const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
        const bool vec = (nb & 3) == 0;   // rows start on 16-byte boundaries
        QsaCursor cur;
        QsaItem item;
        int t_it = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            if (!qsa_find_item(it, B, n, cur, item)) break;
            const int i = QT * item.qt + 32 * qd + lane;   // this lane's query
            const int n_valid = i < n ? (i + 1) / R : 0;  // its complete blocks
            float *dst = scores + ((size_t)item.s * n + (i < n ? i : 0)) * nb;
            for (int j = 0; j < item.nbt; ++j, ++t_it) {
                const int ts = t_it & 1, v = t_it >> 1;
                ok = __all_sync(0xffffffffu, wait(tfull + ts, v & 1));
                if (!ok) break;
                umma::tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    float acc[32], x[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll
                    for (int h = 0; h < HI; ++h) {
                        umma::tmem_ld32(trow + ts * (HI * BN) + h * BN + c, x);
#pragma unroll
                        for (int e = 0; e < 32; ++e) acc[e] += fmaxf(x[e], 0.f);
                    }
                    const int bs = BN * (item.bt0 + j) + c;
                    if (vec && bs + 32 <= n_valid) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + bs);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d4[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (bs + e < n_valid) dst[bs + e] = acc[e];
                    }
                }
                umma::tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_local(tempty + ts);
            }
        }
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
constexpr int TOPK_CAP = 12288;      // row keys kept in shared memory up to this many blocks (48 KB)
constexpr int HB = 2048;             // buckets of the 11-bit digits
constexpr int HB_SLOTS = HB + HB / 32;   // with one pad counter per 32
}  // namespace qsa

// Counter of the bucket at descending rank u (u = NB - 1 - digit): one pad word
// per 32 counters, so the PER consecutive ranks that each thread of a warp scans
// fall in distinct banks (thread t reads ranks PER t .. PER t + PER - 1).
__device__ __forceinline__ int topk_slot(int u) { return u + (u >> 5); }

// One digit of the radix select: among the keys matching `prefix`, the bucket of
// the digit at `shift` (NB buckets) that holds the remaining-th largest key.
// Thread t sums the buckets of ranks PER t .. PER t + PER - 1 (descending
// digits); a block scan of those sums crosses `remaining` at exactly one thread,
// which walks its buckets and publishes the extended prefix, the rank left
// inside the bucket and the bucket's count.  Ends with a block barrier.
template <int NB>
__device__ __forceinline__ void topk_pick(const int *hist, int *wsum, int remaining, unsigned prefix, int shift,
                                          int tid, unsigned *sh_prefix, int *sh_rem, int *sh_cnt) {
    constexpr int PER = NB / 256;
    const int warp = tid >> 5, lane = tid & 31;
    int c = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) c += hist[topk_slot(PER * tid + j)];
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    for (int w = 0; w < warp; ++w) incl += wsum[w];
    int run = incl - c;
    if (incl >= remaining && run < remaining) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int h = hist[topk_slot(PER * tid + j)];
            if (run + h >= remaining) {
                *sh_prefix = prefix | ((unsigned)(NB - 1 - (PER * tid + j)) << shift);
                *sh_rem = remaining - run;
                *sh_cnt = h;
                break;
            }
            run += h;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ unsigned topk_key(float v) {
    return v > 0.f ? __float_as_uint(v) : 0u;   // scores >= 0: bits order like values (-0 -> 0)
}

// Shared state of one row's select.
struct TopkSmem {
    int hist[qsa::HB_SLOTS];
    int wsum[8];
    int wcnt[8][2];
    unsigned prefix;
    int rem, cnt;
};

// Histogram of the digit (key >> shift) & (NB - 1) over the keys with
// (key & mask) == prefix; SMEM: the keys are in shared memory (read 16 bytes at
// a time), else they are read from the score row.
template <bool SMEM, int NB>
__device__ __forceinline__ void topk_count(TopkSmem &S, const uint4 *keys4, const float *sc, int n_valid,
                                           unsigned mask, unsigned prefix, int shift, int tid) {
    if (SMEM) {
        const int n4 = (n_valid + 3) >> 2;
        for (int q = tid; q < n4; q += 256) {
            const uint4 kk = keys4[q];
            const unsigned k[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * q + j < n_valid && (k[j] & mask) == prefix)
                    atomicAdd(&S.hist[topk_slot(NB - 1 - (int)((k[j] >> shift) & (NB - 1)))], 1);
        }
    } else {
        for (int b = tid; b < n_valid; b += 256) {
            const unsigned key = topk_key(sc[b]);
            if ((key & mask) == prefix) atomicAdd(&S.hist[topk_slot(NB - 1 - (int)((key >> shift) & (NB - 1)))], 1);
        }
    }
}

template <bool SMEM>
__device__ __forceinline__ void topk_row(TopkSmem &S, uint4 *keys4, const float *__restrict__ sc, int nb,
                                         int n_valid, int KB, int32_t *__restrict__ out, int tid) {
    unsigned *keys_s = reinterpret_cast<unsigned *>(keys4);
    const int warp = tid >> 5, lane = tid & 31;
    for (int j = tid; j < qsa::HB_SLOTS; j += 256) S.hist[j] = 0;
    __syncthreads();
    // The keys (into shared memory when they fit) and the histogram of their first
    // digit, bits 30..20 (bit 31 of a key is 0).  Rows start on 16-byte boundaries
    // when nb % 4 == 0; the last quad may reach past n_valid, never past the row.
    if (SMEM && (nb & 3) == 0) {
        const float4 *sc4 = reinterpret_cast<const float4 *>(sc);
        const int n4 = (n_valid + 3) >> 2;
        for (int q = tid; q < n4; q += 256) {
            const float4 v = sc4[q];
            const unsigned k[4] = {topk_key(v.x), topk_key(v.y), topk_key(v.z), topk_key(v.w)};
            keys4[q] = make_uint4(k[0], k[1], k[2], k[3]);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * q + j < n_valid) atomicAdd(&S.hist[topk_slot(qsa::HB - 1 - (int)(k[j] >> 20))], 1);
        }
    } else {
        for (int b = tid; b < n_valid; b += 256) {
            const unsigned key = topk_key(sc[b]);
            if (SMEM) keys_s[b] = key;
            atomicAdd(&S.hist[topk_slot(qsa::HB - 1 - (int)(key >> 20))], 1);
        }
    }
    __syncthreads();
    // Radix select of the KB-th largest key with digits of 11, 11 and 9 bits.  A
    // digit whose bucket holds exactly the keys still wanted ends it early: every
    // key of that bucket is taken, so the lower bits need not be resolved.
    topk_pick<qsa::HB>(S.hist, S.wsum, KB, 0u, 20, tid, &S.prefix, &S.rem, &S.cnt);
    unsigned prefix = S.prefix, mask = 0xFFF00000u;
    int remaining = S.rem;
    if (S.cnt != remaining) {   // uniform
        for (int j = tid; j < qsa::HB_SLOTS; j += 256) S.hist[j] = 0;
        __syncthreads();
        topk_count<SMEM, qsa::HB>(S, keys4, sc, n_valid, mask, prefix, 9, tid);
        __syncthreads();
        topk_pick<qsa::HB>(S.hist, S.wsum, remaining, prefix, 9, tid, &S.prefix, &S.rem, &S.cnt);
        prefix = S.prefix;
        remaining = S.rem;
        mask = 0xFFFFFE00u;
        if (S.cnt != remaining) {
            for (int j = tid; j < topk_slot(512); j += 256) S.hist[j] = 0;
            __syncthreads();
            topk_count<SMEM, 512>(S, keys4, sc, n_valid, mask, prefix, 0, tid);
            __syncthreads();
            topk_pick<512>(S.hist, S.wsum, remaining, prefix, 0, tid, &S.prefix, &S.rem, &S.cnt);
            prefix = S.prefix;
            remaining = S.rem;
            mask = 0xFFFFFFFFu;
        }
    }
    // Selection: the keys whose masked bits are above the prefix, and the first
    // `remaining` equal to it in index order.  Warp w owns a contiguous segment of
    // the row (starting on a multiple of 32 when not empty); it counts its keys
    // above and equal, the warps exchange counts once, and each warp then writes
    // its selected blocks at their ascending positions.
    auto key_at = [&](int b) -> unsigned { return SMEM ? keys_s[b] : topk_key(sc[b]); };
    const int seg = (((n_valid + 7) / 8) + 31) / 32 * 32;
    const int b_lo = min(warp * seg, n_valid), b_hi = min(b_lo + seg, n_valid);
    int n_gt = 0, n_eq = 0;
    if (SMEM) {
        for (int q = (b_lo >> 2) + lane; 4 * q < b_hi; q += 32) {
            const uint4 kk = keys4[q];
            const unsigned k[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const unsigned km = k[j] & mask;
                const bool in = 4 * q + j >= b_lo && 4 * q + j < b_hi;   // an empty segment starts mid-quad
                n_gt += in && km > prefix;
                n_eq += in && km == prefix;
            }
        }
    } else {
        for (int b = b_lo + lane; b < b_hi; b += 32) {
            const unsigned km = key_at(b) & mask;
            n_gt += km > prefix;
            n_eq += km == prefix;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
        S.wcnt[warp][0] = n_gt;
        S.wcnt[warp][1] = n_eq;
    }
    __syncthreads();
    int gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
        gt_before += S.wcnt[w][0];
        eq_before += S.wcnt[w][1];
    }
    const unsigned lt = (1u << lane) - 1u;
    int eq_run = eq_before, out_run = gt_before + min(eq_before, remaining);
    for (int b0 = b_lo; b0 < b_hi; b0 += 32) {
        const int b = b0 + lane;
        const bool in = b < b_hi;
        const unsigned km = in ? (key_at(b) & mask) : 0u;
        const bool eq = in && km == prefix;
        bool take = in && km > prefix;
        const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
        if (eq_mask) {   // uniform
            take = take || (eq && eq_run + __popc(eq_mask & lt) < remaining);
            eq_run += __popc(eq_mask);
        }
        const unsigned take_mask = __ballot_sync(0xffffffffu, take);
        if (take) out[out_run + __popc(take_mask & lt)] = b;
        out_run += __popc(take_mask);
    }
}

__global__ void __launch_bounds__(256)
qsa_topk_kernel(const float *__restrict__ scores, int n, int KB, int32_t *__restrict__ sel) {
    extern __shared__ uint4 keys4[];   // the row's keys when n_valid <= TOPK_CAP
    __shared__ TopkSmem S;
    const int tid = threadIdx.x;
    const unsigned row = blockIdx.x;   // s * n + i (batch * n < 2^29)
    const int i = (int)(row % (unsigned)n);
    const int nb = n / qsa::R;
    const int n_valid = (i + 1) / qsa::R;
    const float *sc = scores + (size_t)row * nb;
    int32_t *out = sel + (size_t)row * KB;
    if (n_valid <= KB) {   // every complete block
        for (int j = tid; j < KB; j += 256) out[j] = j < n_valid ? j : -1;
        return;
    }
    if (n_valid <= qsa::TOPK_CAP)   // uniform
        topk_row<true>(S, keys4, sc, nb, n_valid, KB, out, tid);
    else
        topk_row<false>(S, keys4, sc, nb, n_valid, KB, out, tid);
}

// ------------------------------------------------------------------ host
size_t qsa_scores_bytes(int B, int n) { return (size_t)B * n * (n / qsa::R) * 4; }

size_t qsa_workspace_bytes(int B, int n) {
    auto ru = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return ru((size_t)B * n * qsa::HI * qsa::D * 2) + ru((size_t)B * (n / qsa::R) * qsa::D * 2) + ru(qsa_scores_bytes(B, n));
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
        if ((e = cudaFuncSetAttribute(qsa_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM)) != cudaSuccess)
            return e;
        const long long n_items = qsa_score_items(a.B, a.n);
        const int g = (int)(n_items < sms ? n_items : sms);
        if (g > 0) {
            qsa_score_kernel<<<g, 192, SMEM, a.stream>>>(m, a.B, a.n, (int)n_items, scores);
            if ((e = launched()) != cudaSuccess) return e;
        }
    }
    if (a.n > 0) {
        // the row's keys, rounded up to whole 16-byte quads
        const int cap = ((nb < qsa::TOPK_CAP ? nb : qsa::TOPK_CAP) + 3) & ~3;
        if ((e = cudaFuncSetAttribute(qsa_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cap * 4)) !=
            cudaSuccess)
            return e;
        qsa_topk_kernel<<<(unsigned)((long long)a.B * a.n), 256, (size_t)cap * 4, a.stream>>>(scores, a.n, a.KB,
                                                                                             a.sel);
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

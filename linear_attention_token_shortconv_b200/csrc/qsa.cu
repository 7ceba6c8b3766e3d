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
//  K5b qsa_score_kernel: tcgen05, one CTA of 8 warps per (32 queries = 128 rows
//      of (i, h), 256 blocks): both operands by TMA in the 128-byte swizzled
//      K-major layout, eight K = 16 MMAs into 256 TMEM columns; the epilogue
//      (two warps per TMEM lane quadrant, half the columns each) applies ReLU,
//      sums the 4 heads (lanes 4q .. 4q + 3) with two shuffles and stores the
//      scores of complete blocks.  Tiles entirely past the causal limit do nothing.
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
constexpr int QT = 32;          // queries per score tile (128 MMA rows)
constexpr int BT = 256;         // blocks per score tile (MMA N)
constexpr int OFF_A = 0;        // 2 k-blocks x 128 rows x 128 B
constexpr int OFF_B = 32768;    // 2 k-blocks x 256 rows x 128 B
constexpr int OFF_BAR = 98304;
constexpr int SMEM = OFF_BAR + 64 + 1024;
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
// Bounded wait of the score kernel: false (and the device error word raised)
// when the phase does not complete within max_polls polls.
__device__ __forceinline__ bool qsa_wait(uint64_t *bar, uint32_t parity, uint32_t max_polls) {
    const bool ok = umma::mbar_wait_bounded(bar, parity, max_polls);
    if (!ok) atomicOr(&g_qsa_err, 1u);
    return ok;
}

struct QsaMaps {
    CUtensorMap q, k;   // [rows][128] fp16, box {64, 128} and {64, 256}, 128-byte swizzle
};

__global__ void __launch_bounds__(256, 1)
qsa_score_kernel(const __grid_constant__ QsaMaps maps, int n, float *__restrict__ scores) {
    using namespace qsa;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + OFF_BAR);        // operand loads
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(sm + OFF_BAR + 8);   // MMA completion
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = n / R;
    const int bt = blockIdx.x, qt = blockIdx.y, s = blockIdx.z;
    const int i_last = min(QT * qt + QT - 1, n - 1);
    // complete blocks of the tile's last query; nothing to do past them
    if (BT * bt >= (i_last + 1) / R) return;   // uniform per CTA

    if (warp == 0) umma::tmem_alloc(tslot, BT);
    if (tid == 0) {
        umma::mbar_init(bar_ld, 1);
        umma::mbar_init(bar_mma, 1);
        umma::fence_mbar_init();
    }
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = *tslot;
    bool ok = true;
    if (tid == 0) {
        umma::mbar_expect_tx(bar_ld, 2 * 128 * 128 + 2 * 256 * 128);
        const int qrow = (s * n + QT * qt) * HI, krow = s * nb + BT * bt;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            umma::tma_load_3d(sm + OFF_A + kb * 16384, &maps.q, 64 * kb, 0, qrow, bar_ld);
            umma::tma_load_3d(sm + OFF_B + kb * 32768, &maps.k, 64 * kb, 0, krow, bar_ld);
        }
        ok = qsa_wait(bar_ld, 0, 1u << 24);
        if (ok) {
            umma::tc_fence_after();
            const uint32_t a = umma::smem_u32(sm + OFF_A), b = umma::smem_u32(sm + OFF_B);
            const uint32_t idesc = umma::idesc_f16(128, BT, false, false);
#pragma unroll
            for (int st = 0; st < D / 16; ++st) {
                const uint64_t ad = umma::sw128_desc(a + (st / 4) * 16384 + (st % 4) * 32, 16, 1024);
                const uint64_t bd = umma::sw128_desc(b + (st / 4) * 32768 + (st % 4) * 32, 16, 1024);
                umma::mma_f16(tbase, ad, bd, idesc, st > 0);
            }
            umma::mma_commit(bar_mma);
        }
    }
    ok = __syncthreads_and(ok);   // the MMA was issued
    if (ok) ok = __syncthreads_and(qsa_wait(bar_mma, 0, 1u << 24));
    if (ok) {
        umma::tc_fence_after();
        // warps w and w + 4: TMEM lanes 32 (w % 4) .. + 31 = rows (query 8 (w % 4) + l / 4,
        // head l % 4); warp w takes block columns 128 (w / 4) .. + 127
        const int quad = warp & 3, half = warp >> 2;
        const int i = QT * qt + 8 * quad + (lane >> 2);
        const int n_valid = (i + 1) / R;   // complete blocks of query i
        const uint32_t trow = tbase + ((uint32_t)(32 * quad) << 16);
        float *dst = scores + ((size_t)s * n + i) * nb;
        const bool vec = (nb & 3) == 0;   // rows start on 16-byte boundaries
#pragma unroll 1
        for (int c0 = (BT / 2) * half; c0 < (BT / 2) * (half + 1); c0 += 32) {
            if (BT * bt + c0 >= (i_last + 1) / R) break;   // uniform: nothing valid past here
            float v[32];
            umma::tmem_ld32(trow + c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float x = fmaxf(v[j], 0.f);
                x += __shfl_xor_sync(0xffffffffu, x, 1);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                v[j] = x;
            }
            // the 4 lanes of a query hold the same sums: lane 4q + j stores scores
            // 8j .. 8j + 7 of the chunk (two 16-byte stores when rows are aligned)
            const int j8 = 8 * (lane & 3);
            float o[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float a0 = v[x], a1 = v[8 + x], a2 = v[16 + x], a3 = v[24 + x];
                o[x] = j8 == 0 ? a0 : (j8 == 8 ? a1 : (j8 == 16 ? a2 : a3));
            }
            const int b0 = BT * bt + c0 + j8;
            if (i < n) {
                if (vec && b0 + 8 <= n_valid) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + b0);
                    d4[0] = make_float4(o[0], o[1], o[2], o[3]);
                    d4[1] = make_float4(o[4], o[5], o[6], o[7]);
                } else {
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        if (b0 + x < n_valid) dst[b0 + x] = o[x];
                }
            }
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tbase, BT);
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
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.q), qr, false, D, 1, a.B * a.n * HI, 64, 128, true)) != cudaSuccess)
            return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.k), kb, false, D, 1, a.B * nb, 64, BT, true)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(qsa_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM)) != cudaSuccess)
            return e;
        const dim3 g((nb + BT - 1) / BT, (a.n + QT - 1) / QT, a.B);
        qsa_score_kernel<<<g, 256, SMEM, a.stream>>>(m, a.n, scores);
        if ((e = launched()) != cudaSuccess) return e;
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

// The tensor-core prefill kernels: chunk prep (K2a), the chunk chain (K2b), and
// the fused persistent kernel that runs both with per-chunk ready flags, with
// their launchers, the device error words their bounded waits raise and the
// wait self-tests.  The kernel bodies are in prep_body.cuh and chain_body.cuh.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {
__device__ unsigned int g_prep_err;
__device__ unsigned int g_chain_err;
}  // namespace gdn

#include "prep_body.cuh"
#include "chain_body.cuh"

namespace gdn {

template <int DV>
__global__ void __launch_bounds__(256, 2)
chunk_prep_kernel(const PrepArgs pa, const int32_t *__restrict__ cu_seqlens, int n_seq,
                  int n_tok, int c_lo, int c_hi) {
    using namespace prep;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC + 768);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 784);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.x, n = blockIdx.y;
    int s_begin, s_end;
    if (cu_seqlens) { s_begin = __ldg(cu_seqlens + n); s_end = __ldg(cu_seqlens + n + 1); }
    else { const int L = n_tok / n_seq; s_begin = n * L; s_end = s_begin + L; }
    // chunks [c_lo, c_end) of this sequence, strided over blockIdx.z
    const int c_end = min((s_end - s_begin + C - 1) / C, c_hi);
    if (c_lo + (int)blockIdx.z >= c_end) return;   // uniform per block

    if (warp == 0) umma::tmem_alloc(tslot, TMEM_COLS);
    if (tid == 0) { umma::mbar_init(bar, 1); umma::fence_mbar_init(); }
    __syncthreads();
    const uint32_t tbase = *tslot;
    uint32_t phase = 0;
    for (int c = c_lo + blockIdx.z; c < c_end; c += gridDim.z) {
        // this block's next chunk: its raw rows into L2 while this one is processed
        if (c + (int)gridDim.z < c_end)
            prefetch_chunk_rows<DV>(pa.q, pa.k, pa.v, pa.H, h, s_begin + (c + gridDim.z) * C, s_end, tid);
        if (!prep_one_chunk<DV>(PrepBlockSync{}, pa, sm, tbase, bar, phase, tid, h, s_begin, s_end, c)) break;
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tbase, TMEM_COLS);
}

PrepArgs prep_args(const PrefillArgs &a, const TcWorkspace &w) {
    PrepArgs p;
    p.q = (const bf16 *)a.q; p.k = (const bf16 *)a.k; p.v = (const bf16 *)a.v; p.conv_w = a.conv_w;
    p.a_logit = (const bf16 *)a.a_logit; p.b_logit = (const bf16 *)a.b_logit;
    p.A = a.A; p.b_alpha = a.b_alpha; p.H = a.H;
    p.Qt = w.Qt; p.Kt = w.Kt; p.Wn = w.Wn; p.Up = w.Up; p.Aqk = w.Aqk; p.decay = w.decay;
    return p;
}

// Entries of the fused kernel's varlen task list: at most one per chunk of every
// (sequence, head), ceil(len / 64) <= len / 64 + 1 per sequence.
size_t fused_task_capacity(int n_tok, int n_seq, int H) { return ((size_t)n_tok / prep::C + n_seq) * H; }

// Tokens of the longest sequence, or their bound N_tok when cu_seqlens is given
// (device memory, not read on the host).
int longest_seq(const PrefillArgs &a) {
    return a.cu_seqlens || a.n_seq <= 0 ? a.n_tok : a.n_tok / a.n_seq;
}

cudaError_t launch_chunk_prep(const PrefillArgs &a, const TcWorkspace &w, int c_lo, int c_hi,
                              cudaStream_t stream) {
    if (a.n_tok == 0 || c_hi <= c_lo) return cudaSuccess;
    // blocks per (head, sequence): ~8 per SM / H in total, at most one per chunk
    // of the range (the longest sequence may fill it); blocks past the end exit
    const int max_chunks = (longest_seq(a) + 63) / 64;
    int sms = 0;
    if (cudaError_t es = sm_count(&sms)) return es;
    int split = max(1, (8 * sms) / a.H);
    split = min(split, min(c_hi, max_chunks) - c_lo);
    if (split <= 0) return cudaSuccess;
    dim3 grid(a.H, a.n_seq, split);
    cudaError_t e;
#define GDN_PREP(DV_)                                                                             \
    e = cudaFuncSetAttribute(chunk_prep_kernel<DV_>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             prep::SMEM);                                                          \
    if (e != cudaSuccess) return e;                                                                 \
    chunk_prep_kernel<DV_><<<grid, 256, prep::SMEM, stream>>>(prep_args(a, w), a.cu_seqlens, a.n_seq,  \
                                                              a.n_tok, c_lo, c_hi)
    if (!a.in_bf16) return cudaErrorInvalidValue;   // the tensor-core path takes bf16 inputs
    if (a.dv == 128) { GDN_PREP(128); } else { GDN_PREP(64); }
#undef GDN_PREP
    return launched();
}

cudaError_t launch_chunk_prep(const PrefillArgs &a, const TcWorkspace &w) {
    return launch_chunk_prep(a, w, 0, (a.n_tok + 63) / 64, a.stream);
}

// One CTA waits, through prep_wait, for a barrier phase that nothing completes.
__global__ void prep_wait_selftest_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        umma::fence_mbar_init();
    }
    __syncthreads();
    prep_wait(PrepBlockSync{}, &bar, 0, max_polls, threadIdx.x);
}

cudaError_t prep_wait_selftest(uint32_t max_polls, cudaStream_t s) {
    prep_wait_selftest_kernel<<<1, 64, 0, s>>>(max_polls);
    return cudaGetLastError();
}

cudaError_t prep_error_word(unsigned *v, bool clear, cudaStream_t s) {
    return read_error_word(g_prep_err, v, clear, s);
}


template <int DV, typename Tout>
__global__ void __launch_bounds__(4 * DV, 1)
chunk_chain_kernel(const __grid_constant__ ChainMaps maps, const float *__restrict__ decay,
                   const float *__restrict__ norm_w, const float *state_in,
                   const int32_t *__restrict__ cu_seqlens, int n_seq, int n_tok, int H, int c_lo,
                   int c_hi, Tout *__restrict__ out, float *state_out) {
    chain_body<DV, Tout>(maps, decay, norm_w, state_in, cu_seqlens, n_seq, n_tok, H, blockIdx.x, blockIdx.y,
                         c_lo, c_hi, out, state_out, nullptr);
}

cudaError_t launch_chunk_chain(const PrefillArgs &a, const TcWorkspace &w, int c_lo, int c_hi,
                               const float *state_in, float *state_out, cudaStream_t stream) {
    ChainMaps m;
    std::memset(&m, 0, sizeof m);
    if (a.n_tok > 0) {
        cudaError_t e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.wn), w.Wn, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.qt), w.Qt, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.kt), w.Kt, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.aqk), w.Aqk, false, 64, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.up), w.Up, false, a.dv, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.z), a.z, true, a.dv, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
        if (a.out_bf16 &&
            (e = make_tma_3d(reinterpret_cast<TmaMap *>(&m.out), a.out, true, a.dv, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    }
    dim3 grid(a.H, a.n_seq);
    cudaError_t e;
#define GDN_CHAIN(DV_, TOUT)                                                                      \
    e = cudaFuncSetAttribute(chunk_chain_kernel<DV_, TOUT>,                                       \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, chain::SMEM);            \
    if (e != cudaSuccess) return e;                                                               \
    chunk_chain_kernel<DV_, TOUT><<<grid, 4 * DV_, chain::SMEM, stream>>>(                        \
        m, w.decay, a.norm_w, state_in, a.cu_seqlens, a.n_seq, a.n_tok, a.H, c_lo, c_hi,        \
        (TOUT *)a.out, state_out)
    if (a.dv == 128) {
        if (a.out_bf16) { GDN_CHAIN(128, bf16); } else { GDN_CHAIN(128, float); }
    } else {
        if (a.out_bf16) { GDN_CHAIN(64, bf16); } else { GDN_CHAIN(64, float); }
    }
#undef GDN_CHAIN
    return launched();
}

cudaError_t launch_chunk_chain(const PrefillArgs &a, const TcWorkspace &w) {
    return launch_chunk_chain(a, w, 0, (a.n_tok + 63) / 64 + 1, a.S0, a.S_final, a.stream);
}

// One CTA waits, through chain_wait, for a barrier phase that nothing completes.
__global__ void chain_wait_selftest_kernel(uint32_t max_polls) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        abort_flag = 0;
        umma::fence_mbar_init();
    }
    __syncthreads();
    chain_wait(&bar, 0, &abort_flag, max_polls);
}

cudaError_t chain_wait_selftest(uint32_t max_polls, cudaStream_t s) {
    chain_wait_selftest_kernel<<<1, 32, 0, s>>>(max_polls);
    return cudaGetLastError();
}

cudaError_t chain_error_word(unsigned *v, bool clear, cudaStream_t s) {
    return read_error_word(g_chain_err, v, clear, s);
}

// ---------------------------------------------------------------------------
// Fused tensor-core prefill (dk = dv = 128): one persistent CTA of 512 threads
// per SM, launched cooperatively so that all CTAs are resident together.  CTAs
// [0, n_chain) each run the chain of one (sequence, head) over all its chunks;
// every other CTA runs two prep workers of 256 threads (named barriers 1 and 2,
// their own shared memory and 256 TMEM columns each) that take chunk tasks from
// a global counter in chunk-major order and, once a chunk's workspace rows are
// written, publish its ready flag with release semantics.  A chain CTA reads a
// chunk's rows only after acquiring that flag.  Prep workers never wait for a
// chain CTA, so every flag gets set; every wait is bounded all the same.
namespace fused {
constexpr int NT = 512;
constexpr int PREP_REGION = 104448;   // one prep worker's shared memory (1 KB aligned)
constexpr int SMEM = chain::SMEM > 2 * PREP_REGION + 1024 ? chain::SMEM : 2 * PREP_REGION + 1024;
static_assert(prep::OFF_MISC + prep::MISC_BYTES <= PREP_REGION, "prep worker region");
}  // namespace fused

struct FusedParams {
    ChainMaps maps;
    CUtensorMap raw_q, raw_k, raw_v;   // L2 prefetch of a chunk's raw rows (box: 67 rows of one head)
    PrepArgs pa;
    const float *norm_w, *S0;
    float *S_final;
    const int32_t *cu_seqlens;
    void *out;
    int *ready;        // [n_items][max_chunks], zero at launch
    int *next_task;    // zero at launch
    // packed varlen batches: the tasks (chunk << 8 | item) in order, their count, and
    // the items sorted by length (longest first); NULL for equal lengths
    const int *task_table, *n_tasks_dev, *order;
    int n_seq, n_tok, H, max_chunks, n_chain;
};

template <typename Tout>
__global__ void __launch_bounds__(fused::NT, 1) prefill_fused_kernel(const __grid_constant__ FusedParams P) {
    const int n_items = P.H * P.n_seq;
    if ((int)blockIdx.x < P.n_chain) {   // chain role: items blockIdx.x, + n_chain, .. in turn
        __shared__ uint32_t chain_tmem;
        if (threadIdx.x < 32) umma::tmem_alloc(&chain_tmem, 512);   // once: one permit per CTA
        umma::tc_fence_before();
        __syncthreads();
        umma::tc_fence_after();
        const uint32_t tbase = chain_tmem;
        for (int slot = blockIdx.x; slot < n_items; slot += P.n_chain) {
            const int item = P.order ? __ldg(P.order + slot) : slot;
            const int n = item / P.H, h = item % P.H;
            chain_body<128, Tout>(P.maps, P.pa.decay, P.norm_w, P.S0, P.cu_seqlens, P.n_seq, P.n_tok, P.H, h, n, 0,
                                  P.max_chunks + 1, reinterpret_cast<Tout *>(P.out), P.S_final,
                                  P.ready + (size_t)item * P.max_chunks, false, tbase);
        }
        umma::tc_fence_before();
        __syncthreads();
        if (threadIdx.x < 32) umma::tmem_dealloc(tbase, 512);
        return;
    }
    // prep role: two workers
    using namespace prep;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    const int tid = threadIdx.x, half = tid >> 8, wtid = tid & 255;
    uint8_t *wsm = sm + half * fused::PREP_REGION;
    uint64_t *bar = reinterpret_cast<uint64_t *>(wsm + OFF_MISC + 768);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 784);   // the CTA's allocation
    volatile int *task_slot = reinterpret_cast<volatile int *>(wsm + OFF_MISC + 800);   // [2]
    if (tid < 32) umma::tmem_alloc(tslot, 512);
    if (wtid == 0) {
        umma::mbar_init(bar, 1);
        umma::fence_mbar_init();
    }
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = *tslot + 256 * half;
    const PrepGroupSync sy{1 + half};
    const int n_tasks = P.task_table ? __ldg(P.n_tasks_dev) : P.max_chunks * n_items;
    uint32_t phase = 0;
    // the next task index is fetched one task ahead so the atomic's round trip
    // overlaps a chunk, by a thread of warp 7: warps 0 and 1 compute the gates
    // first thing in a chunk, warp 7 has time to wait for the atomic; a chunk's
    // ready flag is published during the next one
    // raw q, k, v rows of a task's chunk (and the three rows before it) into L2
    // Task t -> (chunk c, item): the items come in rounds of n_chain (the chain CTAs
    // take one item of each round in turn), and within a round chunk-major, so a
    // round's chunks are prepped in the order its chains consume them.
    auto task_at = [&](int t, int &c, int &item) {
        if (P.task_table) {
            const int e = __ldg(P.task_table + t);
            c = e >> 8;
            item = e & 255;
            return;
        }
        const int per_round = P.n_chain * P.max_chunks;
        const int r = t / per_round, local = t - r * per_round;
        const int in_round = min(P.n_chain, n_items - r * P.n_chain);
        c = local / in_round;
        item = r * P.n_chain + local % in_round;
    };
    auto prefetch_raw = [&](int t) {
        if (t >= n_tasks) return;
        int tc, it;
        task_at(t, tc, it);
        const int ns = it / P.H, hs = it % P.H;
        const int sb = P.cu_seqlens ? __ldg(P.cu_seqlens + ns) : ns * (P.n_tok / P.n_seq);
        const int row = sb + tc * C - 3;
        umma::tma_prefetch_l2_3d(&P.raw_q, 0, hs, row);
        umma::tma_prefetch_l2_3d(&P.raw_k, 0, hs, row);
        umma::tma_prefetch_l2_3d(&P.raw_v, 0, hs, row);
    };
    constexpr int kFetcher = 224;   // lane 0 of the worker's warp 7
    if (wtid == kFetcher) {
        task_slot[0] = atomicAdd(P.next_task, 1);
        prefetch_raw(task_slot[0]);
    }
    sy.sync();
    int task = task_slot[0];
    int *pending = nullptr;   // ready flag of the last chunk this worker wrote
    // Two task slots in turn: in iteration k the fetcher writes the next task to
    // slot (k + 1) % 2 before the chunk, and every thread reads it after the chunk.
    // The chunk's own barriers order that write before those reads, and the reads
    // of iteration k - 1 (the same slot) before the write.
    for (int k = 0; task < n_tasks; ++k) {
        const int ns = (k + 1) & 1;
        if (wtid == kFetcher) {
            const int nt = atomicAdd(P.next_task, 1);
            task_slot[ns] = nt;
            prefetch_raw(nt);
        }
        int c, item;
        task_at(task, c, item);
        const int n = item / P.H, h = item % P.H;
        int s_begin, s_end;
        if (P.cu_seqlens) { s_begin = __ldg(P.cu_seqlens + n); s_end = __ldg(P.cu_seqlens + n + 1); }
        else { const int L = P.n_tok / P.n_seq; s_begin = n * L; s_end = s_begin + L; }
        if (s_begin + c * C < s_end) {
            if (!prep_one_chunk<128>(sy, P.pa, wsm, tbase, bar, phase, wtid, h, s_begin, s_end, c, pending))
                break;
            pending = P.ready + (size_t)item * P.max_chunks + c;
        } else {
            sy.sync();   // past this sequence's end, no such chunk: the barrier the slots need
        }
        task = task_slot[ns];
    }
    if (pending && wtid == 0) {
        __threadfence();
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(pending), "r"(1) : "memory");
    }
    umma::tc_fence_before();
    __syncthreads();
    if (tid < 32) umma::tmem_dealloc(*tslot, 512);
}

// The fused kernel's task list for a packed varlen batch (one CTA): the items
// sorted by chunk count, longest first (equal counts by item index), taken in
// rounds of n_chain (the chain CTAs take one item of each round in turn), each
// round's tasks chunk-major: chunk c of every item of the round that has one.
// The task at (round r, chunk c, k-th item of the round) sits at
// base_r + sum_k' min(c, chunks_k') + k.
__global__ void fused_tasks_kernel(const int32_t *__restrict__ cu_seqlens, int n_seq, int H, int n_chain,
                                   int *__restrict__ table, int *__restrict__ n_tasks, int *__restrict__ order) {
    __shared__ int ch[256], ord[256], base[256];
    const int n_items = n_seq * H, tid = threadIdx.x;
    for (int i = tid; i < n_items; i += blockDim.x) {
        const int n = i / H;
        ch[i] = (__ldg(cu_seqlens + n + 1) - __ldg(cu_seqlens + n) + prep::C - 1) / prep::C;
    }
    __syncthreads();
    for (int i = tid; i < n_items; i += blockDim.x) {
        int rank = 0;
        for (int j = 0; j < n_items; ++j) rank += ch[j] > ch[i] || (ch[j] == ch[i] && j < i);
        ord[rank] = i;
    }
    __syncthreads();
    const int rounds = (n_items + n_chain - 1) / n_chain;
    if (tid == 0) {
        int run = 0;
        for (int r = 0; r < rounds; ++r) {
            base[r] = run;
            for (int k = r * n_chain; k < min(n_items, (r + 1) * n_chain); ++k) run += ch[ord[k]];
        }
        *n_tasks = run;
    }
    for (int i = tid; i < n_items; i += blockDim.x) order[i] = ord[i];
    __syncthreads();
    for (int r = 0; r < rounds; ++r) {
        const int k0 = r * n_chain, in_r = min(n_chain, n_items - k0);
        const int maxc = ch[ord[k0]];   // the round's longest item
        for (int c = tid; c < maxc; c += blockDim.x) {
            int off = base[r], alive = 0;
            for (int k = 0; k < in_r; ++k) {
                const int chk = ch[ord[k0 + k]];
                off += min(c, chk);
                alive += chk > c;   // the items still alive at c lead the round (sorted)
            }
            for (int k = 0; k < alive; ++k) table[off + k] = (c << 8) | ord[k0 + k];
        }
    }
}

int fused_chain_ctas(const PrefillArgs &a, int sms) {
    // The fused kernel leaves at least three quarters of the SMs to the prep
    // workers: one chain CTA per (sequence, head) up to sms / 4 of them.  With equal
    // lengths and up to one item per SM, sms / 4 chain CTAs take the items in turn
    // (an item's chunks are prepped in chunk order across all items, so the chains
    // a CTA takes later find theirs ready).  Packed varlen batches take a task list
    // built on the device (fused_tasks_kernel; items up to 256, chunk rows up to 2^23).
    const int items = a.H * a.n_seq;
    if (!(a.in_bf16 && a.dk == 128 && a.dv == 128 && a.n_tok > 0)) return 0;
    if (items <= sms / 4 && !a.cu_seqlens) return items;
    if (items > sms || items > 256 || (a.cu_seqlens && a.n_tok / prep::C > (1 << 22))) return 0;
    return items <= sms / 4 ? items : sms / 4;
}

cudaError_t launch_prefill_fused(const PrefillArgs &a, const TcWorkspace &w, int *ready, int sms,
                                 cudaStream_t stream) {
    const int n_chain = fused_chain_ctas(a, sms);
    if (n_chain == 0) return cudaErrorInvalidValue;
    FusedParams P;
    std::memset(&P, 0, sizeof P);
    cudaError_t e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.wn), w.Wn, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.qt), w.Qt, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.kt), w.Kt, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.aqk), w.Aqk, false, 64, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.up), w.Up, false, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.z), a.z, true, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if (a.out_bf16 &&
        (e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.maps.out), a.out, true, 128, a.H, a.n_tok, 64, 64, true)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.raw_q), a.q, true, 128, a.H, a.n_tok, 128, 67, false)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.raw_k), a.k, true, 128, a.H, a.n_tok, 128, 67, false)) != cudaSuccess) return e;
    if ((e = make_tma_3d(reinterpret_cast<TmaMap *>(&P.raw_v), a.v, true, 128, a.H, a.n_tok, 128, 67, false)) != cudaSuccess) return e;
    P.pa = prep_args(a, w);
    P.norm_w = a.norm_w;
    P.S0 = a.S0;
    P.S_final = a.S_final;
    P.cu_seqlens = a.cu_seqlens;
    P.out = a.out;
    P.n_seq = a.n_seq;
    P.n_tok = a.n_tok;
    P.H = a.H;
    P.max_chunks = (longest_seq(a) + 63) / 64;
    P.n_chain = n_chain;
    P.ready = ready;
    P.next_task = ready + (size_t)a.n_seq * a.H * P.max_chunks;
    if ((e = cudaMemsetAsync(ready, 0, ((size_t)a.n_seq * a.H * P.max_chunks + 1) * sizeof(int), stream)) != cudaSuccess)
        return e;
    if (a.cu_seqlens) {   // the task list, after the flags and the counter
        int *tasks = P.next_task + 1;
        int *n_tasks = tasks + fused_task_capacity(a.n_tok, a.n_seq, a.H);
        int *order = n_tasks + 1;
        fused_tasks_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.n_seq, a.H, n_chain, tasks, n_tasks, order);
        if ((e = launched()) != cudaSuccess) return e;
        P.task_table = tasks;
        P.n_tasks_dev = n_tasks;
        P.order = order;
    }
    void *args[] = {&P};
    const void *fn = a.out_bf16 ? reinterpret_cast<const void *>(prefill_fused_kernel<bf16>)
                                : reinterpret_cast<const void *>(prefill_fused_kernel<float>);
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, fused::SMEM)) != cudaSuccess)
        return e;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, fused::NT, fused::SMEM)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    // one CTA per SM: every CTA resident at once (the launch fails otherwise)
    e = cudaLaunchCooperativeKernel(fn, dim3(sms), dim3(fused::NT), args, fused::SMEM, stream);
    if (e != cudaSuccess) return e;
    return launched();
}

}  // namespace gdn

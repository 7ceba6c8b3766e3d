// K2b -- the state-dependent part of the chunked gated delta rule, sequential
// over the chunks of one (sequence, head), with the output gate and the
// zero-centred RMSNorm fused (slinene.github.io write-up of "On the Design of
// Qwen3.8-Next Architecture", 模块 A: 递归状态 and 参数化).
//
// Per chunk, with the chunk-prep tensors (-W, U', Qt, Kt, Aqk, e^{G_C}) and the
// state S before the chunk:
//     P[0:64]   = (-W) S      then U = U' + P[0:64]      (tcgen05 + registers)
//     P[64:128] = Qt S        (= diag(e^G) Q S)
//     P[64:128] += Aqk U      = Y                        (tcgen05)
//     D         = e^{G_C} S   (written into tensor memory ahead of time)
//     D        += Kt^T U      = the next chunk's S        (tcgen05)
//     out       = sigmoid(z) * Y / sqrt(mean(Y^2) + eps) * (1 + w)
// (sigmoid(z) = (1 + tanh(z/2)) / 2 with the hardware tanh on fp16 pairs: absolute
// error about 2^-12 on the gate, applied linearly to the normalised output)
//
// One CTA of 8 * DV / 64 warps per (sequence, head), in three roles that never
// wait for one another except where the data flows.  A warp reaches only its
// own quadrant (w % 4) of the 128 tensor-memory lanes, so:
//   * U warps   (quadrants 0, 1; 64 state columns each): U = U' + P[0:64] ->
//     fp16 B operand; thread 0 issues every MMA;
//   * Y warps   (quadrants 2, 3; 64 columns each): the gated RMSNorm of Y and
//     the output stores; thread 64 also issues the tile loads (operand tiles two
//     chunks ahead, and the z tiles of the gate two chunks ahead);
//   * S warps   (all quadrants, 64 columns each): S = D -> fp16 B operand of the
//     next chunk's first MMA, then e^{G_C} S of the next chunk back into D.
// The fp32 state lives in tensor memory (D) from chunk to chunk.  Per chunk the
// critical path is: P MMA -> U warps -> Kt^T U MMA -> S warps -> next P MMA.
// The Aqk U MMA runs while the S warps work, and the output stage of chunk c
// overlaps the chunks after it (P has three buffers in tensor memory).  Operand tiles
// of chunk c + 2 are loaded by TMA (128-byte swizzled) into the stage chunk c
// used as soon as chunk c's last MMA has completed.  Every wait is bounded.
//
// Device code only: the kernels that run it and the device error word it raises
// (g_chain_err, defined before this header is included) live in prefill_tc.cu.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {


namespace chain {
constexpr int C = 64;
constexpr int DK = 128;
// one stage: [-W; Qt] 32 KB | Kt 16 KB | Aqk 8 KB | U' 16 KB (DV = 128)
constexpr int ST_AP = 0, ST_AS = 32768, ST_AQK = 49152, ST_US = 57344;
constexpr int STAGE = 73728;
constexpr int OFF_BP = 2 * STAGE;          // S fp16 MN-major (rows = dk), 32 KB
constexpr int OFF_BU = OFF_BP + 32768;     // U fp16 MN-major (rows = tokens), 16 KB
constexpr int OFF_Z = OFF_BU + 16384;      // z tiles of two chunks, 2 x 16 KB
constexpr int ZBUF = 16384;
constexpr int OFF_MISC = OFF_Z + 2 * ZBUF;
// misc: barriers [0, 120), 1 + w [128, 640), partial sums [640, 1152); + alignment slack
constexpr int SMEM = OFF_MISC + 1152 + 1024;
static_assert(SMEM <= 232448, "227 KB per block");
constexpr uint32_t kMaxPolls = 1u << 24;
}  // namespace chain

struct ChainMaps {
    CUtensorMap wn, qt, kt, aqk, up, z;
};

// tanh of two halves on the special-function unit, one instruction for the pair
// (absolute error about 2^-11, the f16 result's own rounding)
__device__ __forceinline__ uint32_t tanh_approx_h2(uint32_t x) {
    uint32_t r;
    asm("tanh.approx.f16x2 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(umma::pack_half2(x[0], x[1]), umma::pack_half2(x[2], x[3]),
                      umma::pack_half2(x[4], x[5]), umma::pack_half2(x[6], x[7]));
}

__device__ __forceinline__ void unpack8h(uint4 u, float *x) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

template <typename Tout> __device__ __forceinline__ void store8_out(Tout *p, const float (&x)[8]);
template <> __device__ __forceinline__ void store8_out<float>(float *p, const float (&x)[8]) {
    store8(p, x);
}
template <> __device__ __forceinline__ void store8_out<bf16>(bf16 *p, const float (&x)[8]) {
    uint4 u;
    uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t *>(&b);
    }
    *reinterpret_cast<uint4 *>(p) = u;
}

// Bounded wait; on expiry raise the CTA's abort flag and the device error word.
// Once the flag is up every other wait of the CTA gives up quickly, so the
// kernel always finishes.
__device__ __forceinline__ bool chain_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           uint32_t max_polls = chain::kMaxPolls) {
    for (uint32_t i = 0; i < max_polls; ++i) {
        if (umma::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicOr(&g_chain_err, 1u);
    return false;
}

// Spin (bounded, with back-off) until a chunk's ready flag, published with release
// semantics by the prep worker that wrote its workspace rows, is set; then make the
// async proxy (the TMA loads that follow) observe those rows.
__device__ __forceinline__ bool wait_ready(const int *flag, volatile int *abort_flag) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        if (*abort_flag) return false;
        __nanosleep(i < 64 ? 32 : 256);
    }
    *abort_flag = 1;
    atomicOr(&g_chain_err, 1u);
    return false;
}

// chain_wait by lane 0 of a warp, its result broadcast: the warp leaves together
// (the tensor-memory loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = chain_wait(bar, parity, abort_flag);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(umma::smem_u32(bar)) : "memory");
}

// Threads of the chain CTA for a head dimension dv (8 warps per 64 columns).
template <int DV> constexpr int chain_threads() { return 8 * (DV / 64) * 32; }

// The chain of head h of sequence n over chunks [c_lo, c_hi), by a CTA of
// chain_threads<DV>() threads.  With `ready` non-NULL (the fused prefill kernel)
// the workspace rows of chunk c are read only after ready[c] is set.
template <int DV, typename Tout>
__device__ __forceinline__ void chain_body(const ChainMaps &maps, const float *__restrict__ decay,
                                           const float *__restrict__ norm_w, const float *state_in,
                                           const int32_t *__restrict__ cu_seqlens, int n_seq, int n_tok,
                                           int H, int h, int n, int c_lo, int c_hi,
                                           const bf16 *__restrict__ z, Tout *__restrict__ out,
                                           float *state_out, const int *ready) {
    using namespace chain;
    constexpr int CH = DV / 64;                 // 64-column halves of the state
    constexpr int NRW = 4 * CH;                 // warps of the U and Y roles (rows x halves)
    constexpr int N_U = 64 * CH;                // U threads (quadrants 0, 1)
    constexpr int N_Y = 64 * CH;                // Y threads (quadrants 2, 3)
    constexpr int N_S = 128 * CH;               // S threads
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint8_t *sBP = sm + OFF_BP, *sBU = sm + OFF_BU;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_MISC);   // [2] tiles of a stage landed
    uint64_t *full_z = full + 2;       // [2] z tile of a chunk landed
    uint64_t *pfree = full + 4;        // [3] output stage done reading P buffer b
    uint64_t *bar_p = full + 7;        // P MMA done
    uint64_t *u_ready = full + 8;      // U tile written
    uint64_t *bar_s = full + 9;        // D = next S complete
    uint64_t *s_ready = full + 10;     // fp16 S written
    uint64_t *d_ready = full + 11;     // e^{G_C} S stored into D
    // [3] Y of the chunk in P buffer b complete.  One barrier per buffer: the output
    // warps may fall up to two chunks behind, and a parity wait must never see a
    // barrier that has completed two phases past the one it waits for.
    uint64_t *bar_y = full + 12;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 120);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 124);
    float *w1 = reinterpret_cast<float *>(sm + OFF_MISC + 128);      // 1 + norm_w  [DV]
    float *red = w1 + 128;                                            // [CH][64] partial sums of Y^2
    constexpr uint32_t TMEM_COLS = DV == 128 ? 512 : 256;   // P0, P1, P2, D
    constexpr uint32_t BYTES_Z = C * DV * 2;
    constexpr uint32_t BYTES_A = 4 * 8192 + 2 * 8192 + 8192 + C * DV * 2;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3;
    int s_begin, s_end;
    if (cu_seqlens) { s_begin = __ldg(cu_seqlens + n); s_end = __ldg(cu_seqlens + n + 1); }
    else { const int L = n_tok / n_seq; s_begin = n * L; s_end = s_begin + L; }
    // chunks [c_lo, c_end) of this sequence; the state enters from state_in (NULL:
    // zeros) and leaves to state_out (NULL: dropped); they may be the same buffer
    const int c_end = min((s_end - s_begin + C - 1) / C, c_hi);
    const int n_chunks = max(0, c_end - c_lo);   // chunks handled by this launch
    const size_t sbase = ((size_t)n * H + h) * DK * DV;

    if (warp == 0) umma::tmem_alloc(tslot, TMEM_COLS);
    if (tid == 0) {
        umma::mbar_init(full, 1);
        umma::mbar_init(full + 1, 1);
        umma::mbar_init(full_z, 1);
        umma::mbar_init(full_z + 1, 1);
        umma::mbar_init(pfree, N_Y);
        umma::mbar_init(pfree + 1, N_Y);
        umma::mbar_init(pfree + 2, N_Y);
        umma::mbar_init(bar_p, 1);
        umma::mbar_init(u_ready, N_U);
        umma::mbar_init(bar_s, 1);
        umma::mbar_init(bar_y, 1);
        umma::mbar_init(bar_y + 1, 1);
        umma::mbar_init(bar_y + 2, 1);
        umma::mbar_init(s_ready, N_S);
        umma::mbar_init(d_ready, N_S);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    for (int j = tid; j < DV; j += blockDim.x) w1[j] = 1.0f + __ldg(norm_w + j);
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t tD = tbase + 3 * DV;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;

    auto stage = [&](int b) { return sm + b * STAGE; };
    // Tile loads of chunk cc (index within this launch) into stage b, after its
    // ready flag (fused kernel).  Issued by one thread.
    auto issue = [&](int cc, int b) {
        const int t0 = s_begin + (c_lo + cc) * C;
        uint8_t *st = stage(b);
        if (ready) wait_ready(ready + c_lo + cc, abort_flag);
        umma::mbar_expect_tx(full + b, BYTES_A);
        umma::tma_load_3d(st + ST_AP, &maps.wn, 0, h, t0, full + b);
        umma::tma_load_3d(st + ST_AP + 8192, &maps.qt, 0, h, t0, full + b);
        umma::tma_load_3d(st + ST_AP + 16384, &maps.wn, 64, h, t0, full + b);
        umma::tma_load_3d(st + ST_AP + 24576, &maps.qt, 64, h, t0, full + b);
        umma::tma_load_3d(st + ST_AS, &maps.kt, 0, h, t0, full + b);
        umma::tma_load_3d(st + ST_AS + 8192, &maps.kt, 64, h, t0, full + b);
        umma::tma_load_3d(st + ST_AQK, &maps.aqk, 0, h, t0, full + b);
#pragma unroll
        for (int x = 0; x < DV; x += 64) umma::tma_load_3d(st + ST_US + x * 128, &maps.up, x, h, t0, full + b);
    };
    // z tile (the gate's input) of chunk cc into z buffer b
    auto issue_z = [&](int cc, int b) {
        const int t0 = s_begin + (c_lo + cc) * C;
        umma::mbar_expect_tx(full_z + b, BYTES_Z);
#pragma unroll
        for (int x = 0; x < DV; x += 64)
            umma::tma_load_3d(sm + OFF_Z + b * ZBUF + x * 128, &maps.z, x, h, t0, full_z + b);
    };
    constexpr int kTma = 64;   // the loads' issuing thread: lane 0 of warp 2 (a Y warp)
    if (tid == kTma) {
        umma::prefetch_tensormap(&maps.wn);
        umma::prefetch_tensormap(&maps.qt);
        umma::prefetch_tensormap(&maps.kt);
        umma::prefetch_tensormap(&maps.aqk);
        umma::prefetch_tensormap(&maps.up);
        umma::prefetch_tensormap(&maps.z);
        for (int cc = 0; cc < 2 && cc < n_chunks; ++cc) issue_z(cc, cc);
        for (int cc = 0; cc < 2 && cc < n_chunks; ++cc) issue(cc, cc);
    }
    // byte offset of the 8-column chunk `col` of row i in a 64-column-block swizzled tile
    auto tile_off = [](int i, int col) { return (col / 64) * 8192 + umma::sw128_offset(i, (col % 64) / 8); };

    if (warp >= NRW) {
        // ===================================================== S warps
        const int ch = (warp - NRW) >> 2, col0 = 64 * ch;
        const int srow = 32 * q + lane;
        // the state entering the first chunk: fp16 copy (B operand) and e^{G_C} S into D
        float S[64];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            float x[8];
            if (state_in) load8(state_in + sbase + (size_t)srow * DV + col0 + 8 * m, x);
            else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) S[8 * m + e] = x[e];
            const int col = col0 + 8 * m;
            umma::st_chunk(sBP + (col / 64) * 16384, srow, (col % 64) / 8, pack8(x));
        }
        umma::fence_proxy_async_smem();
        mbar_arrive(s_ready);
        for (int c = 0; c < n_chunks; ++c) {
            // e^{G_C} S of chunk c into D (the accumulator of its Kt^T U MMA)
            if (!warp_wait(full + (c & 1), (uint32_t)(c >> 1) & 1u, abort_flag)) break;
            const float dec = __ldcg(decay + (size_t)(s_begin + (c_lo + c) * C) * H + h);
#pragma unroll
            for (int j = 0; j < 64; ++j) S[j] *= dec;   // S is reloaded from D after the chunk
            umma::tmem_st32(tD + lane_off + col0, *reinterpret_cast<const float(*)[32]>(S));
            umma::tmem_st32(tD + lane_off + col0 + 32, *reinterpret_cast<const float(*)[32]>(S + 32));
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            umma::tc_fence_before();
            mbar_arrive(d_ready);
            // the state after chunk c: fp16 copy for chunk c + 1's first MMA
            if (!warp_wait(bar_s, (uint32_t)c & 1u, abort_flag)) break;
            umma::tc_fence_after();
            umma::tmem_ld32(tD + lane_off + col0, *reinterpret_cast<float(*)[32]>(S));
            umma::tmem_ld32(tD + lane_off + col0 + 32, *reinterpret_cast<float(*)[32]>(S + 32));
            if (c + 1 < n_chunks) {
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int col = col0 + 8 * m;
                    umma::st_chunk(sBP + (col / 64) * 16384, srow, (col % 64) / 8, pack8(S + 8 * m));
                }
                umma::fence_proxy_async_smem();
                umma::tc_fence_before();
                mbar_arrive(s_ready);
            }
        }
        if (state_out && !*abort_flag) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = S[8 * m + e];
                store8(state_out + sbase + (size_t)srow * DV + col0 + 8 * m, x);
            }
        }
    } else if (q < 2) {
        // ===================================================== U warps (+ the MMA issuer)
        const int ch = warp >> 2, col0 = 64 * ch;
        const int i = 32 * q + lane;   // token row of the chunk
        const uint64_t dBP = umma::sw128_desc(umma::smem_u32(sBP), 16384, 1024);
        const uint64_t dBU = umma::sw128_desc(umma::smem_u32(sBU), 8192, 1024);
        const uint32_t id_p = umma::idesc_f16(128, DV, false, true);
        const uint32_t id_s = umma::idesc_f16(128, DV, true, true);
        for (int c = 0; c < n_chunks; ++c) {
            const int b = c & 1;
            const int t0 = s_begin + (c_lo + c) * C;
            const int len = min(C, s_end - t0);
            const uint32_t ph_stage = (uint32_t)(c >> 1) & 1u, ph = (uint32_t)c & 1u;
            uint8_t *st = stage(b);
            const int pb = c % 3;
            const uint32_t tP = tbase + pb * DV;
            if (tid == 0) {
                // ---- P = [-W; Qt] S  (M=128, N=DV, K=dk)
                bool ok = chain_wait(full + b, ph_stage, abort_flag);
                ok = ok && chain_wait(s_ready, ph, abort_flag);
                if (c >= 3) ok = ok && chain_wait(pfree + pb, (uint32_t)((c - 3) / 3) & 1u, abort_flag);
                umma::tc_fence_after();
                if (ok) {
                    const uint64_t dA = umma::sw128_desc(umma::smem_u32(st + ST_AP), 16, 1024);
#pragma unroll
                    for (int s = 0; s < DK / 16; ++s)
                        umma::mma_f16(tP, dA + (uint64_t)(((s / 4) * 16384 + (s % 4) * 32) >> 4),
                                      dBP + (uint64_t)((s * 2048) >> 4), id_p, s > 0);
                }
                umma::mma_commit(bar_p);
            }
            __syncwarp();
            // U' of this thread's row and columns, read while the MMA runs
            if (!warp_wait(full + b, ph_stage, abort_flag)) break;
            uint4 upk[8];
#pragma unroll
            for (int m = 0; m < 8; ++m)
                upk[m] = *reinterpret_cast<const uint4 *>(st + ST_US + tile_off(i, col0 + 8 * m));
            if (i >= len) {
                // rows past the end of a ragged chunk belong to another sequence (or lie
                // past the tensor) and may not be written yet: Kt^T U multiplies them by
                // U = 0, so make them zero rather than trust them to be finite (row i of
                // both 64-column blocks of Kt: block ch, and block 1 too when CH = 1)
                for (int kb = ch; kb < 2; kb += CH) {
#pragma unroll
                    for (int m = 0; m < 8; ++m)
                        *reinterpret_cast<uint4 *>(st + ST_AS + kb * 8192 + i * 128 + 16 * m) = make_uint4(0, 0, 0, 0);
                }
            }
            if (!warp_wait(bar_p, ph, abort_flag)) break;
            umma::tc_fence_after();
            // ---- U = U' + P[0:64] (zero past the sequence end) -> fp16 MN-major B operand
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                umma::tmem_ld32(tP + lane_off + col0 + 32 * half, v);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int col = col0 + 32 * half + 8 * m;
                    float up[8], u[8];
                    unpack8h(upk[4 * half + m], up);
#pragma unroll
                    for (int e = 0; e < 8; ++e) u[e] = (i < len) ? v[8 * m + e] + up[e] : 0.f;
                    umma::st_chunk(sBU + (col / 64) * 8192, i, (col % 64) / 8, pack8(u));
                }
            }
            umma::fence_proxy_async_smem();
            umma::tc_fence_before();
            mbar_arrive(u_ready);
            if (tid == 0) {
                // ---- D += Kt^T U (D holds e^{G_C} S): the next state;  P[64:128] += [*; Aqk] U
                bool ok = chain_wait(u_ready, ph, abort_flag);
                ok = ok && chain_wait(d_ready, ph, abort_flag);
                umma::tc_fence_after();
                if (ok) {
                    const uint64_t dS = umma::sw128_desc(umma::smem_u32(st + ST_AS), 8192, 1024);
                    const uint64_t dY = umma::sw128_desc(umma::smem_u32(st + ST_AS + 8192), 16, 1024);
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        umma::mma_f16(tD, dS + (uint64_t)((s * 2048) >> 4), dBU + (uint64_t)((s * 2048) >> 4), id_s, 1u);
                    umma::mma_commit(bar_s);
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        umma::mma_f16(tP, dY + (uint64_t)((s * 32) >> 4), dBU + (uint64_t)((s * 2048) >> 4), id_p, 1u);
                }
                umma::mma_commit(bar_y + pb);
                if (!ok) umma::mma_commit(bar_s);
            }
            __syncwarp();
        }
    } else {
        // ===================================================== Y warps (+ the tile loads)
        const int ch = warp >> 2, col0 = 64 * ch;
        const int i = 32 * (q - 2) + lane;   // token row of the chunk
        // output gain of this thread's columns, halved: sigmoid(z) (1 + w) y =
        // (1 + tanh(z / 2)) * ((1 + w) / 2) * y
        for (int c = 0; c < n_chunks; ++c) {
            const int b = c & 1, pb = c % 3;
            const int t0 = s_begin + (c_lo + c) * C;
            const int len = min(C, s_end - t0);
            const uint32_t tP = tbase + pb * DV;
            const size_t g = ((size_t)(t0 + i) * H + h) * DV + col0;
            if (!warp_wait(bar_y + pb, (uint32_t)(c / 3) & 1u, abort_flag)) break;
            umma::tc_fence_after();
            // chunk c's stage is free (its last MMA is done): load chunk c + 2 into it
            if (tid == kTma && c + 2 < n_chunks) issue(c + 2, b);
            __syncwarp();
            float ss = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float y[32];
                umma::tmem_ld32(tP + lane_off + col0 + 32 * half, y);
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 32; ++j) s4[j & 3] = fmaf(y[j], y[j], s4[j & 3]);
                ss += (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            red[ch * 64 + i] = ss;
            umma::named_bar_sync(1, N_Y);
            float tot = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < CH; ++g2) tot += red[g2 * 64 + i];
            const float rr = 0.5f * rsqrtf(tot / DV + kNormEps);
            if (!warp_wait(full_z + b, (uint32_t)(c >> 1) & 1u, abort_flag)) break;
            const uint8_t *zt = sm + OFF_Z + b * ZBUF;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float y[32];
                umma::tmem_ld32(tP + lane_off + col0 + 32 * half, y);
                if (i < len) {
                    const float2 rr2 = make_float2(rr, rr);
                    const float2 half2f = make_float2(0.5f, 0.5f);
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int col = col0 + 32 * half + 8 * m;
                        const uint4 zz = *reinterpret_cast<const uint4 *>(zt + tile_off(i, col));
                        const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
                        const float4 wa = *reinterpret_cast<const float4 *>(w1 + col);
                        const float4 wb = *reinterpret_cast<const float4 *>(w1 + col + 4);
                        const float2 wp[4] = {make_float2(wa.x, wa.y), make_float2(wa.z, wa.w),
                                              make_float2(wb.x, wb.y), make_float2(wb.z, wb.w)};
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 8 * m + 2 * e;
                            // (1 + tanh(z / 2)) * y * rr * (1 + w) / 2, two columns at a time
                            const float2 zh = fmul2(make_float2(bf16lo(zw[e]), bf16hi(zw[e])), half2f);
                            const uint32_t th = tanh_approx_h2(umma::pack_half2(zh.x, zh.y));
                            const float2 tf = __half22float2(*reinterpret_cast<const __half2 *>(&th));
                            const float2 a = fmul2(fmul2(make_float2(y[j], y[j + 1]), wp[e]), rr2);
                            const float2 r2 = ffma2(a, tf, a);
                            o[2 * e] = r2.x;
                            o[2 * e + 1] = r2.y;
                        }
                        store8_out<Tout>(out + g + 32 * half + 8 * m, o);
                    }
                }
            }
            // P buffer pb may be overwritten (by chunk c + 3's first MMA) once every
            // output thread has read it
            umma::tc_fence_before();
            mbar_arrive(pfree + pb);
            // every partial sum and z element of this chunk read: z buffer b takes chunk c + 2
            umma::named_bar_sync(1, N_Y);
            if (tid == kTma && c + 2 < n_chunks) issue_z(c + 2, b);
            __syncwarp();
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0 && n_chunks > 0) {
        // let any tile copy still in flight land before the CTA exits (bounded)
        for (int b = 0; b < 2 && b < n_chunks; ++b) {
            const int last = ((n_chunks - 1 - b) / 2) * 2 + b;   // last chunk that used stage b
            umma::mbar_wait_bounded(full + b, (uint32_t)(last >> 1) & 1u, 1u << 16);
            umma::mbar_wait_bounded(full_z + b, (uint32_t)(last >> 1) & 1u, 1u << 16);
        }
    }
    if (warp == 0) umma::tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn

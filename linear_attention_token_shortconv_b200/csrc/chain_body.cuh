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
//     dS        = Kt^T U                                  (tcgen05)
//     S         = e^{G_C} S + dS                          (fp32, registers)
//     out       = sigmoid(z) * Y / sqrt(mean(Y^2) + eps) * (1 + w)
// (sigmoid(z) = (1 + tanh(z/2)) / 2 with the hardware tanh: absolute error
// about 2^-12 on the gate, applied linearly to the normalised output)
//
// One CTA of 4 * dv threads per (sequence, head).  Warp w reads tensor-memory
// lane quadrant w % 4 and owns the 32-column group w / 4: each thread holds 32
// columns of one row of the fp32 state S [dk=128][dv], and an fp16 copy of S in
// shared memory is the B operand of the next chunk.  Tiles of the next chunk
// arrive by TMA (128-byte swizzled) into a second stage while the current chunk
// runs; P is double-buffered in tensor memory so the output stage of chunk c
// (quadrants 2, 3) overlaps the first MMA and the U conversion of chunk c + 1
// (quadrants 0, 1).  Every wait is bounded.
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
// one stage: [-W; Qt] 32 KB | Kt 16 KB | Aqk 8 KB | U' 16 KB | z 16 KB
constexpr int ST_AP = 0, ST_AS = 32768, ST_AQK = 49152, ST_US = 57344, ST_ZS = 73728;
constexpr int STAGE = 90112;
constexpr int OFF_BP = 2 * STAGE;          // S fp16 MN-major (rows = dk), 32 KB
constexpr int OFF_BU = OFF_BP + 32768;     // U fp16 MN-major (rows = tokens), 16 KB
constexpr int OFF_MISC = OFF_BU + 16384;
// misc: barriers [0, 128), 1 + w [128, 640), partial sums [640, 1664); + alignment slack
constexpr int SMEM = OFF_MISC + 1664 + 1024;
static_assert(SMEM <= 232448, "227 KB per block");
constexpr uint32_t kMaxPolls = 1u << 24;
}  // namespace chain

struct ChainMaps {
    CUtensorMap wn, qt, kt, aqk, up, z, out;   // `out` only for bf16 output
};

// tanh on the special-function unit (absolute error about 2^-11)
__device__ __forceinline__ float tanh_approx(float x) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
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

// The chain of head h of sequence n over chunks [c_lo, c_hi), by a CTA of 4 * DV
// threads.  With `ready` non-NULL (the fused prefill kernel) the workspace rows of
// chunk c are read only after ready[c] is set.
template <int DV, typename Tout>
__device__ __forceinline__ void chain_body(const ChainMaps &maps, const float *__restrict__ decay,
                                           const float *__restrict__ norm_w, const float *state_in,
                                           const int32_t *__restrict__ cu_seqlens, int n_seq, int n_tok,
                                           int H, int h, int n, int c_lo, int c_hi,
                                           Tout *__restrict__ out, float *state_out,
                                           const int *ready, bool own_tmem = true, uint32_t tmem_given = 0) {
    using namespace chain;
    // 4 * DV threads: warp w reads TMEM lane quadrant q = w % 4 and owns the
    // 32-column group cg = w / 4 of every row it touches.
    constexpr int NT = 4 * DV;
    constexpr int NCG = DV / 32;
    constexpr int HALF = NT / 2;                             // threads of one role
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = umma::align_smem<1024>(smem_raw);
    uint8_t *sBP = sm + OFF_BP, *sBU = sm + OFF_BU;
    uint64_t *full_a = reinterpret_cast<uint64_t *>(sm + OFF_MISC);   // [2]
    uint64_t *full_z = full_a + 2;                                     // [2]
    uint64_t *bar_p = full_a + 4, *bar_s = full_a + 5, *bar_y = full_a + 6;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 64);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 68);
    float *w1 = reinterpret_cast<float *>(sm + OFF_MISC + 128);      // 1 + norm_w  [DV]
    float *red = w1 + DV;                                             // [NCG][64] partial sums
    constexpr uint32_t TMEM_COLS = DV == 128 ? 512 : 256;   // P0, P1, dS
    constexpr uint32_t BYTES_A = 4 * 8192 + 2 * 8192 + 8192 + C * DV * 2;
    constexpr uint32_t BYTES_Z = C * DV * 2;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, cg = warp >> 2, col0 = 32 * cg;
    int s_begin, s_end;
    if (cu_seqlens) { s_begin = __ldg(cu_seqlens + n); s_end = __ldg(cu_seqlens + n + 1); }
    else { const int L = n_tok / n_seq; s_begin = n * L; s_end = s_begin + L; }
    // chunks [c_lo, c_end) of this sequence; the state enters from state_in (NULL:
    // zeros) and leaves to state_out (NULL: dropped); they may be the same buffer
    const int c_end = min((s_end - s_begin + C - 1) / C, c_hi);
    const int n_chunks = max(0, c_end - c_lo);   // chunks handled by this launch

    // the tensor memory: allocated here, or (a CTA that runs several chains in turn:
    // an allocation gives up the CTA's permit to allocate again) passed in
    if (own_tmem && warp == 0) umma::tmem_alloc(tslot, TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) umma::mbar_init(full_a + i, 1);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }
    for (int j = tid; j < DV; j += NT) w1[j] = 1.0f + __ldg(norm_w + j);
    // fp32 master state: this thread owns S[32 q + lane][col0 .. col0 + 32); fp16 copy in sBP
    const int srow = 32 * q + lane;
    const size_t sbase = ((size_t)n * H + h) * DK * DV;
    float S[32];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
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
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tbase = own_tmem ? *tslot : tmem_given;
    const uint32_t tD = tbase + 2 * DV;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    // output gain of this thread's 32 columns, halved: sigmoid(z) (1 + w) y =
    // (1 + tanh(z / 2)) * ((1 + w) / 2) * y
    float w1h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) w1h[j] = 0.5f * w1[col0 + j];

    auto stage = [&](int b) { return sm + b * STAGE; };
    auto issue_a = [&](int cc, int b) {   // cc: chunk index within this launch
        const int t0 = s_begin + (c_lo + cc) * C;
        uint8_t *st = stage(b);
        if (ready) wait_ready(ready + c_lo + cc, abort_flag);
        umma::mbar_expect_tx(full_a + b, BYTES_A);
        umma::tma_load_3d(st + ST_AP, &maps.wn, 0, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AP + 8192, &maps.qt, 0, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AP + 16384, &maps.wn, 64, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AP + 24576, &maps.qt, 64, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AS, &maps.kt, 0, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AS + 8192, &maps.kt, 64, h, t0, full_a + b);
        umma::tma_load_3d(st + ST_AQK, &maps.aqk, 0, h, t0, full_a + b);
#pragma unroll
        for (int x = 0; x < DV; x += 64) umma::tma_load_3d(st + ST_US + x * 128, &maps.up, x, h, t0, full_a + b);
    };
    auto issue_z = [&](int cc, int b) {
        umma::mbar_expect_tx(full_z + b, BYTES_Z);
#pragma unroll
        for (int x = 0; x < DV; x += 64)
            umma::tma_load_3d(stage(b) + ST_ZS + x * 128, &maps.z, x, h, s_begin + (c_lo + cc) * C, full_z + b);
    };
    // Tile producers: tid kTmaA (a U-warp lane, idle while the first MMA runs)
    // refills, at the start of chunk c, the stage of chunk c - 1 (drained before
    // the last block barrier) with the operand tiles of chunk c + 1; tid kTma (an
    // output-stage lane) issues the z tiles one chunk ahead and the TMA stores of
    // finished bf16 output tiles.
    constexpr int kTmaA = 32, kTma = 64;
    constexpr bool kTmaOut = sizeof(Tout) == 2;
    if (tid == kTma) {
        umma::prefetch_tensormap(&maps.wn);
        umma::prefetch_tensormap(&maps.qt);
        umma::prefetch_tensormap(&maps.kt);
        umma::prefetch_tensormap(&maps.aqk);
        umma::prefetch_tensormap(&maps.up);
        umma::prefetch_tensormap(&maps.z);
        if (kTmaOut) umma::prefetch_tensormap(&maps.out);
        for (int cc = 0; cc < 2 && cc < n_chunks; ++cc) issue_a(cc, cc);
        if (n_chunks > 0) issue_z(0, 0);
    }
    __syncthreads();   // the ready flags of chunks 0, 1 were acquired before any decay read
    // byte offset of the 8-column chunk `col` of row i in a 64-column-block swizzled tile
    auto tile_off = [](int i, int col) { return (col / 64) * 8192 + umma::sw128_offset(i, (col % 64) / 8); };
    // descriptor bases (start-address field advanced by offset >> 4 per K step)
    const uint64_t dBP = umma::sw128_desc(umma::smem_u32(sBP), 16384, 1024);
    const uint64_t dBU = umma::sw128_desc(umma::smem_u32(sBU), 8192, 1024);
    const uint32_t id_p = umma::idesc_f16(128, DV, false, true);
    const uint32_t id_y = umma::idesc_f16(128, DV, false, true);
    const uint32_t id_s = umma::idesc_f16(128, DV, true, true);

    for (int c = 0; c < n_chunks; ++c) {   // c: chunk index within this launch
        const int b = c & 1;
        const int t0 = s_begin + (c_lo + c) * C;
        const int len = min(C, s_end - t0);
        const uint32_t ph_stage = (uint32_t)(c >> 1) & 1u, ph = (uint32_t)c & 1u;
        uint8_t *st = stage(b);
        const uint32_t tP = tbase + b * DV;
        const float dec = __ldcg(decay + (size_t)t0 * H + h);
        if (tid == kTmaA && c >= 1 && c + 1 < n_chunks) issue_a(c + 1, b ^ 1);
        if (q < 2) {
            // ---- P = [-W; Qt] S  (M=128, N=DV, K=dk)
            if (tid == 0) {
                chain_wait(full_a + b, ph_stage, abort_flag);
                umma::tc_fence_after();
                const uint64_t dA = umma::sw128_desc(umma::smem_u32(st + ST_AP), 16, 1024);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    umma::mma_f16(tP, dA + (uint64_t)(((s / 4) * 16384 + (s % 4) * 32) >> 4),
                                  dBP + (uint64_t)((s * 2048) >> 4), id_p, s > 0);
                umma::mma_commit(bar_p);
            }
            // U' of this thread's row and columns, read while the MMA runs
            const int i = srow;
            chain_wait(full_a + b, ph_stage, abort_flag);
            uint4 upk[4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                upk[m] = *reinterpret_cast<const uint4 *>(st + ST_US + tile_off(i, col0 + 8 * m));
            if (i >= len) {
                // rows past the end of a ragged chunk belong to another sequence (or lie
                // past the tensor) and may not be written yet: dS = Kt^T U multiplies
                // them by U = 0, so make them zero rather than trust them to be finite
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *reinterpret_cast<uint4 *>(st + ST_AS + (cg >> 1) * 8192 + i * 128 + (cg & 1) * 64 + 16 * m) =
                        make_uint4(0, 0, 0, 0);
            }
            chain_wait(bar_p, ph, abort_flag);
            umma::tc_fence_after();
            // ---- U = U' + P[0:64] (zero past the sequence end) -> fp16 MN-major B operand
            float v[32];
            umma::tmem_ld32(tP + lane_off + col0, v);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int col = col0 + 8 * m;
                float up[8], u[8];
                unpack8h(upk[m], up);
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] = (i < len) ? v[8 * m + e] + up[e] : 0.f;
                umma::st_chunk(sBU + (col / 64) * 8192, i, (col % 64) / 8, pack8(u));
            }
            umma::fence_proxy_async_smem();
            umma::tc_fence_before();
            umma::named_bar_sync(1, HALF);
            // ---- dS = Kt^T U (on the state path, committed first);  P[64:128] += [*; Aqk] U
            if (tid == 0) {
                umma::tc_fence_after();
                const uint64_t dS = umma::sw128_desc(umma::smem_u32(st + ST_AS), 8192, 1024);
                const uint64_t dY = umma::sw128_desc(umma::smem_u32(st + ST_AS + 8192), 16, 1024);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    umma::mma_f16(tD, dS + (uint64_t)((s * 2048) >> 4), dBU + (uint64_t)((s * 2048) >> 4), id_s, s > 0);
                umma::mma_commit(bar_s);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    umma::mma_f16(tP, dY + (uint64_t)((s * 32) >> 4), dBU + (uint64_t)((s * 2048) >> 4), id_y, 1u);
                umma::mma_commit(bar_y);
            }
        }
        chain_wait(bar_s, ph, abort_flag);
        umma::tc_fence_after();
        // ---- S = e^{G_C} S + dS; fp16 copy for the next chunk
        {
            float v[32];
            umma::tmem_ld32(tD + lane_off + col0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = fmaf(dec, S[j], v[j]);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int col = col0 + 8 * m;
                umma::st_chunk(sBP + (col / 64) * 16384, srow, (col % 64) / 8, pack8(S + 8 * m));
            }
        }
        umma::fence_proxy_async_smem();
        if (q >= 2) {
            // Y of this chunk is complete (waited before the block barrier, so this
            // barrier's phases never run ahead of the waits); stage b is drained.
            chain_wait(bar_y, ph, abort_flag);
        }
        umma::tc_fence_before();
        __syncthreads();
        umma::tc_fence_after();
        // ---- output stage of this chunk on P[64:128] (quadrants 2, 3): overlaps chunk c + 1
        if (q >= 2) {
            const int i = srow - 64;
            float v[32];
            umma::tmem_ld32(tP + lane_off + col0, v);
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 32; ++j) s4[j & 3] = fmaf(v[j], v[j], s4[j & 3]);
            red[cg * 64 + i] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            chain_wait(full_z + b, ph_stage, abort_flag);
            umma::named_bar_sync(2, HALF);
            float tot = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < NCG; ++g2) tot += red[g2 * 64 + i];
            const float rr = rsqrtf(tot / DV + kNormEps);
            float rw[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) rw[j] = rr * w1h[j];
            // full chunks of a bf16 output leave through one TMA store of the z tile,
            // overwritten in place; ragged chunks store their valid rows directly
            const bool tile_store = kTmaOut && len == C;
            const size_t g = ((size_t)(t0 + i) * H + h) * DV;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int col = col0 + 8 * m;
                uint4 *zp = reinterpret_cast<uint4 *>(st + ST_ZS + tile_off(i, col));
                const uint4 zz = *zp;
                const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
                float o[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float t0z = tanh_approx(0.5f * bf16lo(zw[e])), t1z = tanh_approx(0.5f * bf16hi(zw[e]));
                    const float a0 = v[8 * m + 2 * e] * rw[8 * m + 2 * e];
                    const float a1 = v[8 * m + 2 * e + 1] * rw[8 * m + 2 * e + 1];
                    o[2 * e] = fmaf(a0, t0z, a0);
                    o[2 * e + 1] = fmaf(a1, t1z, a1);
                }
                if (tile_store) store8_out<bf16>(reinterpret_cast<bf16 *>(zp), o);
                else if (i < len) store8_out<Tout>(out + g + col, o);
            }
            if (tile_store) umma::fence_proxy_async_smem();
            umma::named_bar_sync(2, HALF);
            if (tid == kTma) {
                if (tile_store) {
#pragma unroll
                    for (int x = 0; x < DV; x += 64)
                        umma::tma_store_3d(&maps.out, x, h, t0, st + ST_ZS + x * 128);
                    umma::bulk_commit();
                }
                // the z tile of stage b ^ 1 is free once the store of chunk c - 1 has read it
                umma::bulk_wait_read<1>();
                if (c + 1 < n_chunks) issue_z(c + 1, b ^ 1);
            }
        }
    }
    if (tid == kTma) umma::bulk_wait_all();
    if (state_out && !*abort_flag) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = S[8 * m + e];
            store8(state_out + sbase + (size_t)srow * DV + col0 + 8 * m, x);
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0 && n_chunks > 0) {
        // let any tile copy still in flight land before the CTA exits (bounded)
        for (int b = 0; b < 2 && b < n_chunks; ++b) {
            const int last = ((n_chunks - 1 - b) / 2) * 2 + b;   // last chunk that used stage b
            umma::mbar_wait_bounded(full_a + b, (uint32_t)(last >> 1) & 1u, 1u << 16);
            umma::mbar_wait_bounded(full_z + b, (uint32_t)(last >> 1) & 1u, 1u << 16);
        }
    }
    if (own_tmem && warp == 0) umma::tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn

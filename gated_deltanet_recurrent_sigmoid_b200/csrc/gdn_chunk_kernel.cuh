// gdn_chunk_kernel.cuh -- chunked (prefill-style) sm_100a kernel of the
// Gated DeltaNet update on the 5th-generation tensor cores (tcgen05).
//
// It computes exactly the recurrence stated in include/gdn_decode.h (same
// gating, normalisation and output), but a chunk of C = 64 tokens at a time
// in the closed form of the delta rule over a chunk (the WY representation
// behind the pages' chunked GDN kernels: chunk_scaled_dot_kkt, solve_tril,
// recompute_w_u, CHUNK_SIZE 64).  Within a chunk, with gamma_j the
// cumulative sum of the log-decays g of tokens 0..j of the chunk, hats the
// normalised vectors and S0 the state before the chunk:
//     A[j][i] = beta_j e^(gamma_j - gamma_i) k^_j . k^_i    (i < j, else 0)
//     T       = (I + A)^-1                                  (forward substitution)
//     W = T diag(beta e^gamma) K^ ,   U = T diag(beta) V
//     Delta   = U - W S0                                    (the per-token deltas)
//     O[j]    = e^gamma_j S0^T q^_j + sum_{i<=j} e^(gamma_j - gamma_i) (q^_j . k^_i) Delta_i
//     S       = e^gamma_last S0 + sum_i e^(gamma_last - gamma_i) k^_i Delta_i^T
// (all exponents are <= 0).  Every matrix product runs on tcgen05 with fp32
// accumulators in tensor memory; raw bf16 q, k, v are exact MMA operands and
// the per-token scalars are applied outside; fp32 operands (T, W, Delta, P,
// the state) are split into a bf16 high part plus a bf16 low part, and the
// products hi*hi + hi*lo + lo*hi keep ~16 mantissa bits, so the state stays
// well within 1e-4 of the fp32 recurrence.
//
// One CTA (4 warps; thread t owns TMEM lane t) per (sequence, value head);
// the state lives in TMEM across the chunks of the sequence, in transposed
// form S^T[v][k] (lane v, column k).  Single-thread MMA issue, one mbarrier
// with bounded waits between the dependent products.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn_decode.h"
#include "gdn_decode_kernel.cuh"
#include "mbarrier_sm100.cuh"
#include "tc_sm100.cuh"

namespace gdn {
namespace chunk {

constexpr int K = 128;
constexpr int V = 128;
constexpr int C = 64;            // tokens per chunk
constexpr int THREADS = 128;     // thread t <-> TMEM lane t
constexpr uint32_t TMEM_COLS = 512;
// TMEM column map (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_S = 0;     // S^T [v][k]          128 columns
constexpr uint32_t COL_KQ = 128;  // [K;Q] K^T [r][i]     64
constexpr uint32_t COL_O1 = 192;  // S0^T Q^T [v][j]      64
constexpr uint32_t COL_WT = 256;  // W^T [k][j]           64
constexpr uint32_t COL_DT = 320;  // Delta^T [v][j]       64
constexpr uint32_t COL_O2 = 384;  // Delta^T P^T [v][j]   64

// Shared memory (bf16 operand tiles in the K-major core-matrix layout of
// tc_sm100.cuh; sizes in bytes).
struct Smem {
    alignas(1024) unsigned char kq[128 * 128 * 2];   // rows 0..63: raw k, 64..127: raw q   [r][k]
    alignas(1024) unsigned char kt[128 * 64 * 2];    // raw k transposed                    [k][i]
    alignas(1024) unsigned char vt[128 * 64 * 2];    // raw v transposed                    [v][i]
    alignas(1024) unsigned char tw[2][64 * 64 * 2];  // T diag(beta e^gamma rk), hi / lo    [j][i]
    alignas(1024) unsigned char tu[2][64 * 64 * 2];  // T diag(beta), hi / lo               [j][i]
    alignas(1024) unsigned char p[2][64 * 64 * 2];   // masked scaled q.k, hi / lo          [j][i]
    alignas(1024) unsigned char st[2][128 * 128 * 2];// S^T hi / lo                         [v][k]
    // W hi / lo [j][k] (64 x 128 each); later Delta^T hi / lo [v][i] (128 x 64
    // each); before both, the fp32 matrix A [64][64] for the solve.
    alignas(1024) unsigned char wd[2][128 * 64 * 2];
    float rk[C], rqs[C], gam[C], beta[C], g[C];
    unsigned long long mbar;
    uint32_t tmem_base;
    int failed;
};

__device__ __forceinline__ void split2(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

__device__ __forceinline__ void st_bf16(unsigned char *tile, uint32_t r, uint32_t c, uint32_t cols, __nv_bfloat16 x)
{
    *reinterpret_cast<__nv_bfloat16 *>(tile + tc::kmajor_offset(r, c, cols)) = x;
}

// Eight consecutive columns c0..c0+7 (c0 % 8 == 0) of row r: one 16-byte store.
__device__ __forceinline__ void st_row8(unsigned char *tile, uint32_t r, uint32_t c0, uint32_t cols, const float *x,
                                        bool lo_part)
{
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat16 h0, l0, h1, l1;
        split2(x[2 * e], h0, l0);
        split2(x[2 * e + 1], h1, l1);
        const __nv_bfloat16 a = lo_part ? l0 : h0, b = lo_part ? l1 : h1;
        w[e] = static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
    }
    *reinterpret_cast<uint4 *>(tile + tc::kmajor_offset(r, c0, cols)) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Issue a product over `slices` 16-column k-slices: D (+)= A * B^T.
__device__ __forceinline__ void mma_tiles(uint32_t d, const unsigned char *a, uint32_t a_cols, const unsigned char *b,
                                          uint32_t b_cols, uint32_t slices, uint32_t idesc, bool accumulate)
{
    for (uint32_t s = 0; s < slices; ++s)
        tc::mma_bf16(d, tc::kslice_desc(a, a_cols, s), tc::kslice_desc(b, b_cols, s), idesc,
                     (accumulate || s > 0) ? 1u : 0u);
}

template <bool L2NORM>
__global__ void __launch_bounds__(THREADS, 1) gdn_chunk_kernel(const __grid_constant__ DecodeParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int i = blockIdx.x / p.HV;
    const int hv = blockIdx.x - i * p.HV;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);

    // ---- token range and slot (uniform over the CTA) -----------------
    int64_t bos;
    int len;
    if (p.cu_seqlens) {
        const int b0 = __ldg(p.cu_seqlens + i);
        const int e0 = __ldg(p.cu_seqlens + i + 1);
        if (b0 < 0 || e0 < b0 || e0 > p.T_tot) {
            if (tid == 0 && hv == 0)
                report(p.status, GDN_DEV_BAD_SEQLENS);
            return;
        }
        bos = b0;
        len = e0 - b0;
    } else {
        bos = static_cast<int64_t>(i) * p.T_fixed;
        len = p.T_fixed;
    }
    const int slot = __ldg(p.indices + i);
    if (slot < -1 || slot >= p.num_slots) {
        if (tid == 0 && hv == 0)
            report(p.status, GDN_DEV_BAD_SLOT);
        return;
    }
    if (slot < 0) {
        for (int t = 0; t < len; ++t)
            out[(bos + t) * p.o_tok + hv * p.o_head + tid] = __float2bfloat16_rn(0.f);
        return;
    }
    if (len == 0)
        return;

    const int h = hv / p.G;
    const float neg_A = -expf(__ldg(p.A_log + hv * p.A_stride));
    const float dt_b = __ldg(p.dt_bias + hv * p.dt_stride);
    float *const s_gmem = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head;

    // ---- set-up: mbarrier, TMEM, state into TMEM and into the S^T tiles --
    if (tid == 0) {
        sync::mbar_init(&sm.mbar, 1);
        sm.failed = 0;
        sync::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, warp * 32, 0);   // + column

    // thread t = v: column v of S (rows k) -> lane v of S^T
    for (int k0 = 0; k0 < K; k0 += 16) {
        float x[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
            x[e] = __ldcs(s_gmem + (k0 + e) * V + tid);
        tc::tmem_st16(my_lane + COL_S + k0, x);
        st_row8(sm.st[0], tid, k0, K, x, false);
        st_row8(sm.st[0], tid, k0 + 8, K, x + 8, false);
        st_row8(sm.st[1], tid, k0, K, x, true);
        st_row8(sm.st[1], tid, k0 + 8, K, x + 8, true);
    }
    tc::tmem_wait_st();

    uint32_t phase = 0;
    bool ok = true;
    // Wait for the MMAs committed last; uniform verdict over the CTA.
    auto wait_mma = [&]() {
        bool w = ok && sync::mbar_wait(&sm.mbar, phase, &sm.failed);
        phase ^= 1u;
        if (!w && ok) {
            sm.failed = 1;
            report(p.status, GDN_DEV_TIMEOUT);
        }
        ok = __syncthreads_and(w) != 0;
        tc::fence_after_sync();
    };
    auto publish_smem = [&]() {     // operand tiles written by threads -> visible to the tensor cores
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };

    const uint32_t ID_M128_N64 = tc::idesc_bf16_f32(128, 64);
    const uint32_t ID_M128_N64_NEG = tc::idesc_bf16_f32(128, 64, true);
    const uint32_t ID_M128_N128 = tc::idesc_bf16_f32(128, 128);

    for (int c0 = 0; c0 < len && ok; c0 += C) {
        const int n = len - c0 < C ? len - c0 : C;
        const bool last = c0 + C >= len;

        // ---- step 1: raw q, k, v of the chunk into the operand tiles ----
        {
            const int j = tid >> 1;             // token of the chunk
            const int half = tid & 1;           // columns [64 half, 64 half + 64)
            const bool live = j < n;
            const int64_t tok = bos + c0 + j;
            float kk = 0.f, qq = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int col = 64 * half + 8 * m;
                uint4 kr = make_uint4(0u, 0u, 0u, 0u), qr = kr, vr = kr;
                if (live) {
                    kr = __ldg(reinterpret_cast<const uint4 *>(k + tok * p.k_tok + h * p.k_head + col));
                    qr = __ldg(reinterpret_cast<const uint4 *>(q + tok * p.q_tok + h * p.q_head + col));
                    vr = __ldg(reinterpret_cast<const uint4 *>(v + tok * p.v_tok + hv * p.v_head + col));
                }
                *reinterpret_cast<uint4 *>(sm.kq + tc::kmajor_offset(j, col, K)) = kr;
                *reinterpret_cast<uint4 *>(sm.kq + tc::kmajor_offset(64 + j, col, K)) = qr;
                float kf[8], qf[8], vf[8];
                unpack8(kr, kf);
                unpack8(qr, qf);
                unpack8(vr, vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk = fmaf(kf[e], kf[e], kk);
                    qq = fmaf(qf[e], qf[e], qq);
                    st_bf16(sm.kt, col + e, j, C, __float2bfloat16_rn(kf[e]));
                    st_bf16(sm.vt, col + e, j, C, __float2bfloat16_rn(vf[e]));
                }
            }
            kk += __shfl_xor_sync(0xffffffffu, kk, 1);
            qq += __shfl_xor_sync(0xffffffffu, qq, 1);
            if (half == 0) {
                float rk = 0.f, rq = 0.f, g = 0.f, be = 0.f;
                if (live) {
                    rk = L2NORM ? rsqrtf(kk + 1e-6f) : 1.f;
                    rq = (L2NORM ? rsqrtf(qq + 1e-6f) : 1.f) * p.scale;
                    const float a_t = gate_value(gate_raw(p.a, tok * p.a_tok + hv * p.a_head, p.a_f32), p.a_f32);
                    const float b_t = gate_value(gate_raw(p.b, tok * p.b_tok + hv * p.b_head, p.b_f32), p.b_f32);
                    const float x = a_t + dt_b;
                    g = neg_A * (x > 20.f ? x : log1pf(expf(x)));
                    be = 1.f / (1.f + expf(-b_t));
                }
                sm.rk[j] = rk;
                sm.rqs[j] = rq;
                sm.g[j] = g;
                sm.beta[j] = be;
            }
        }
        __syncthreads();
        if (tid < 32) {     // inclusive prefix sum of the log-decays (warp scan over 64 values)
            float a0 = sm.g[tid], a1 = sm.g[32 + tid];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, a0, off);
                const float y1 = __shfl_up_sync(0xffffffffu, a1, off);
                if (tid >= off) {
                    a0 += y0;
                    a1 += y1;
                }
            }
            const float total0 = __shfl_sync(0xffffffffu, a0, 31);
            sm.gam[tid] = a0;
            sm.gam[32 + tid] = a1 + total0;
        }
        publish_smem();

        // ---- step 2: [K;Q] K^T and S0^T Q^T --------------------------------
        if (tid == 0) {
            mma_tiles(tmem + COL_KQ, sm.kq, K, sm.kq, K, K / 16, ID_M128_N64, false);
            const unsigned char *qtile = sm.kq + tc::kmajor_offset(64, 0, K);
            mma_tiles(tmem + COL_O1, sm.st[0], K, qtile, K, K / 16, ID_M128_N64, false);
            mma_tiles(tmem + COL_O1, sm.st[1], K, qtile, K, K / 16, ID_M128_N64, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 3: A (rows 0..63) and P (rows 64..127) --------------------
        float *Amat = reinterpret_cast<float *>(sm.wd[0]);     // [64][64] fp32
        {
            float row[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16)
                tc::tmem_ld16(my_lane + COL_KQ + c, row + c);
            tc::tmem_wait_ld();
            if (tid < 64) {
                const int j = tid;
                const float fj = sm.beta[j] * sm.rk[j];
                const float gj = sm.gam[j];
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    Amat[j * 64 + c] = (c < j) ? fj * sm.rk[c] * expf(gj - sm.gam[c]) * row[c] : 0.f;
            } else {
                const int j = tid - 64;
                const float fj = sm.rqs[j];
                const float gj = sm.gam[j];
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    row[c] = (c <= j) ? fj * sm.rk[c] * expf(gj - sm.gam[c]) * row[c] : 0.f;
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    st_row8(sm.p[0], j, c, C, row + c, false);
                    st_row8(sm.p[1], j, c, C, row + c, true);
                }
            }
        }
        __syncthreads();

        // ---- step 4: T = (I + A)^-1 by forward substitution, column per thread
        if (tid < 64) {
            const int col = tid;
            float tcol[64];
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                float acc = (r == col) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m)
                    acc = fmaf(-Amat[r * 64 + m], tcol[m], acc);
                tcol[r] = (r < col) ? 0.f : acc;
            }
            const float fw = sm.beta[col] * expf(sm.gam[col]) * sm.rk[col];
            const float fu = sm.beta[col];
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                __nv_bfloat16 hi, lo;
                split2(tcol[r] * fw, hi, lo);
                st_bf16(sm.tw[0], r, col, C, hi);
                st_bf16(sm.tw[1], r, col, C, lo);
                split2(tcol[r] * fu, hi, lo);
                st_bf16(sm.tu[0], r, col, C, hi);
                st_bf16(sm.tu[1], r, col, C, lo);
            }
        }
        publish_smem();

        // ---- step 5: W^T = K^T T_w^T and U^T = V^T T_u^T ---------------------
        if (tid == 0) {
            mma_tiles(tmem + COL_WT, sm.kt, C, sm.tw[0], C, C / 16, ID_M128_N64, false);
            mma_tiles(tmem + COL_WT, sm.kt, C, sm.tw[1], C, C / 16, ID_M128_N64, true);
            mma_tiles(tmem + COL_DT, sm.vt, C, sm.tu[0], C, C / 16, ID_M128_N64, false);
            mma_tiles(tmem + COL_DT, sm.vt, C, sm.tu[1], C, C / 16, ID_M128_N64, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 6: W (thread = k) into the W hi / lo tiles [j][k] -----------
        {
            float wcol[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16)
                tc::tmem_ld16(my_lane + COL_WT + c, wcol + c);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                __nv_bfloat16 hi, lo;
                split2(wcol[j], hi, lo);
                st_bf16(sm.wd[0], j, tid, K, hi);
                st_bf16(sm.wd[1], j, tid, K, lo);
            }
        }
        publish_smem();

        // ---- step 7: Delta^T = U^T - S0^T W^T (3 split products, A negated) ---
        if (tid == 0) {
            mma_tiles(tmem + COL_DT, sm.st[0], K, sm.wd[0], K, K / 16, ID_M128_N64_NEG, true);
            mma_tiles(tmem + COL_DT, sm.st[0], K, sm.wd[1], K, K / 16, ID_M128_N64_NEG, true);
            mma_tiles(tmem + COL_DT, sm.st[1], K, sm.wd[0], K, K / 16, ID_M128_N64_NEG, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 8: Delta^T (thread = v) into the hi / lo tiles [v][i] -------
        {
            float drow[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16)
                tc::tmem_ld16(my_lane + COL_DT + c, drow + c);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 64; c += 8) {
                st_row8(sm.wd[0], tid, c, C, drow + c, false);
                st_row8(sm.wd[1], tid, c, C, drow + c, true);
            }
        }
        publish_smem();

        // ---- step 9: O2^T = Delta^T P^T (3 split products) --------------------
        if (tid == 0) {
            mma_tiles(tmem + COL_O2, sm.wd[0], C, sm.p[0], C, C / 16, ID_M128_N64, false);
            mma_tiles(tmem + COL_O2, sm.wd[0], C, sm.p[1], C, C / 16, ID_M128_N64, true);
            mma_tiles(tmem + COL_O2, sm.wd[1], C, sm.p[0], C, C / 16, ID_M128_N64, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 10: outputs; Delta' for the state; decay the state ----------
        {
            const float gl = sm.gam[n - 1];
#pragma unroll
            for (int cb = 0; cb < 64; cb += 16) {
                float o1[16], o2[16], d[16];
                tc::tmem_ld16(my_lane + COL_O1 + cb, o1);
                tc::tmem_ld16(my_lane + COL_O2 + cb, o2);
                tc::tmem_ld16(my_lane + COL_DT + cb, d);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j = cb + e;
                    if (j < n) {
                        const float f = expf(sm.gam[j]) * sm.rqs[j];
                        out[(bos + c0 + j) * p.o_tok + hv * p.o_head + tid] =
                            __float2bfloat16_rn(fmaf(f, o1[e], o2[e]));
                    }
                    d[e] *= expf(gl - sm.gam[j]) * sm.rk[j];     // Delta' = Delta e^(gamma_last - gamma_i) rk_i
                }
                st_row8(sm.wd[0], tid, cb, C, d, false);
                st_row8(sm.wd[0], tid, cb + 8, C, d + 8, false);
                st_row8(sm.wd[1], tid, cb, C, d, true);
                st_row8(sm.wd[1], tid, cb + 8, C, d + 8, true);
            }
            const float decay = expf(gl);
            for (int k0 = 0; k0 < K; k0 += 16) {
                float x[16];
                tc::tmem_ld16(my_lane + COL_S + k0, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] *= decay;
                tc::tmem_st16(my_lane + COL_S + k0, x);
            }
            tc::tmem_wait_st();
        }
        publish_smem();

        // ---- step 11: S^T += Delta'^T K (2 split products, K exact) -----------
        if (tid == 0) {
            mma_tiles(tmem + COL_S, sm.wd[0], C, sm.kt, C, C / 16, ID_M128_N128, true);
            mma_tiles(tmem + COL_S, sm.wd[1], C, sm.kt, C, C / 16, ID_M128_N128, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 12: the next chunk's S^T tiles, or the final write-back -----
        for (int k0 = 0; k0 < K; k0 += 16) {
            float x[16];
            tc::tmem_ld16(my_lane + COL_S + k0, x);
            tc::tmem_wait_ld();
            if (!last) {
                st_row8(sm.st[0], tid, k0, K, x, false);
                st_row8(sm.st[0], tid, k0 + 8, K, x + 8, false);
                st_row8(sm.st[1], tid, k0, K, x, true);
                st_row8(sm.st[1], tid, k0 + 8, K, x + 8, true);
            } else if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    __stcs(s_gmem + (k0 + e) * V + tid, x[e]);
            }
        }
        publish_smem();
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace chunk
}  // namespace gdn

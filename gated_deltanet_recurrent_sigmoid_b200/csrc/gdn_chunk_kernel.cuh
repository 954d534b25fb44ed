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
    // per-token factors of the chunk (computed once after the scan)
    float fa[C];   // beta_j rk_j          (row factor of A)
    float fw[C];   // beta_i e^gamma_i rk_i (column factor of T for W)
    float fo[C];   // e^gamma_j rqs_j      (factor of S0^T q_j in the output)
    float fd[C];   // e^(gamma_last - gamma_i) rk_i (factor of Delta_i in the state update)
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

// fp32 64 x 64 matrices in shared memory (A and T of the solve): row-major
// with the column XOR-swizzled by the row, so that both a row and a column
// are spread over all 32 banks.
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + (c ^ (r & 31)); }

// Transpose an 8 x 8 block of bf16 held as 8 rows of 16 bytes: out[c] holds
// column c of the input (8 rows, as bf16 pairs).
__device__ __forceinline__ void transpose8x8(const uint4 (&in)[8], uint4 (&out)[8])
{
    uint32_t pw[8][4];
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) {
        const uint32_t a[4] = {in[2 * s2].x, in[2 * s2].y, in[2 * s2].z, in[2 * s2].w};
        const uint32_t b[4] = {in[2 * s2 + 1].x, in[2 * s2 + 1].y, in[2 * s2 + 1].z, in[2 * s2 + 1].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            pw[2 * s2][w] = __byte_perm(a[w], b[w], 0x5410);       // column 2w of rows 2s2, 2s2+1
            pw[2 * s2 + 1][w] = __byte_perm(a[w], b[w], 0x7632);   // column 2w+1
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
        out[c] = make_uint4(pw[c & 1][c >> 1], pw[2 + (c & 1)][c >> 1], pw[4 + (c & 1)][c >> 1],
                            pw[6 + (c & 1)][c >> 1]);
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
        // thread (tg, kg): tokens 8 tg .. 8 tg + 7, columns 8 kg .. 8 kg + 7
        {
            const int tg = tid >> 4, kg = tid & 15, col = 8 * kg;
            uint4 kr[8], qr[8], vr[8];
            float kk[8], qq[8];
            // all 24 loads in flight before any is used
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int j = 8 * tg + r;
                const int64_t tok = bos + c0 + (j < n ? j : 0);
                kr[r] = __ldg(reinterpret_cast<const uint4 *>(k + tok * p.k_tok + h * p.k_head + col));
                qr[r] = __ldg(reinterpret_cast<const uint4 *>(q + tok * p.q_tok + h * p.q_head + col));
                vr[r] = __ldg(reinterpret_cast<const uint4 *>(v + tok * p.v_tok + hv * p.v_head + col));
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int j = 8 * tg + r;
                if (j >= n)
                    kr[r] = qr[r] = vr[r] = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(sm.kq + tc::kmajor_offset(j, col, K)) = kr[r];
                *reinterpret_cast<uint4 *>(sm.kq + tc::kmajor_offset(64 + j, col, K)) = qr[r];
                float kf[8], qf[8];
                unpack8(kr[r], kf);
                unpack8(qr[r], qf);
                kk[r] = 0.f;
                qq[r] = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk[r] = fmaf(kf[e], kf[e], kk[r]);
                    qq[r] = fmaf(qf[e], qf[e], qq[r]);
                }
            }
            uint4 tr[8];
            transpose8x8(kr, tr);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                *reinterpret_cast<uint4 *>(sm.kt + tc::kmajor_offset(col + e, 8 * tg, C)) = tr[e];
            transpose8x8(vr, tr);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                *reinterpret_cast<uint4 *>(sm.vt + tc::kmajor_offset(col + e, 8 * tg, C)) = tr[e];
            // sum the 16 column groups of each token (lanes differing in bits 0..3)
#pragma unroll
            for (int off = 1; off < 16; off <<= 1)
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    kk[r] += __shfl_xor_sync(0xffffffffu, kk[r], off);
                    qq[r] += __shfl_xor_sync(0xffffffffu, qq[r], off);
                }
            if (kg < 8) {
                const int j = 8 * tg + kg;
                const int64_t tok = bos + c0 + j;
                float rk = 0.f, rq = 0.f, g = 0.f, be = 0.f;
                float kk_j = kk[0], qq_j = qq[0];
#pragma unroll
                for (int r = 1; r < 8; ++r)
                    if (kg == r) {
                        kk_j = kk[r];
                        qq_j = qq[r];
                    }
                if (j < n) {
                    rk = L2NORM ? rsqrtf(kk_j + 1e-6f) : 1.f;
                    rq = (L2NORM ? rsqrtf(qq_j + 1e-6f) : 1.f) * p.scale;
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
        __syncthreads();
        if (tid < C) {      // per-token factors, once
            const float gl = sm.gam[n - 1], gj = sm.gam[tid];
            sm.fa[tid] = sm.beta[tid] * sm.rk[tid];
            sm.fw[tid] = sm.beta[tid] * expf(gj) * sm.rk[tid];
            sm.fo[tid] = expf(gj) * sm.rqs[tid];
            sm.fd[tid] = expf(gl - gj) * sm.rk[tid];
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
        float *Amat = reinterpret_cast<float *>(sm.wd[0]);     // [64][64] fp32, swizzled
        float *Tmat = reinterpret_cast<float *>(sm.wd[1]);     // [64][64] fp32, swizzled
        {
            float row[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16)
                tc::tmem_ld16(my_lane + COL_KQ + c, row + c);
            tc::tmem_wait_ld();
            if (tid < 64) {
                const int j = tid;
                const float fj = sm.fa[j];
                const float gj = sm.gam[j];
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    Amat[sw64(j, c)] = (c < j) ? fj * sm.rk[c] * expf(gj - sm.gam[c]) * row[c] : 0.f;
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

        // ---- step 4: T = (I + A)^-1, blocked by 16 x 16 ---------------------
        // T_II = (I + A_II)^-1 (forward substitution, one column per thread);
        // then T_IJ = -T_II sum_{M=J}^{I-1} A_IM T_MJ, one block diagonal at a
        // time (each level is two small products spread over all threads).
        float *X = reinterpret_cast<float *>(sm.tw[0]);        // scratch [3][16][16]
        if (tid < 64) {
            const int I = tid >> 4, cc = tid & 15, c = 16 * I + cc;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m)
                    acc = fmaf(-Amat[sw64(16 * I + r, 16 * I + m)], x[m], acc);
                x[r] = (r < cc) ? 0.f : acc;
                Tmat[sw64(16 * I + r, c)] = x[r];
            }
        } else {
            // the strictly upper blocks of T are zero
            for (int e = tid - 64; e < 6 * 256; e += 64) {
                const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                const int J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                Tmat[sw64(16 * I + r, 16 * J + cc)] = 0.f;
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {           // block diagonal I - J = d
            const int nb = 4 - d;               // blocks (J + d, J), J = 0 .. nb - 1
            // X_J = sum_{M=J}^{J+d-1} A_{J+d,M} T_{M,J}
            for (int e = tid; e < nb * 256; e += THREADS) {
                const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15, I = J + d;
                float acc = 0.f;
                for (int M = J; M < I; ++M)
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc = fmaf(Amat[sw64(16 * I + r, 16 * M + m)], Tmat[sw64(16 * M + m, 16 * J + cc)], acc);
                X[e] = acc;
            }
            __syncthreads();
            // T_{I,J} = -T_{I,I} X_J
            for (int e = tid; e < nb * 256; e += THREADS) {
                const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15, I = J + d;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc = fmaf(Tmat[sw64(16 * I + r, 16 * I + m)], X[(J << 8) + (m << 4) + cc], acc);
                Tmat[sw64(16 * I + r, 16 * J + cc)] = -acc;
            }
            __syncthreads();
        }
        // T' = T diag(fw), T'' = T diag(beta): thread = (row, half of the columns)
        {
            const int r = tid >> 1, cbase = 32 * (tid & 1);
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
                float tw8[8], tu8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int col = cbase + c + e;
                    const float t = Tmat[sw64(r, col)];
                    tw8[e] = t * sm.fw[col];
                    tu8[e] = t * sm.beta[col];
                }
                st_row8(sm.tw[0], r, cbase + c, C, tw8, false);
                st_row8(sm.tw[1], r, cbase + c, C, tw8, true);
                st_row8(sm.tu[0], r, cbase + c, C, tu8, false);
                st_row8(sm.tu[1], r, cbase + c, C, tu8, true);
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

        // ---- step 8: Delta^T (thread = v) into the hi / lo tiles [v][i] of wd;
        // Delta'^T = Delta^T diag(e^(gamma_last - gamma_i) rk_i) into the tw / tu
        // area (free since W and U are done); the state in TMEM decayed ------
        unsigned char *dp_hi = sm.tw[0];     // 128 x 64 bf16 (tw[0..1] contiguous)
        unsigned char *dp_lo = sm.tu[0];     // 128 x 64 bf16 (tu[0..1] contiguous)
        {
#pragma unroll
            for (int cb = 0; cb < 64; cb += 16) {
                float d[16];
                tc::tmem_ld16(my_lane + COL_DT + cb, d);
                tc::tmem_wait_ld();
                st_row8(sm.wd[0], tid, cb, C, d, false);
                st_row8(sm.wd[0], tid, cb + 8, C, d + 8, false);
                st_row8(sm.wd[1], tid, cb, C, d, true);
                st_row8(sm.wd[1], tid, cb + 8, C, d + 8, true);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    d[e] *= sm.fd[cb + e];
                st_row8(dp_hi, tid, cb, C, d, false);
                st_row8(dp_hi, tid, cb + 8, C, d + 8, false);
                st_row8(dp_lo, tid, cb, C, d, true);
                st_row8(dp_lo, tid, cb + 8, C, d + 8, true);
            }
            const float decay = expf(sm.gam[n - 1]);
#pragma unroll
            for (int k0 = 0; k0 < K; k0 += 64) {
                float x[64];
#pragma unroll
                for (int e = 0; e < 64; e += 16)
                    tc::tmem_ld16(my_lane + COL_S + k0 + e, x + e);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    x[e] *= decay;
#pragma unroll
                for (int e = 0; e < 64; e += 16)
                    tc::tmem_st16(my_lane + COL_S + k0 + e, x + e);
            }
            tc::tmem_wait_st();
        }
        publish_smem();

        // ---- step 9: O2^T = Delta^T P^T (3 split products) and
        //      S^T += Delta'^T K (2 split products, K exact), one batch ------
        if (tid == 0) {
            mma_tiles(tmem + COL_O2, sm.wd[0], C, sm.p[0], C, C / 16, ID_M128_N64, false);
            mma_tiles(tmem + COL_O2, sm.wd[0], C, sm.p[1], C, C / 16, ID_M128_N64, true);
            mma_tiles(tmem + COL_O2, sm.wd[1], C, sm.p[0], C, C / 16, ID_M128_N64, true);
            mma_tiles(tmem + COL_S, dp_hi, C, sm.kt, C, C / 16, ID_M128_N128, true);
            mma_tiles(tmem + COL_S, dp_lo, C, sm.kt, C, C / 16, ID_M128_N128, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
        if (!ok)
            break;

        // ---- step 10: outputs o_j = fo_j (S0^T q_j) + (Delta^T P^T)_j ----------
#pragma unroll
        for (int cb = 0; cb < 64; cb += 16) {
            float o1[16], o2[16];
            tc::tmem_ld16(my_lane + COL_O1 + cb, o1);
            tc::tmem_ld16(my_lane + COL_O2 + cb, o2);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = cb + e;
                if (j < n)
                    out[(bos + c0 + j) * p.o_tok + hv * p.o_head + tid] =
                        __float2bfloat16_rn(fmaf(sm.fo[j], o1[e], o2[e]));
            }
        }

        // ---- step 11: the next chunk's S^T tiles, or the final write-back -----
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

    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace chunk
}  // namespace gdn

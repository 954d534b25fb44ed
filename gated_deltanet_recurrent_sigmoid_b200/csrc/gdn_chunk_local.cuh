// gdn_chunk_local.cuh -- the chunked Gated DeltaNet update in ONE sm_100a
// kernel with every product of a chunk kept on chip (GDN_SCHEDULE_CHUNKED):
// one CTA per (sequence, value head), chunks of 64 tokens aligned to the
// sequence, no workspace.
//
// The closed form of the delta rule over a chunk (the pages' chunked GDN
// prefill, "sglang PR #21411 summary", 实现拆解: chunk_scaled_dot_kkt +
// solve_tril, CHUNK_SIZE 64; gdn_chunk_split.cuh holds its WY form), with
// the state-dependent part arranged so that the state enters one product
// early instead of through W = T diag(beta e^gamma rk) K.  With S0 the state before the chunk,
// gamma_t the running sum of g from the chunk start, hats the normalised
// vectors:
//     A[t][i] = beta_t e^(gamma_t - gamma_i) k^_t . k^_i   (i < t),  T = (I + A)^-1
//     R_t     = beta_t (v_t - e^gamma_t S0^T k^_t)
//     Delta   = T R                          (= U - W S0 of the WY form)
//     o_j     = e^gamma_j rqs_j S0^T q_j + sum_{i <= j} P[j][i] Delta_i
//     S'      = e^gamma_last S0 + sum_i fd_i k_i Delta_i^T
// (unrolling the per-token rule over the chunk: delta_t = beta_t (v_t -
// S_dec^T k^_t) with S_dec the decayed state before token t, which is
// e^gamma_t S0 plus the earlier deltas' contributions -- moving those to the
// left gives (I + A) Delta = R).
//
// Per chunk, with the fp32 state S~^T (S = cs S~) in tensor memory across
// chunks:
//   rows      k, q rows -> one K-major [K;Q] tile (128 x 128 bf16); norms,
//             gates, gamma (threads 0..63)
//   product D S~^T [K;Q]^T -> (K S~)^T and (Q S~)^T in TMEM (S~ as bf16
//             hi / lo tiles, [K;Q] exact)
//   R         R~^T = R^T / cs' from (K S~)^T and the v rows -> hi / lo tiles
//   product G [K;Q] K^T -> K K^T (lanes 0..63, symmetric) and Q K^T (lanes
//             64..127): A by columns, P by rows (hi / lo tiles)
//   solve     T = (I + A)^-1 (recursive doubling, shared with the split
//             schedule's block kernel); T as hi / lo row tiles
//   product X Delta~^T = R~^T T^T (hi / lo pairs), while K' = diag(fd) K is
//             built as hi / lo row tiles (read MN-major below)
//   product Y [S~^T | O2] += Delta~^T [K' | P^T]
//   out       o_j = fo_j cs (Q S~)_j + cs' O2_j; the next chunk's S~ tiles, or
//             the final write-back
// The tiles live in six 16 KB pieces of shared memory whose lifetimes are
// staggered (see Smem), so two CTAs share an SM (~101 KB and 256 TMEM
// columns each) and one CTA's products and loads overlap the other's
// CUDA-core phases.
#pragma once

#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn_chunk_common.cuh"
#include "gdn_chunk_split.cuh"
#include "gdn_decode.h"
#include "gdn_decode_kernel.cuh"
#include "mbarrier_sm100.cuh"
#include "tc_sm100.cuh"

namespace gdn {
namespace local {

using chunk::mma_tiles;
using chunk::st_row8;
using split::ex2_approx;
using split::mma_tiles_bmn;
using split::solve_unit_lower64;

constexpr int K = 128;
constexpr int V = 128;
constexpr int C = 64;                 // tokens per chunk
constexpr int THREADS = 256;          // two threads per TMEM lane
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_S = 0;         // S~^T [v][k]                                      128 columns
constexpr uint32_t COL_X = 128;       // (K S~)^T [v][i]; then [K;Q] K^T [r][i]; then
                                      // Delta~^T [v][i]; then O2^T [v][j]                  64
constexpr uint32_t COL_QS = 192;      // (Q S~)^T [v][j]                                   64
constexpr uint32_t PIECE = 16384;

// Shared memory: six 16 KB pieces, s0..s3 (region s) and k0, k1 (region kq).
//   raw fp32 state [k][v]   s0..s3                 (first chunk, before the tiles)
//   S~^T hi / lo [v][k]     s0 s1 / s2 s3          until product D is done
//   [K;Q] rows [r][k]       k0 (k rows) k1 (q rows) until product G is done
//   R~^T hi / lo [v][i]     s0 / s1                until product X is done
//   P hi | lo [j][i]        k0 (8 KB each)         until product Y is done
//   A by columns (fp32)     k1                     until the solve is done
//   T by columns (fp32)     s2                     until the T tiles are built
//   T hi | lo [i][i']       s3 (8 KB each)         until product X is done
//   K' hi [i][k]            k1                     until product Y is done
//   K' lo [i][k]            s2                     until product Y is done
//   Delta~^T hi / lo [v][i] s0 / s1                until product Y is done
struct Smem {
    alignas(1024) unsigned char s[4 * PIECE];
    alignas(1024) unsigned char kq[2 * PIECE];
    float kk[4][C], qq[4][C];       // partial |k_j|^2, |q_j|^2 over four column quarters
    float rk[C], rqs[C], g[C], beta[C], gam[C];
    float fo[C], fd[C], fr[C];
    float ua[C], uq[C], wc[C];      // base-2 exponents of the A and P factors
    unsigned long long bar_x, bar_m; // the state's bulk copy; the products
    uint32_t tmem_base;
    int failed;
};

static_assert(offsetof(Smem, ua) % 16 == 0 && offsetof(Smem, wc) % 16 == 0, "ua and wc are read as 16-byte vectors");

template <bool L2NORM>
__global__ void __launch_bounds__(THREADS, 2) gdn_chunk_local_kernel(const __grid_constant__ DecodeParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    // thread (v, part): TMEM lane v (state column v), half `part` of the
    // columns of every per-lane phase
    const int v = tid & 127, part = tid >> 7;
    const int i = blockIdx.x / p.HV;
    const int hv = blockIdx.x - i * p.HV;
    const int h = hv / p.G;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const unsigned short *vg = static_cast<const unsigned short *>(p.v);

    // ---- token range and slot (uniform over the CTA) -----------------------
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
        for (int t = part; t < len; t += 2)
            out[(bos + t) * p.o_tok + hv * p.o_head + v] = __float2bfloat16_rn(0.f);
        return;
    }
    if (len == 0)
        return;
    const int64_t eos = bos + len;
    float *const s_gmem = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head;

    unsigned char *const s0 = sm.s, *const s1 = sm.s + PIECE, *const s2 = sm.s + 2 * PIECE, *const s3 = sm.s + 3 * PIECE;
    unsigned char *const k0 = sm.kq, *const k1 = sm.kq + PIECE;

    if (tid == 0) {
        sync::mbar_init(&sm.bar_x, 1);
        sync::mbar_init(&sm.bar_m, 1);
        sm.failed = 0;
        sync::fence_barrier_init();
        // the state S [k][v] (64 KB, contiguous) in one bulk copy
        sync::mbar_arrive_expect_state_tx(&sm.bar_x, K * V * 4);
        sync::bulk_load(sm.s, s_gmem, K * V * 4, &sm.bar_x);
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, (warp & 3) * 32, 0);

    uint32_t ph_x = 0, ph_m = 0;
    bool ok = true, pend_x = true;
    // bounded wait on one of the barriers; uniform verdict over the CTA
    auto wait_bar = [&](unsigned long long *bar, uint32_t &ph) {
        bool w = ok && sync::mbar_wait(bar, ph, &sm.failed);
        ph ^= 1u;
        if (!w && ok) {
            sm.failed = 1;
            report(p.status, GDN_DEV_TIMEOUT);
        }
        ok = __syncthreads_and(w) != 0;
        tc::fence_after_sync();
    };
    // generic-proxy shared-memory writes (and finished TMEM accesses) -> the
    // tensor cores; a barrier
    auto publish_smem = [&]() {
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    const uint32_t ID_N128 = tc::idesc_bf16_f32(128, 128);
    const uint32_t ID_N64 = tc::idesc_bf16_f32(128, C);
    const uint32_t ID_N128_BMN = tc::idesc_bf16_f32(128, 128, false, false, true);
    const int ib = 32 * part;          // this thread's token columns (of 64)

    float cs = 1.f;
    for (int64_t t0 = bos; t0 < eos && ok; t0 += C) {
        const int n = eos - t0 < C ? static_cast<int>(eos - t0) : C;
        const bool more = t0 + n < eos;

        // ---- rows: k and q rows of the chunk into the [K;Q] tile (zeros past
        // the end), their squared norms by column quarter, the gates; the v
        // rows into L2.  Thread (j, qtr): row j, columns 32 qtr .. + 31.
        uint32_t a_raw = 0, b_raw = 0;
        {
            const int j = tid & 63, qtr = tid >> 6;
            const int64_t tok = t0 + (j < n ? j : 0);
            const uint4 *kp = reinterpret_cast<const uint4 *>(kg + tok * p.k_tok + h * p.k_head + 32 * qtr);
            const uint4 *qp = reinterpret_cast<const uint4 *>(qg + tok * p.q_tok + h * p.q_head + 32 * qtr);
            uint4 kr[4], qr[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                kr[c] = __ldg(kp + c);
                qr[c] = __ldg(qp + c);
            }
            if (j < n) {
                if (qtr == 0) {
                    a_raw = gate_raw(p.a, tok * p.a_tok + hv * p.a_head, p.a_f32);
                    b_raw = gate_raw(p.b, tok * p.b_tok + hv * p.b_head, p.b_f32);
                } else if (qtr == 1) {
                    sync::prefetch_l2(vg + tok * p.v_tok + hv * p.v_head, V * 2);
                }
            }
            float kk = 0.f, qq = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (j >= n)
                    kr[c] = qr[c] = make_uint4(0u, 0u, 0u, 0u);
                const int col = 32 * qtr + 8 * c;
                *reinterpret_cast<uint4 *>(k0 + tc::kmajor_offset(j, col, K)) = kr[c];
                *reinterpret_cast<uint4 *>(k0 + tc::kmajor_offset(64 + j, col, K)) = qr[c];
                float kf[8], qf[8];
                unpack8(kr[c], kf);
                unpack8(qr[c], qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kk = fmaf(kf[e], kf[e], kk);
                    qq = fmaf(qf[e], qf[e], qq);
                }
            }
            sm.kk[qtr][j] = kk;
            sm.qq[qtr][j] = qq;
        }
        __syncthreads();
        if (tid < C) {
            const int j = tid;
            float rk = 0.f, rq = 0.f, g = 0.f, be = 0.f;
            if (j < n) {
                rk = L2NORM ? rsqrtf(sm.kk[0][j] + sm.kk[1][j] + sm.kk[2][j] + sm.kk[3][j] + 1e-6f) : 1.f;
                rq = (L2NORM ? rsqrtf(sm.qq[0][j] + sm.qq[1][j] + sm.qq[2][j] + sm.qq[3][j] + 1e-6f) : 1.f) * p.scale;
                const float a_t = gate_value(a_raw, p.a_f32), b_t = gate_value(b_raw, p.b_f32);
                const float x = a_t + __ldg(p.dt_bias + hv * p.dt_stride);
                g = -expf(__ldg(p.A_log + hv * p.A_stride)) * (x > 20.f ? x : log1pf(expf(x)));
                be = 1.f / (1.f + expf(-b_t));
            }
            sm.rk[j] = rk;
            sm.rqs[j] = rq;
            sm.g[j] = g;
            sm.beta[j] = be;
        }
        __syncthreads();
        if (tid < C) {
            // gamma_j: running sum of g over rows 0..j, in index order (rows past
            // the end add exact zeros)
            const int j = tid;
            float acc = 0.f;
#pragma unroll
            for (int q4 = 0; q4 < C / 4; ++q4) {
                const float4 g4 = reinterpret_cast<const float4 *>(sm.g)[q4];
                const int r = 4 * q4;
                acc += r <= j ? g4.x : 0.f;
                acc += r + 1 <= j ? g4.y : 0.f;
                acc += r + 2 <= j ? g4.z : 0.f;
                acc += r + 3 <= j ? g4.w : 0.f;
            }
            sm.gam[j] = acc;
        }
        __syncthreads();
        if (tid < C) {
            const int j = tid;
            const float gj = sm.gam[j], gl = sm.gam[n - 1], ej = expf(gj);
            sm.fo[j] = ej * sm.rqs[j];
            sm.fd[j] = expf(gl - gj) * sm.rk[j];
            sm.fr[j] = ej * sm.rk[j];
            // A[j][c] = beta_j rk_j rk_c e^(gamma_j - gamma_c) (K K^T)[j][c] and
            // P[j][i] = rqs_j rk_i e^(gamma_j - gamma_i) (Q K^T)[j][i] as one power
            // of two each: 2^(ua_j - wc_c), 2^(uq_j - wc_i).  A zero factor (beta = 0,
            // or a row past the end) gives an exponent of -inf, hence an exact 0.
            const float g2 = gj * 1.4426950408889634f;
            sm.ua[j] = g2 + log2f(sm.beta[j] * sm.rk[j]);
            sm.uq[j] = g2 + log2f(sm.rqs[j]);
            sm.wc[j] = g2 - log2f(sm.rk[j]);
        }
        // the chunk's decay and the state scale after it (S = cs S~ before,
        // cs' after; S~ is rescaled once cs' leaves [2^-60, 2^60])
        __syncthreads();
        const float cn = cs * expf(sm.gam[n - 1]);
        const bool rescale = !(cn >= 0x1p-60f && cn <= 0x1p60f);
        const float dscale = rescale ? 1.f : __fdividef(1.f, cn);
        const float cs_new = rescale ? 1.f : cn;

        // ---- the state, first chunk: column v of S (this thread's rows k) from
        // the copied state into registers; then into TMEM (lane v of S~^T) and
        // the S~^T hi / lo tiles over the same region (later chunks: built from
        // TMEM at the end of the previous one)
        if (t0 == bos) {
            wait_bar(&sm.bar_x, ph_x);
            if (!ok)
                break;
            pend_x = false;
            const float *raw = reinterpret_cast<const float *>(sm.s);
            float x[64];
#pragma unroll
            for (int kk = 0; kk < 64; ++kk)
                x[kk] = raw[(64 * part + kk) * V + v];
            __syncthreads();
#pragma unroll
            for (int c = 0; c < 64; c += 16) {
                tc::tmem_st16(my_lane + COL_S + 64 * part + c, x + c);
                st_row8(s0, v, 64 * part + c, K, x + c, false);
                st_row8(s0, v, 64 * part + c + 8, K, x + c + 8, false);
                st_row8(s2, v, 64 * part + c, K, x + c, true);
                st_row8(s2, v, 64 * part + c + 8, K, x + c + 8, true);
            }
            tc::tmem_wait_st();
        }
        publish_smem();

        // ---- product D: S~^T [K;Q]^T -> (K S~)^T in COL_X, (Q S~)^T in COL_QS
        if (tid == 0) {
            mma_tiles(tmem + COL_X, s0, K, k0, K, K / 16, ID_N128, false);
            mma_tiles(tmem + COL_X, s2, K, k0, K, K / 16, ID_N128, true);
            tc::mma_commit(&sm.bar_m);
        }
        // meanwhile the chunk's v rows (thread (j, qtr): row j, columns 32 qtr ..
        // + 31, zeros past the end), 16 bytes at a time from L2
        uint4 vr[4];
        {
            const int j = tid & 63, qtr = tid >> 6;
            const uint4 *vp = reinterpret_cast<const uint4 *>(vg + (t0 + (j < n ? j : 0)) * p.v_tok + hv * p.v_head +
                                                              32 * qtr);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                vr[c] = j < n ? __ldg(vp + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;
        // the v rows into s3 (dead once product D is done), row-major with the
        // 16-byte chunks of row j XOR-swizzled by j % 16, so that both these
        // row stores and the column reads below spread over all banks
        unsigned short *const vrow = reinterpret_cast<unsigned short *>(s3);
        {
            const int j = tid & 63, qtr = tid >> 6;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4 *>(vrow + j * V + 8 * ((4 * qtr + c) ^ (j & 15))) = vr[c];
        }
        __syncthreads();

        // ---- R~^T[v][i] = beta_i (v_i[v] - e^gamma_i rk_i cs (K S~)_i[v]) / cs'
        // into its hi / lo tiles (over the S~ tiles, whose product is done); the
        // TMEM state rescaled if cs' left its range
        {
            float d[32], r[32];
            tc::tmem_ld16(my_lane + COL_X + ib, d);
            tc::tmem_ld16(my_lane + COL_X + ib + 16, d + 16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int ii = ib + e;
                const float vv = __uint_as_float(static_cast<uint32_t>(vrow[ii * V + 8 * ((v >> 3) ^ (ii & 15)) + (v & 7)])
                                                 << 16);
                r[e] = ii < n ? sm.beta[ii] * dscale * fmaf(-sm.fr[ii] * cs, d[e], vv) : 0.f;
            }
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
                st_row8(s0, v, ib + c, C, r + c, false);
                st_row8(s1, v, ib + c, C, r + c, true);
            }
        }
        if (rescale) {
#pragma unroll 1
            for (int c = 64 * part; c < 64 * part + 64; c += 16) {
                float x[16];
                tc::tmem_ld16(my_lane + COL_S + c, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] *= cn;
                tc::tmem_st16(my_lane + COL_S + c, x);
            }
            tc::tmem_wait_st();
        }
        publish_smem();

        // ---- product G: [K;Q] K^T -> lanes 0..63 K K^T, lanes 64..127 Q K^T
        if (tid == 0) {
            mma_tiles(tmem + COL_X, k0, K, k0, K, K / 16, ID_N64, false);
            tc::mma_commit(&sm.bar_m);
        }
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;

        // ---- A by columns into k1 (lanes 0..63: lane c holds row c of K K^T;
        // A[c][j] is nonzero for j < c < n, stored at column j, row c, so the
        // lanes' stores are consecutive words), and P by rows (lanes 64..127:
        // row j of Q K^T; P[j][i] for i <= j < n) as hi / lo tiles into k0.
        // Each lane's two threads take half of the columns.
        float *const At = reinterpret_cast<float *>(k1);
        if ((warp & 3) < 2) {
            const int c = v;
            const float uc = sm.ua[c];
#pragma unroll
            for (int jb = ib; jb < ib + 32; jb += 16) {
                float kk16[16];
                tc::tmem_ld16(my_lane + COL_X + jb, kk16);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const int j0 = jb + 4 * e4;
                    const float4 w4 = *reinterpret_cast<const float4 *>(sm.wc + j0);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = j0 + e;
                        At[j * 64 + c] = (j < c && c < n) ? kk16[4 * e4 + e] * ex2_approx(uc - wv[e]) : 0.f;
                    }
                }
            }
        } else {
            const int j = v - 64;
            const float u = sm.uq[j];
#pragma unroll
            for (int cb = ib; cb < ib + 32; cb += 16) {
                float pr[16];
                tc::tmem_ld16(my_lane + COL_X + cb, pr);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c = cb + e;
                    pr[e] = (c <= j && j < n) ? pr[e] * ex2_approx(u - sm.wc[c]) : 0.f;
                }
                st_row8(k0, j, cb, C, pr, false);
                st_row8(k0, j, cb + 8, C, pr + 8, false);
                st_row8(k0 + PIECE / 2, j, cb, C, pr, true);
                st_row8(k0 + PIECE / 2, j, cb + 8, C, pr + 8, true);
            }
        }
        tc::fence_before_sync();
        __syncthreads();

        // ---- T = (I + A)^-1 (by columns into s2), then its hi / lo row tiles
        // into s3
        float *const Tcol = reinterpret_cast<float *>(s2);
        solve_unit_lower64(At, Tcol, tid, n);
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            // rows past the end are rows of the identity (A is zero there); the
            // solve leaves them unwritten
            const int qi = tid + THREADS * it, r = qi & 63, c0 = (qi >> 6) * 8;
            float x8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                x8[e] = r < n ? (c0 + e <= r ? Tcol[(c0 + e) * 64 + (r ^ ((c0 + e) & 31))] : 0.f)
                              : (c0 + e == r ? 1.f : 0.f);
            st_row8(s3, r, c0, C, x8, false);
            st_row8(s3 + PIECE / 2, r, c0, C, x8, true);
        }
        publish_smem();

        // ---- product X: Delta~^T = R~^T T^T (hi / lo pairs) -> COL_X
        if (tid == 0) {
            mma_tiles(tmem + COL_X, s0, C, s3, C, C / 16, ID_N64, false);
            mma_tiles(tmem + COL_X, s0, C, s3 + PIECE / 2, C, C / 16, ID_N64, true);
            mma_tiles(tmem + COL_X, s1, C, s3, C, C / 16, ID_N64, true);
            tc::mma_commit(&sm.bar_m);
        }
        // meanwhile K' = diag(fd) K as hi / lo row tiles [i][k] (k1, s2: the A
        // and T column buffers are dead); the k rows again from global memory
        {
            const int ii = tid & 63, qtr = tid >> 6;
            const float f = sm.fd[ii];
            const int64_t tok = t0 + (ii < n ? ii : 0);
            const uint4 *kp = reinterpret_cast<const uint4 *>(kg + tok * p.k_tok + h * p.k_head + 32 * qtr);
            uint4 kr[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                kr[c] = __ldg(kp + c);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x[8];
                unpack8(kr[c], x);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    x[e] = ii < n ? x[e] * f : 0.f;
                st_row8(k1, ii, 32 * qtr + 8 * c, K, x, false);
                st_row8(s2, ii, 32 * qtr + 8 * c, K, x, true);
            }
        }
        tc::fence_proxy_async_smem();
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;

        // ---- Delta~^T (lane v) into its hi / lo tiles (over R~, whose product
        // is done)
        {
            float d[32];
            tc::tmem_ld16(my_lane + COL_X + ib, d);
            tc::tmem_ld16(my_lane + COL_X + ib + 16, d + 16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
                st_row8(s0, v, ib + c, C, d + c, false);
                st_row8(s1, v, ib + c, C, d + c, true);
            }
        }
        publish_smem();

        // ---- product Y: S~^T += Delta~^T K' (K' read MN-major), O2^T =
        // Delta~^T P^T -> COL_X
        if (tid == 0) {
            mma_tiles_bmn(tmem + COL_S, s0, C, k1, K, C / 16, ID_N128_BMN, true);
            mma_tiles_bmn(tmem + COL_S, s0, C, s2, K, C / 16, ID_N128_BMN, true);
            mma_tiles_bmn(tmem + COL_S, s1, C, k1, K, C / 16, ID_N128_BMN, true);
            mma_tiles(tmem + COL_X, s0, C, k0, C, C / 16, ID_N64, false);
            mma_tiles(tmem + COL_X, s0, C, k0 + PIECE / 2, C, C / 16, ID_N64, true);
            mma_tiles(tmem + COL_X, s1, C, k0, C, C / 16, ID_N64, true);
            tc::mma_commit(&sm.bar_m);
        }
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;

        // ---- outputs o_j = fo_j cs (Q S~)_j + cs' O2_j: thread (v, part) puts
        // column v of its 32 tokens into a row-major bf16 [j][v] stage (s0: the
        // Delta~ tiles are dead), then whole rows go out 8 bytes at a time
        __nv_bfloat16 *const stage = reinterpret_cast<__nv_bfloat16 *>(s0);
#pragma unroll
        for (int cl = 0; cl < 32; cl += 16) {
            const int cb = ib + cl;
            float o1[16], o2[16];
            tc::tmem_ld16(my_lane + COL_QS + cb, o1);
            tc::tmem_ld16(my_lane + COL_X + cb, o2);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = cb + e;
                stage[j * V + v] = __float2bfloat16_rn(fmaf(sm.fo[j] * cs, o1[e], cs_new * o2[e]));
            }
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < C * V / 4 / THREADS; ++it) {
            const int idx = tid + THREADS * it, j = idx >> 5, c4 = 4 * (idx & 31);
            if (j < n)
                *reinterpret_cast<uint2 *>(out + (t0 + j) * p.o_tok + hv * p.o_head + c4) =
                    *reinterpret_cast<const uint2 *>(stage + j * V + c4);
        }
        __syncthreads();

        // ---- the next chunk's S~^T tiles (all tiles of this chunk are dead),
        // or the final write-back
#pragma unroll 1
        for (int c = 64 * part; c < 64 * part + 64; c += 16) {
            float x[16];
            tc::tmem_ld16(my_lane + COL_S + c, x);
            tc::tmem_wait_ld();
            if (more) {
                st_row8(s0, v, c, K, x, false);
                st_row8(s0, v, c + 8, K, x + 8, false);
                st_row8(s2, v, c, K, x, true);
                st_row8(s2, v, c + 8, K, x + 8, true);
            } else if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    __stcs(s_gmem + (c + e) * V + v, cs_new * x[e]);
            }
        }
        cs = cs_new;
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }

    // a failed wait may leave the state's copy in flight: let it land
    // (bounded) before the shared memory is released
    if (pend_x) {
        volatile int never = 0;
        sync::mbar_wait(&sm.bar_x, 0, &never);
    }

    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace local
}  // namespace gdn

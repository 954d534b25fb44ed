// gdn_chunk_split.cuh -- the chunked Gated DeltaNet update split into two
// sm_100a kernels around a caller-provided workspace (GDN_SCHEDULE_CHUNKED_SPLIT).
//
// The chunk form of the update (the WY representation behind the pages'
// chunked GDN kernels) has two kinds of work per chunk: products that need
// only the chunk's own inputs (the decay scan, A, the triangular solve
// T = (I + A)^-1, W, U and the masked q.k matrix P -- the pages'
// chunk_scaled_dot_kkt, solve_tril and recompute_w_u steps) and the
// recurrence through the state (Delta = U - W S0, the outputs, the state
// update -- chunk_gated_delta_rule_fwd_h and chunk_fwd_o).  The single-kernel
// schedule (gdn_chunk_local.cuh) runs both in one CTA per (sequence, head),
// chunk after chunk, so the state-independent work sits on the sequential
// critical path; with few, long sequences that path is what counts.  Here:
//
//   gdn_chunk_wy_kernel     one CTA per (64-token block of the packed token
//                           range, value head), all in parallel: writes the
//                           block's W^T, Q^T, K' = diag(fd) K, P^T and U^T
//                           into the workspace as the byte images of the
//                           operand tiles the second kernel feeds to tcgen05
//                           (row by row, as the block kernel produces them).
//   gdn_chunk_state_kernel  one 544-thread CTA per (sequence, value head) (or, for
//                           many short sequences, gdn_chunk_state_compact_kernel:
//                           256 threads, two CTAs per SM; for few pairs,
//                           gdn_chunk_state_half_kernel in
//                           gdn_chunk_state_half.cuh: two CTAs per pair, each
//                           on half of the state's columns): walks the
//                           blocks the sequence covers, fetching each block's
//                           tiles with bulk copies one step ahead, and runs
//                           only the state-dependent products.
//
// Blocks are aligned to the packed token range, not to sequences: a block may
// hold the end of one sequence and the start of the next.  Each token's
// quantities are therefore taken within its SEGMENT (the part of its sequence
// inside the block): the decay scan restarts at the segment start and A, P
// are masked to the segment, which makes T, W, U block-diagonal by segment.
// The state kernel processes a sequence as the pieces it has in each block.
//
// Within a segment, with gamma_j the running sum of g from the segment start,
// hats the normalised vectors and S0 the state before the piece:
//     A[j][i] = beta_j e^(gamma_j - gamma_i) k^_j . k^_i   (i < j, same segment)
//     T = (I + A)^-1,  W = T diag(beta e^gamma rk) K,  U = T diag(beta) V
//     Delta  = U - W S0
//     o_j    = e^gamma_j rqs_j S0^T q_j + sum_i P[j][i] Delta_i,
//              P[j][i] = e^(gamma_j - gamma_i) rqs_j rk_i q_j . k_i  (i <= j, same segment)
//     S'     = e^gamma_last S0 + sum_i fd_i k_i Delta_i^T,  fd_i = e^(gamma_last - gamma_i) rk_i
// Operands that are not exact bf16 are split into bf16 hi + lo parts and
// multiplied as hi*hi + hi*lo + lo*hi (fp32 accumulators in TMEM; see
// gdn_chunk_common.cuh).
#pragma once

#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn_chunk_common.cuh"
#include "gdn_decode.h"
#include "gdn_decode_kernel.cuh"
#include "mbarrier_sm100.cuh"
#include "tc_sm100.cuh"

namespace gdn {
namespace split {

using chunk::mma_tiles;
using chunk::st_row8;
using chunk::st_row8_hilo;

// D (+)= A B^T with A a K-major [128][a_cols] tile (k-slices of 16 columns)
// and B stored as the [kdim][b_cols] row tile of B^T, read MN-major: core
// matrices 128 bytes apart along N (= b_cols), (b_cols / 8) * 128 bytes apart
// along the contraction.
__device__ __forceinline__ void mma_tiles_bmn(uint32_t d, const unsigned char *a, uint32_t a_cols,
                                              const unsigned char *b, uint32_t b_cols, uint32_t slices,
                                              uint32_t idesc, bool accumulate)
{
    const uint32_t kstride = (b_cols >> 3) * 128u;
#pragma unroll 1
    for (uint32_t s = 0; s < slices; ++s)
        tc::mma_bf16(d, tc::kslice_desc(a, a_cols, s), tc::mn_desc(tc::smem_u32(b) + s * 2u * kstride, kstride, 128u),
                     idesc, (accumulate || s > 0) ? 1u : 0u);
}

// 2^x with the hardware approximation (PTX ex2.approx.ftz: a few ulp of
// relative error; results below 2^-126 flush to zero), for the A and P
// factors: values that small are far below what the fp32 products resolve,
// and entries outside the masks are discarded by a select, whatever they are.
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr int K = 128;
constexpr int V = 128;
constexpr int C = 64;            // tokens per block
constexpr int THREADS = 128;

// One workspace record per (block, value head): byte offsets.  Tiles are in
// the core-matrix layout of tc_sm100.cuh (tc::kmajor_offset) for [r][c]: 16-byte
// rows of 8 consecutive c, r being the contraction index of the product that
// reads them; they are read as MN-major operands, [W^T hi | Q^T] as one
// 128-wide operand and [K' | P^T] as one 192-wide operand.
constexpr uint32_t REC_WQ_HI = 0;         // [W^T hi | Q^T]    [k][i | j]    32 KB
constexpr uint32_t REC_W_LO = 32768;      // W^T lo            [k][i]        16 KB
constexpr uint32_t WQ_COLS = C + C;       // 128
constexpr uint32_t REC_KP_HI = 49152;     // [K' | P^T] hi     [i][k | j]    24 KB
constexpr uint32_t REC_KP_LO = 73728;     // [K' | P^T] lo     [i][k | j]    24 KB
constexpr uint32_t KP_COLS = K + C;       // 192
constexpr uint32_t REC_UT = 98304;        // U^T fp32, row-major [v][i]  32 KB
constexpr uint32_t REC_FO = 131072;       // fo_j = e^gamma_j rqs_j     256 B
constexpr uint32_t REC_GAM = 131328;      // gamma_j                    256 B
constexpr uint32_t REC_BYTES = 131584;    // a multiple of 256
constexpr uint32_t REC_A_BYTES = REC_KP_HI;               // [W^T hi | Q^T], W^T lo
constexpr uint32_t REC_B_BYTES = REC_UT - REC_KP_HI;      // [K' | P^T] hi, lo
constexpr uint32_t REC_S_BYTES = REC_BYTES - REC_FO;      // fo, gamma

__host__ __device__ constexpr uint64_t workspace_bytes(int64_t T_tot, int64_t HV)
{
    return static_cast<uint64_t>((T_tot + C - 1) / C) * static_cast<uint64_t>(HV) * REC_BYTES;
}

// Index of A[j][c] in the by-columns fp32 store of A (64 x 64): column c is
// 64 contiguous floats.  (An XOR swizzle of its 16-byte groups removes the
// bank conflicts of the column writes but its index arithmetic in the
// unrolled solve cost more than it saved: 1.3 % on the split schedule.)
__device__ __forceinline__ int at_idx(int c, int j) { return c * 64 + j; }

// T = (I + A)^-1 for A strictly lower triangular (64 x 64, fp32), by
// recursive doubling over 16 x 16 blocks:
//   level 1: the diagonal blocks by substitution, a thread per column;
//   level 2: T_10 = -T_11 (A_10 T_00) and T_32 = -T_33 (A_32 T_22);
//   level 3: T_[23][01] = -T_[23][23] (A_[23][01] T_[01][01]) (32 x 32).
// A is stored by columns (At[at_idx(c, r)] = A[r][c]); the intermediate
// products sit in its upper triangle, whose entries (A[r][c] = 0 for r < c)
// are never read: level 2's at column block 2p + 1, rows of block 2p; level
// 3's at columns 32.., rows ..31.  T is written by columns with the row index
// XOR-swizzled by the column (Tcol[c * 64 + (r ^ (c & 31))]); the diagonal
// blocks are written in full (their upper triangles zero), the blocks above
// them never, and every read that can reach one selects zero instead.
// Threads 0..127 compute; every thread of the CTA must call this (it holds
// the CTA's barriers), and it ends with one.  When only the first n rows of A
// can be nonzero (n uniform over the CTA), the blocks of T in rows >= n --
// rows of the identity -- are skipped: level 1's blocks starting at or past
// n, level 2's pairs whose lower block does, and level 3 for n <= 32; the
// caller must then take T's rows >= n as identity rows instead of reading
// them.  n = 64 computes every block.
__device__ __forceinline__ void solve_unit_lower64(float *At, float *Tcol, int tid, int n = 64)
{
    const int warp = tid >> 5;
    auto T_at = [&](int r, int c) -> float & { return Tcol[c * 64 + (r ^ (c & 31))]; };
    if (tid < 64 && 16 * (tid >> 4) < n) {
        // level 1: thread (bw, cl) takes column cl of diagonal block bw
        // (rows b .. b + 15, b = 16 bw), all 16 rows in registers: x = e_cl;
        // for r = 0 .. 14, x_rho -= A[rho][r] x_r for every rho (A[rho][r] = 0
        // unless rho > r; x_r is final once the steps before r are done).
        // Column r of the block is read as the 16-byte groups holding rows
        // > r; no lane exchanges, so the only dependent chain is the FMAs.
        const int b = 16 * (tid >> 4), cl = tid & 15;
        float x[16];
#pragma unroll
        for (int rho = 0; rho < 16; ++rho)
            x[rho] = (rho == cl) ? 1.f : 0.f;
#pragma unroll
        for (int r = 0; r < 15; ++r) {
#pragma unroll
            for (int g = (r + 1) >> 2; g < 4; ++g) {
                const float4 a4 = *reinterpret_cast<const float4 *>(At + at_idx(b + r, b + 4 * g));
                x[4 * g] = fmaf(-a4.x, x[r], x[4 * g]);
                x[4 * g + 1] = fmaf(-a4.y, x[r], x[4 * g + 1]);
                x[4 * g + 2] = fmaf(-a4.z, x[r], x[4 * g + 2]);
                x[4 * g + 3] = fmaf(-a4.w, x[r], x[4 * g + 3]);
            }
        }
#pragma unroll
        for (int rho = 0; rho < 16; ++rho)
            T_at(b + rho, b + cl) = x[rho];
    }
    __syncthreads();
    const int t64 = tid & 63, pr = warp >> 1, C0 = 32 * pr, R1 = C0 + 16;
    const bool level2 = tid < 128 && R1 < n, level3 = n > 32;
    if (level2) {
        // level 2, product 1: M1 = A_[R1][C0] T_[C0][C0] (16 x 16) of pair
        // pr; thread: column j, rows 4 rg .. 4 rg + 3
        const int j = t64 & 15, rg = t64 >> 4;
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const float t = T_at(C0 + kk, C0 + j);
            const float4 a4 = *reinterpret_cast<const float4 *>(At + at_idx(C0 + kk, R1 + 4 * rg));
            m[0] = fmaf(a4.x, t, m[0]);
            m[1] = fmaf(a4.y, t, m[1]);
            m[2] = fmaf(a4.z, t, m[2]);
            m[3] = fmaf(a4.w, t, m[3]);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
            At[at_idx(R1 + 4 * rg + ii, C0 + j)] = m[ii];      // M1[i][j]
    }
    __syncthreads();
    if (level2) {
        // level 2, product 2: T_[R1][C0] = -T_[R1][R1] M1; thread: row i,
        // columns 4 cg .. 4 cg + 3
        const int i = t64 & 15, cg = t64 >> 4;
        float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const float t = T_at(R1 + i, R1 + kk);
            const float4 m4 = *reinterpret_cast<const float4 *>(At + at_idx(R1 + kk, C0 + 4 * cg));
            o[0] = fmaf(-t, m4.x, o[0]);
            o[1] = fmaf(-t, m4.y, o[1]);
            o[2] = fmaf(-t, m4.z, o[2]);
            o[3] = fmaf(-t, m4.w, o[3]);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            T_at(R1 + i, C0 + 4 * cg + jj) = o[jj];
    }
    __syncthreads();
    if (!level3)
        return;
    if (tid < 128) {
        // level 3, product 1: M = A_[23][01] T_[01][01] (32 x 32); thread:
        // column j = lane, rows 8 w .. 8 w + 7
        const int j = tid & 31;
        float m[8];
#pragma unroll
        for (int ii = 0; ii < 8; ++ii)
            m[ii] = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            const float t = kk >= j ? T_at(kk, j) : 0.f;
            const float4 a0 = *reinterpret_cast<const float4 *>(At + at_idx(kk, 32 + 8 * warp));
            const float4 a1 = *reinterpret_cast<const float4 *>(At + at_idx(kk, 36 + 8 * warp));
            m[0] = fmaf(a0.x, t, m[0]);
            m[1] = fmaf(a0.y, t, m[1]);
            m[2] = fmaf(a0.z, t, m[2]);
            m[3] = fmaf(a0.w, t, m[3]);
            m[4] = fmaf(a1.x, t, m[4]);
            m[5] = fmaf(a1.y, t, m[5]);
            m[6] = fmaf(a1.z, t, m[6]);
            m[7] = fmaf(a1.w, t, m[7]);
        }
#pragma unroll
        for (int ii = 0; ii < 8; ++ii)
            At[at_idx(32 + 8 * warp + ii, j)] = m[ii];       // M[i][j]
    }
    __syncthreads();
    if (tid < 128) {
        // level 3, product 2: T_[23][01] = -T_[23][23] M; thread: row
        // 32 + i (i = lane), columns 8 w .. 8 w + 7
        const int i = tid & 31;
        float o[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            o[jj] = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            const float t = kk <= i ? T_at(32 + i, 32 + kk) : 0.f;
            const float4 m0 = *reinterpret_cast<const float4 *>(At + at_idx(32 + kk, 8 * warp));
            const float4 m1 = *reinterpret_cast<const float4 *>(At + at_idx(32 + kk, 4 + 8 * warp));
            o[0] = fmaf(-t, m0.x, o[0]);
            o[1] = fmaf(-t, m0.y, o[1]);
            o[2] = fmaf(-t, m0.z, o[2]);
            o[3] = fmaf(-t, m0.w, o[3]);
            o[4] = fmaf(-t, m1.x, o[4]);
            o[5] = fmaf(-t, m1.y, o[5]);
            o[6] = fmaf(-t, m1.z, o[6]);
            o[7] = fmaf(-t, m1.w, o[7]);
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            T_at(32 + i, 8 * warp + jj) = o[jj];
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Kernel 1: the state-independent products of one (block, value head).
// ---------------------------------------------------------------------------
struct WySmem {
    // raw k rows 0..63 [i][k] (kept until the record's K' is written; also
    // the MN-major A operand K^T of the W product) and raw q rows 64..127
    // (until the K K^T / Q K^T product; then A by columns (fp32), then the
    // T diag(fw) hi / lo tiles and, once the W product is done, the
    // T diag(beta) ones)
    alignas(1024) unsigned char kq[128 * 128 * 2];
    // T by columns (fp32), then the raw v rows [i][v] (the MN-major A operand
    // V^T of the U product)
    alignas(1024) unsigned char r2[64 * 128 * 2];
    float kk[2][C], qq[2][C];                          // |k_j|^2, |q_j|^2 over each half of the row
    float rk[C], rqs[C], g[C], beta[C], gam[C];
    float fw[C], fo[C], fd[C];
    // base-2 exponents of the A and P factors (see step 3)
    float ua[C], uq[C], wc[C];
    int ss[C], se[C];                                  // segment [ss, se) of row j within the block
    unsigned long long mbar;
    uint32_t tmem_base;
    int failed;
};

static_assert(offsetof(WySmem, g) % 16 == 0 && offsetof(WySmem, ua) % 16 == 0 && offsetof(WySmem, wc) % 16 == 0,
              "g, ua and wc are read as 16-byte vectors");

constexpr uint32_t WY_TMEM_COLS = 128;
constexpr uint32_t WY_COL_KQ = 0;     // K [K;Q]^T  [i][c | j] 128 columns (read before the W / U products)
constexpr uint32_t WY_COL_WT = 0;     // W^T        [k][j]   64
constexpr uint32_t WY_COL_UT = 64;    // U^T        [v][j]   64

template <bool L2NORM>
__global__ void __launch_bounds__(THREADS, 4) gdn_chunk_wy_kernel(const __grid_constant__ DecodeParams p,
                                                                unsigned char *__restrict__ ws)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    WySmem &sm = *reinterpret_cast<WySmem *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int blk = blockIdx.x / p.HV;
    const int hv = blockIdx.x - blk * p.HV;
    const int h = hv / p.G;
    const int64_t t0 = static_cast<int64_t>(blk) * C;
    const int n = p.T_tot - t0 < C ? static_cast<int>(p.T_tot - t0) : C;
    unsigned char *const rec = ws + (static_cast<int64_t>(blk) * p.HV + hv) * REC_BYTES;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
    unsigned char *const kq = sm.kq, *const ktile = sm.kq, *const qhalf = sm.kq + 16384, *const vtile = sm.r2;
    // the T diag() operand tiles, in turn over the q half of kq
    unsigned char *const tw_hi = qhalf, *const tw_lo = qhalf + 8192, *const tu_hi = qhalf, *const tu_lo = qhalf + 8192;

    if (tid == 0) {
        sync::mbar_init(&sm.mbar, 1);
        sm.failed = 0;
        sync::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, WY_TMEM_COLS);
        tc::tmem_relinquish();
    }

    uint32_t a_raw = 0, b_raw = 0;      // raw gates of row tid (threads 0..63)
    // ---- step 1: raw k and q rows of the block into the operand tile
    // (K-major for the K K^T / Q K^T product; the k rows also serve the W
    // product as the MN-major operand K^T); raw q also straight into the
    // record; squared norms of k and q; the v rows (needed from the U
    // product on) are only fetched into L2.  Thread (j, half) handles row
    // j, columns 64 half .. 64 half + 63, so a warp's 16-byte stores cover
    // 32 consecutive rows (no bank conflicts).
    {
        const int j = tid & 63, half = tid >> 6;
        const int64_t tok = t0 + (j < n ? j : 0);
        const __nv_bfloat16 *kp = k + tok * p.k_tok + h * p.k_head + 64 * half;
        const __nv_bfloat16 *qp = q + tok * p.q_tok + h * p.q_head + 64 * half;
        uint4 kr[8], qr[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            kr[c] = __ldg(reinterpret_cast<const uint4 *>(kp) + c);
            qr[c] = __ldg(reinterpret_cast<const uint4 *>(qp) + c);
        }
        if (half == 0) {
            // row j's gates (used after the barrier) and its v row into L2
            if (j < n) {
                sync::prefetch_l2(v + tok * p.v_tok + hv * p.v_head, V * 2);
                a_raw = gate_raw(p.a, tok * p.a_tok + hv * p.a_head, p.a_f32);
                b_raw = gate_raw(p.b, tok * p.b_tok + hv * p.b_head, p.b_f32);
            }
        } else {
            // segment [ss, se) of row j within the block (rows past the end:
            // a segment of their own), while the loads above are in flight
            int ss = j, se = j + 1;
            if (j < n) {
                int64_t s_beg, s_end;
                if (p.cu_seqlens) {
                    // the last sequence starting at or before tok (binary search
                    // over cu_seqlens[0..N]; kept in bounds even if it is invalid)
                    int lo = 0, hi = p.N;            // cu[lo] <= tok < cu[hi] when valid
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (__ldg(p.cu_seqlens + mid) <= tok)
                            lo = mid;
                        else
                            hi = mid;
                    }
                    s_beg = __ldg(p.cu_seqlens + lo);
                    s_end = __ldg(p.cu_seqlens + lo + 1);
                } else {
                    const int64_t s = tok / p.T_fixed;
                    s_beg = s * p.T_fixed;
                    s_end = s_beg + p.T_fixed;
                }
                if (s_beg <= tok && tok < s_end) {
                    ss = static_cast<int>((s_beg > t0 ? s_beg : t0) - t0);
                    se = static_cast<int>((s_end < t0 + n ? s_end : t0 + n) - t0);
                }
            }
            sm.ss[j] = ss;
            sm.se[j] = se;
        }
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (j >= n)
                kr[c] = qr[c] = make_uint4(0u, 0u, 0u, 0u);
            const int col = 64 * half + 8 * c;
            *reinterpret_cast<uint4 *>(kq + tc::kmajor_offset(j, col, K)) = kr[c];
            *reinterpret_cast<uint4 *>(kq + tc::kmajor_offset(64 + j, col, K)) = qr[c];
            float kf[8], qf[8];
            unpack8(kr[c], kf);
            unpack8(qr[c], qf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                kk = fmaf(kf[e], kf[e], kk);
                qq = fmaf(qf[e], qf[e], qq);
            }
        }
        sm.kk[half][j] = kk;
        sm.qq[half][j] = qq;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, warp * 32, 0);

    // Q^T into the record (columns 64.. of [W^T hi | Q^T]) by warps 2 and 3
    // while warps 0 and 1 compute the per-row scalars: each 8 x 8 block (rows
    // 8 jg.., columns 8 kg..) of the q rows is one core matrix of the row tile,
    // loaded transposed with ldmatrix; lane t then holds Q^T[8 kg + t/4][8 jg +
    // 2 (t%4) + {0, 1}], and a warp's 4-byte stores fill the block's 128 bytes.
    auto q_transposed = [&](int it0, int it1) {
        const int lane = tid & 31;
        for (int it = it0; it < it1; ++it) {
            const int mb = ((warp - 2) * 16 + it) * 4;          // 4 blocks per load
            const int mr = mb + (lane >> 3);
            const uint32_t src = tc::smem_u32(qhalf + tc::kmajor_offset(8 * (mr & 7) + (lane & 7), 8 * (mr >> 3), K));
            uint32_t d[4];
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                         : "r"(src));
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int m = mb + x;
                *reinterpret_cast<uint32_t *>(rec + REC_WQ_HI +
                                              tc::kmajor_offset(8 * (m >> 3) + (lane >> 2), C + 8 * (m & 7) + 2 * (lane & 3),
                                                                WQ_COLS)) = d[x];
            }
        }
    };

    // ---- per-row scalars: gates and norms (threads 0..63) ----------------
    if (tid >= C)
        q_transposed(0, 8);
    if (tid < C) {
        const int j = tid;
        float rk = 0.f, rq = 0.f, g = 0.f, be = 0.f;
        if (j < n) {
            rk = L2NORM ? rsqrtf(sm.kk[0][j] + sm.kk[1][j] + 1e-6f) : 1.f;
            rq = (L2NORM ? rsqrtf(sm.qq[0][j] + sm.qq[1][j] + 1e-6f) : 1.f) * p.scale;
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
    if (tid >= C)
        q_transposed(8, 16);
    if (tid < C) {
        // gamma_j: running sum of g over the row's segment, in index order
        // (the masked-out terms add exact zeros); the 16-byte reads of g are
        // the same for every thread
        const int j = tid, s0 = sm.ss[j];
        float acc = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < C / 4; ++q4) {
            const float4 g4 = reinterpret_cast<const float4 *>(sm.g)[q4];
            const int i = 4 * q4;
            acc += (i >= s0 && i <= j) ? g4.x : 0.f;
            acc += (i + 1 >= s0 && i + 1 <= j) ? g4.y : 0.f;
            acc += (i + 2 >= s0 && i + 2 <= j) ? g4.z : 0.f;
            acc += (i + 3 >= s0 && i + 3 <= j) ? g4.w : 0.f;
        }
        sm.gam[j] = acc;
    }
    __syncthreads();
    if (tid < C) {
        const int j = tid;
        const float gj = sm.gam[j], gl = sm.gam[sm.se[j] - 1];
        sm.fw[j] = sm.beta[j] * expf(gj) * sm.rk[j];
        sm.fo[j] = expf(gj) * sm.rqs[j];
        sm.fd[j] = expf(gl - gj) * sm.rk[j];
        // A[j][c] = beta_j rk_j rk_c e^(gamma_j - gamma_c) (K K^T)[j][c] and
        // P[j][i] = rqs_j rk_i e^(gamma_j - gamma_i) (Q K^T)[j][i] as one power
        // of two each: 2^(ua_j - wc_c), 2^(uq_j - wc_i).  A zero factor (beta = 0,
        // or a row past the end) gives an exponent of -inf, hence an exact 0.
        const float g2 = gj * 1.4426950408889634f;
        sm.ua[j] = g2 + log2f(sm.beta[j] * sm.rk[j]);
        sm.uq[j] = g2 + log2f(sm.rqs[j]);
        sm.wc[j] = g2 - log2f(sm.rk[j]);
        reinterpret_cast<float *>(rec + REC_FO)[j] = sm.fo[j];
        reinterpret_cast<float *>(rec + REC_GAM)[j] = gj;
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    uint32_t phase = 0;
    bool ok = true;
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
    auto publish_smem = [&]() {
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    // D[128 x 64] (+)= A B^T, A read MN-major from a raw [64][128] row tile
    // (its transpose), B a K-major [64][64] tile
    auto mma_amn = [&](uint32_t d, const unsigned char *a, const unsigned char *b, bool acc) {
        const uint32_t ID_AMN = tc::idesc_bf16_f32(128, 64, false, true);
        for (uint32_t sl = 0; sl < C / 16; ++sl)
            tc::mma_bf16(d, tc::mn_desc(tc::smem_u32(a) + sl * 2u * 2048u, 2048u, 128u), tc::kslice_desc(b, C, sl),
                         ID_AMN, (acc || sl > 0) ? 1u : 0u);
    };

    // ---- step 2: [K;Q] [K;Q]^T, of which lanes 0..63 (the k rows) are used:
    // K K^T in columns 0..63, K Q^T in 64..127 -------------------------------
    if (tid == 0) {
        mma_tiles(tmem + WY_COL_KQ, kq, K, kq, K, K / 16, tc::idesc_bf16_f32(128, 128), false);
        tc::mma_commit(&sm.mbar);
    }
    wait_mma();

    // A stored by columns, At[at_idx(c, j)] = A[j][c] (fp32 [64][64], over the
    // q half of kq, consumed by the product above), and T by columns with the
    // row index XOR-swizzled by the column (fp32 [64][64], in r2)
    float *At = reinterpret_cast<float *>(qhalf);
    float *Tcol = reinterpret_cast<float *>(sm.r2);
    float t8[4][8];     // rows of T, kept for the two T diag() tile pairs
    if (ok) {
        // ---- step 3: A and P^T by columns of K [K;Q]^T (warps 0, 1) and the
        // K' rows (warps 2, 3).  TMEM lane c holds row c of K K^T and of
        // K Q^T: thread c writes row c of A into At (column j, row c: the
        // lanes' stores are consecutive words; writing column c of the
        // symmetric K K^T as 16-byte vectors instead was a 32-way bank
        // conflict) and row c of P^T to the record.  A[c][j] is nonzero for
        // j < c in the same segment, i.e. ss_c <= j < c; P[j][c] for
        // c <= j < se_c.
        if (tid < 64) {
            const int c = tid, cs0 = sm.ss[c], ce = sm.se[c];
            const float uc = sm.ua[c], w = sm.wc[c];
#pragma unroll 1
            for (int jb = 0; jb < 64; jb += 16) {
                float kk16[16];
                tc::tmem_ld16(my_lane + WY_COL_KQ + jb, kk16);
                tc::tmem_wait_ld();
                // A[c][j] = 2^(ua_c - wc_j) (K K^T)[c][j]
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const int j0 = jb + 4 * e4;
                    const float4 w4 = *reinterpret_cast<const float4 *>(sm.wc + j0);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = j0 + e;
                        At[at_idx(j, c)] = (j < c && j >= cs0) ? kk16[4 * e4 + e] * ex2_approx(uc - wv[e]) : 0.f;
                    }
                }
            }

#pragma unroll 1
            for (int jb = 0; jb < 64; jb += 16) {
                float pt[16];
                tc::tmem_ld16(my_lane + WY_COL_KQ + 64 + jb, pt);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 u4 = *reinterpret_cast<const float4 *>(sm.uq + jb + 4 * e4);
                    const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = jb + 4 * e4 + e;
                        pt[4 * e4 + e] = (j >= c && j < ce) ? pt[4 * e4 + e] * ex2_approx(uv[e] - w) : 0.f;
                    }
                }
                st_row8_hilo(rec + REC_KP_HI, rec + REC_KP_LO, c, K + jb, KP_COLS, pt);
                st_row8_hilo(rec + REC_KP_HI, rec + REC_KP_LO, c, K + jb + 8, KP_COLS, pt + 8);
            }
        } else {
            // K' = diag(fd) K: row j of the raw k rows, scaled, hi / lo
            const int j = tid - 64;
            const float f = sm.fd[j];
#pragma unroll 4
            for (int col = 0; col < K; col += 8) {
                float x[8];
                unpack8(*reinterpret_cast<const uint4 *>(ktile + tc::kmajor_offset(j, col, K)), x);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    x[e] *= f;
                st_row8_hilo(rec + REC_KP_HI, rec + REC_KP_LO, j, col, KP_COLS, x);
            }
        }
        __syncthreads();

        // ---- step 4: T = (I + A)^-1 (A strictly lower triangular)
        solve_unit_lower64(At, Tcol, tid);

        // T diag(fw) and T diag(beta) as hi / lo operand tiles, in turn over
        // the q half of kq: each thread keeps four 8-column chunks of rows of
        // T in registers (thread: row r = qi & 63, so a warp's reads of T and
        // its 16-byte tile stores cover 32 consecutive rows)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const int qi = tid + 128 * ch, r = qi & 63, c0 = (qi >> 6) * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                t8[ch][e] = c0 + e <= r ? Tcol[(c0 + e) * 64 + (r ^ ((c0 + e) & 31))] : 0.f;
        }
        __syncthreads();
        // the raw v rows into r2, asynchronously (rows past the end: zeros)
        {
            const int j = tid & 63, half = tid >> 6;
            const __nv_bfloat16 *vp = v + (t0 + (j < n ? j : 0)) * p.v_tok + hv * p.v_head + 64 * half;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                sync::cp_async16(vtile + tc::kmajor_offset(j, 64 * half + 8 * c, V), vp + 8 * c, j < n ? 16u : 0u);
            sync::cp_async_commit();
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const int qi = tid + 128 * ch, r = qi & 63, c0 = (qi >> 6) * 8;
            float x8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                x8[e] = t8[ch][e] * sm.fw[c0 + e];
            st_row8_hilo(tw_hi, tw_lo, r, c0, C, x8);
        }
        publish_smem();

        // ---- step 5: W^T = K^T T_w^T, then U^T = V^T T_u^T, with K^T and V^T
        // read MN-major straight from the raw row tiles (8-row groups of
        // tokens 2048 bytes apart, 8-column chunks 128 bytes apart) -----------
        if (tid == 0) {
            mma_amn(tmem + WY_COL_WT, ktile, tw_hi, false);
            mma_amn(tmem + WY_COL_WT, ktile, tw_lo, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
    }
    if (ok) {
        // T diag(beta) over the T diag(fw) tiles, whose product is done
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const int qi = tid + 128 * ch, r = qi & 63, c0 = (qi >> 6) * 8;
            float x8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                x8[e] = t8[ch][e] * sm.beta[c0 + e];
            st_row8_hilo(tu_hi, tu_lo, r, c0, C, x8);
        }
        sync::cp_async_wait_all();
        publish_smem();
        if (tid == 0) {
            mma_amn(tmem + WY_COL_UT, vtile, tu_hi, false);
            mma_amn(tmem + WY_COL_UT, vtile, tu_lo, true);
            tc::mma_commit(&sm.mbar);
        }
        wait_mma();
    }
    if (ok) {
        // ---- step 6: the record's remaining tiles -------------------------
        // W^T (thread = k): row k of W^T from TMEM, hi / lo, straight to the
        // record
#pragma unroll 1
        for (int c = 0; c < 64; c += 16) {
            float w[16];
            tc::tmem_ld16(my_lane + WY_COL_WT + c, w);
            tc::tmem_wait_ld();
            st_row8(rec + REC_WQ_HI, tid, c, WQ_COLS, w, false);
            st_row8(rec + REC_WQ_HI, tid, c + 8, WQ_COLS, w + 8, false);
            st_row8(rec + REC_W_LO, tid, c, C, w, true);
            st_row8(rec + REC_W_LO, tid, c + 8, C, w + 8, true);
        }
        // U^T (thread = v): one fp32 row of 64
        {
            float4 *dst = reinterpret_cast<float4 *>(rec + REC_UT) + tid * 16;
#pragma unroll
            for (int c = 0; c < 64; c += 16) {
                float u[16];
                tc::tmem_ld16(my_lane + WY_COL_UT + c, u);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    dst[(c + e) / 4] = make_float4(u[e], u[e + 1], u[e + 2], u[e + 3]);
            }
        }
    }

    sync::cp_async_wait_all();      // the v rows' copies, on a path that skipped their use
    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, WY_TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Kernel 2: the recurrence through the state of one (sequence, value head).
// ---------------------------------------------------------------------------

// Product 1 of a piece, issued by one thread and committed to `bar`:
// [D | O1] = -S~^T [W hi; Q]^T (N = 128, from column dq_col) from the hi and
// lo state tiles (K-major [v][k]), then D -= S~hi^T W lo^T; the record tiles
// [W^T hi | Q^T] and W^T lo are read MN-major.
__device__ __forceinline__ void state_product1(uint32_t tmem, uint32_t dq_col, const unsigned char *st_hi,
                                               const unsigned char *st_lo, const unsigned char *wq_hi,
                                               const unsigned char *w_lo, unsigned long long *bar)
{
    const uint32_t ID_WQ = tc::idesc_bf16_f32(128, WQ_COLS, true, false, true);  // negated; B MN-major
    const uint32_t ID_W = tc::idesc_bf16_f32(128, C, true, false, true);
    mma_tiles_bmn(tmem + dq_col, st_hi, K, wq_hi, WQ_COLS, K / 16, ID_WQ, false);
    mma_tiles_bmn(tmem + dq_col, st_lo, K, wq_hi, WQ_COLS, K / 16, ID_WQ, true);
    mma_tiles_bmn(tmem + dq_col, st_hi, K, w_lo, C, K / 16, ID_W, true);
    tc::mma_commit(bar);
}

// Product 2 of a piece, issued by one thread and committed to `bar`:
// [S~^T | O2] += Delta~^T [K' | P^T] (N = 192, from column s_col) for the split
// pairs (hi, hi), (hi, lo), (lo, hi); the [K' | P^T] tiles ([i][k | j]) are
// read MN-major.
__device__ __forceinline__ void state_product2(uint32_t tmem, uint32_t s_col, const unsigned char *dt_hi,
                                               const unsigned char *dt_lo, const unsigned char *kp_hi,
                                               const unsigned char *kp_lo, unsigned long long *bar)
{
    const uint32_t ID = tc::idesc_bf16_f32(128, KP_COLS, false, false, true);  // B MN-major
    mma_tiles_bmn(tmem + s_col, dt_hi, C, kp_hi, KP_COLS, C / 16, ID, true);
    mma_tiles_bmn(tmem + s_col, dt_hi, C, kp_lo, KP_COLS, C / 16, ID, true);
    mma_tiles_bmn(tmem + s_col, dt_lo, C, kp_hi, KP_COLS, C / 16, ID, true);
    tc::mma_commit(bar);
}
struct StSmem {
    alignas(1024) unsigned char st[2][128 * 128 * 2];   // S~^T hi / lo [v][k]
    alignas(1024) unsigned char rec_a[REC_A_BYTES];     // [W^T hi | Q^T], W^T lo of the piece (record bytes 0 .. 49151)
    alignas(1024) unsigned char rec_b[REC_B_BYTES];     // [K' | P^T] hi, lo (record bytes 49152 .. 98303)
    alignas(1024) unsigned char dt[2][128 * 64 * 2];    // Delta~^T hi / lo [v][i]
    alignas(16) float rec_s[REC_S_BYTES / 4];           // fo, gamma of the piece (record tail)
    float fo[2][C];                                     // fo of the last two pieces (by piece parity)
    // bar_d: -S~^T [W; Q]^T done; bar_s: S~^T += Delta~^T [K'; P]^T done;
    // bar_a / bar_b / bar_r: the bulk copies of a piece's W / Q, K' / P and
    // fo / gamma; bar_x: the copy of the state at the start
    unsigned long long bar_d, bar_s, bar_a, bar_b, bar_r, bar_x;
    uint32_t tmem_base;
    int failed;
};

// state kernel: ST_PARTS threads per TMEM lane, each handling 1 / ST_PARTS of
// the columns of every per-thread phase (the workers), plus one warp whose
// first thread issues the products and the bulk copies, so that issuing the
// first product does not hold back a worker warp's output stores
constexpr int ST_PARTS = 4;
constexpr int ST_WORKERS = 128 * ST_PARTS;
constexpr int ST_THREADS = ST_WORKERS + 32;
constexpr int ST_ISSUER = ST_WORKERS;
constexpr uint32_t ST_TMEM_COLS = 512;
// TMEM columns.  Product 2 writes [S~^T | O2] (192 columns) in one MMA,
// product 1 [D | O1] (128) in one MMA; [D | O1] is double-buffered by piece
// parity so that a piece's O1 can be read during the next piece.
constexpr uint32_t ST_COL_S = 0;      // S~^T              [v][k]   128 columns
constexpr uint32_t ST_COL_O2 = 128;   // Delta~^T P^T      [v][j]    64
constexpr uint32_t ST_COL_DQ = 256;   // -S~^T W^T (64), then -S~^T Q^T (64); 2 x 128 by piece parity

// The state is kept as S = cs * S~ for a per-CTA scale cs, so a piece's
// decay e^gamma_last multiplies cs instead of the 16 K state elements in
// TMEM: with cs' = cs e^gamma_last the update is S~ += Delta~^T K'^T where
// Delta~ = Delta / cs'.  When cs' leaves [2^-60, 2^60] the TMEM state is
// rescaled once (S~ <- cs' S~) and cs returns to 1.
__global__ void __launch_bounds__(ST_THREADS, 1) gdn_chunk_state_kernel(const __grid_constant__ DecodeParams p,
                                                                       const unsigned char *__restrict__ ws)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    StSmem &sm = *reinterpret_cast<StSmem *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    // worker thread (v, part): TMEM lane v = state column v; `part` picks
    // which 1 / ST_PARTS of the columns of each per-thread phase it handles
    const int v = tid & 127, part = tid >> 7;
    const bool worker = tid < ST_WORKERS;
    const int i = blockIdx.x / p.HV;
    const int hv = blockIdx.x - i * p.HV;
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
        if (worker)
            for (int t = part; t < len; t += ST_PARTS)
                out[(bos + t) * p.o_tok + hv * p.o_head + v] = __float2bfloat16_rn(0.f);
        return;
    }
    if (len == 0)
        return;
    const int64_t eos = bos + len;
    float *const s_gmem = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head;
    auto rec_of = [&](int64_t b) { return ws + (b * p.HV + hv) * static_cast<int64_t>(REC_BYTES); };

    // ---- set-up: barriers, TMEM, the first piece's tiles in flight, the
    // state into TMEM and into the S~^T tiles (cs = 1) ----------------------
    int64_t blk = bos / C;
    if (tid == ST_ISSUER) {
        sync::mbar_init(&sm.bar_d, 1);
        sync::mbar_init(&sm.bar_s, 1);
        sync::mbar_init(&sm.bar_a, 1);
        sync::mbar_init(&sm.bar_b, 1);
        sync::mbar_init(&sm.bar_r, 1);
        sync::mbar_init(&sm.bar_x, 1);
        sm.failed = 0;
        sync::fence_barrier_init();
        // the state S [k][v] (64 KB, contiguous) into the state-tile region in
        // one bulk copy, beside the first piece's records
        sync::mbar_arrive_expect_state_tx(&sm.bar_x, K * V * 4);
        sync::bulk_load(sm.st, s_gmem, K * V * 4, &sm.bar_x);
        const unsigned char *r = rec_of(blk);
        sync::mbar_arrive_expect_tx(&sm.bar_a, REC_A_BYTES);
        sync::bulk_load(sm.rec_a, r, REC_A_BYTES, &sm.bar_a);
        sync::mbar_arrive_expect_tx(&sm.bar_b, REC_B_BYTES);
        sync::bulk_load(sm.rec_b, r + REC_KP_HI, REC_B_BYTES, &sm.bar_b);
        sync::mbar_arrive_expect_tx(&sm.bar_r, REC_S_BYTES);
        sync::bulk_load(sm.rec_s, r + REC_FO, REC_S_BYTES, &sm.bar_r);
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, ST_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, (warp & 3) * 32, 0);
    constexpr int KP = K / ST_PARTS, CP = C / ST_PARTS;   // columns per part: of S~^T, of the tokens
    const int kh = KP * part;                   // this thread's k columns of S~^T

    uint32_t ph_d = 0, ph_s = 0, ph_a = 0, ph_b = 0, ph_r = 0, ph_x = 0;
    // copies issued and not yet waited for, with the parity their wait checks
    bool ok = true, pend_a = true, pend_b = true, pend_r = true, pend_x = true;
    uint32_t pa = 0, pb = 0, pr = 0;
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

    // column v of S (this thread's rows k) from the copied state into
    // registers; once every thread holds its part, into TMEM (lane v of
    // S~^T) and the S~^T hi / lo tiles over the same region
    wait_bar(&sm.bar_x, ph_x);
    if (ok) {
        pend_x = false;
        const float *raw = reinterpret_cast<const float *>(sm.st);
        float x[KP];
        if (worker) {
#pragma unroll
            for (int kk = 0; kk < KP; ++kk)
                x[kk] = raw[(kh + kk) * V + v];
        }
        __syncthreads();
        if (worker) {
#pragma unroll
            for (int c = 0; c < KP; c += 16) {
                tc::tmem_st16(my_lane + ST_COL_S + kh + c, x + c);
                st_row8_hilo(sm.st[0], sm.st[1], v, kh + c, K, x + c);
                st_row8_hilo(sm.st[0], sm.st[1], v, kh + c + 8, K, x + c + 8);
            }
            tc::tmem_wait_st();
        }
    }
    auto publish_smem = [&]() {
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    publish_smem();

    const unsigned char *wq_hi = sm.rec_a + REC_WQ_HI, *w_lo = sm.rec_a + REC_W_LO;
    const unsigned char *kp_hi = sm.rec_b, *kp_lo = sm.rec_b + (REC_KP_LO - REC_KP_HI);

    // Outputs of a piece are written during the next piece (while its first
    // products run); these describe the piece whose outputs are pending.
    int64_t out_base = 0;
    int out_r0 = 0, out_r1 = 0, out_buf = 0;
    float out_cs = 0.f, out_cs_new = 0.f;
    bool out_pending = false;
    auto write_outputs = [&]() {
        const uint32_t o1c = ST_COL_DQ + 128u * out_buf + 64u, o2c = ST_COL_O2;
#pragma unroll
        for (int cl = 0; cl < CP && worker; cl += 16) {
            const int cb = CP * part + cl;
            float o1[16], o2[16];
            tc::tmem_ld16(my_lane + o1c + cb, o1);
            tc::tmem_ld16(my_lane + o2c + cb, o2);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = cb + e;
                if (j >= out_r0 && j < out_r1)
                    out[(out_base + j) * p.o_tok + hv * p.o_head + v] =
                        __float2bfloat16_rn(fmaf(-sm.fo[out_buf][j] * out_cs, o1[e], out_cs_new * o2[e]));
            }
        }
        out_pending = false;
    };

    float cs = 1.f;
    int buf = 0;
    for (int64_t t = bos; t < eos && ok; ++blk, buf ^= 1) {
        const int64_t base = blk * C;
        const int r0 = static_cast<int>(t - base);
        const int r1 = static_cast<int>((eos < base + C ? eos : base + C) - base);
        const bool more = base + r1 < eos;
        const unsigned char *rec = rec_of(blk);

        // this thread's part of the row of U^T (needed after the first product)
        const int ih = CP * part;                 // this thread's token columns
        float u[CP];
        if (worker) {
            const float4 *src = reinterpret_cast<const float4 *>(rec + REC_UT) + v * 16 + ih / 4;
#pragma unroll
            for (int m = 0; m < CP / 4; ++m) {
                const float4 x = __ldg(src + m);
                u[4 * m] = x.x;
                u[4 * m + 1] = x.y;
                u[4 * m + 2] = x.z;
                u[4 * m + 3] = x.w;
            }
        }

        // ---- product 1: [D | O1] = -S~^T [W hi; Q]^T (hi and lo parts of S~)
        // and D -= S~hi^T W lo^T (bar_d) -------------------------------------
        wait_bar(&sm.bar_a, ph_a);
        if (!ok)
            break;
        pend_a = false;
        const uint32_t dq = ST_COL_DQ + 128u * buf;
        if (tid == ST_ISSUER)
            state_product1(tmem, dq, sm.st[0], sm.st[1], wq_hi, w_lo, &sm.bar_d);
        // the previous piece's outputs, while these products run
        if (out_pending)
            write_outputs();

        // ---- Delta~^T (thread = v) into its hi / lo tiles -----------------
        wait_bar(&sm.bar_d, ph_d);
        if (!ok)
            break;
        if (more && tid == ST_ISSUER) {     // W and Q of the next piece, into the buffer just read
            sync::mbar_arrive_expect_tx(&sm.bar_a, REC_A_BYTES);
            sync::bulk_load(sm.rec_a, rec_of(blk + 1), REC_A_BYTES, &sm.bar_a);
        }
        pend_a = more;
        pa = ph_a;
        wait_bar(&sm.bar_r, ph_r);
        if (!ok)
            break;
        pend_r = false;
        wait_bar(&sm.bar_b, ph_b);            // K' and P of this piece
        if (!ok)
            break;
        pend_b = false;
        const float decay = expf(sm.rec_s[C + r1 - 1]);    // e^gamma at the piece's last row
        const float cn = cs * decay;
        const bool rescale = !(cn >= 0x1p-60f && cn <= 0x1p60f);
        const float dscale = rescale ? 1.f : __fdividef(1.f, cn);
        if (tid < C)
            sm.fo[buf][tid] = sm.rec_s[tid];
#pragma unroll
        for (int cl = 0; cl < CP && worker; cl += 16) {
            const int cb = ih + cl;
            float d[16];
            tc::tmem_ld16(my_lane + dq + cb, d);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int ii = cb + e;
                d[e] = (ii >= r0 && ii < r1) ? fmaf(cs, d[e], u[cl + e]) * dscale : 0.f;
            }
            st_row8_hilo(sm.dt[0], sm.dt[1], v, cb, C, d);
            st_row8_hilo(sm.dt[0], sm.dt[1], v, cb + 8, C, d + 8);
        }
        {                            // O2 accumulates from zero in product 2
            float z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                z[e] = 0.f;
#pragma unroll
            for (int cl = 0; cl < CP && worker; cl += 16)
                tc::tmem_st16(my_lane + ST_COL_O2 + ih + cl, z);
        }
        if (rescale && worker) {     // S~ <- cs' S~ in TMEM; the scale returns to 1
#pragma unroll 1
            for (int k0 = kh; k0 < kh + KP; k0 += 16) {
                float x[16];
                tc::tmem_ld16(my_lane + ST_COL_S + k0, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] *= cn;
                tc::tmem_st16(my_lane + ST_COL_S + k0, x);
            }
            tc::tmem_wait_st();
        }
        const float cs_new = rescale ? 1.f : cn;
        tc::tmem_wait_st();
        publish_smem();

        // ---- product 2: [S~^T | O2] += Delta~^T [K' | P^T] (3 split products;
        // bar_s) ------------------------------------------------------------
        if (tid == ST_ISSUER) {
            state_product2(tmem, ST_COL_S, sm.dt[0], sm.dt[1], kp_hi, kp_lo, &sm.bar_s);
            if (more) {              // fo / gamma of the next piece (read above)
                sync::mbar_arrive_expect_tx(&sm.bar_r, REC_S_BYTES);
                sync::bulk_load(sm.rec_s, rec_of(blk + 1) + REC_FO, REC_S_BYTES, &sm.bar_r);
            }
        }
        pend_r = more;
        pr = ph_r;

        // K' and P of the next piece once both products that read them are done
        wait_bar(&sm.bar_s, ph_s);
        if (!ok)
            break;
        if (more && tid == ST_ISSUER) {
            sync::mbar_arrive_expect_tx(&sm.bar_b, REC_B_BYTES);
            sync::bulk_load(sm.rec_b, rec_of(blk + 1) + REC_KP_HI, REC_B_BYTES, &sm.bar_b);
        }
        pend_b = more;
        pb = ph_b;
        out_base = base;
        out_r0 = r0;
        out_r1 = r1;
        out_buf = buf;
        out_cs = cs;
        out_cs_new = cs_new;
        out_pending = true;

        // ---- the next piece's S~^T tiles, or the final write-back -----------
        for (int k0 = kh; k0 < kh + KP && worker; k0 += 16) {
            float x[16];
            tc::tmem_ld16(my_lane + ST_COL_S + k0, x);
            tc::tmem_wait_ld();
            if (more) {
                st_row8_hilo(sm.st[0], sm.st[1], v, k0, K, x);
                st_row8_hilo(sm.st[0], sm.st[1], v, k0 + 8, K, x + 8);
            } else if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    __stcs(s_gmem + (k0 + e) * V + v, cs_new * x[e]);
            }
        }
        cs = cs_new;
        t = base + r1;
        publish_smem();
    }
    if (ok && out_pending)
        write_outputs();

    // a failed wait left copies in flight: let them land (bounded) before the
    // shared memory is released
    if (pend_a || pend_b || pend_r || pend_x) {
        volatile int never = 0;
        if (pend_a)
            sync::mbar_wait(&sm.bar_a, pa, &never);
        if (pend_b)
            sync::mbar_wait(&sm.bar_b, pb, &never);
        if (pend_r)
            sync::mbar_wait(&sm.bar_r, pr, &never);
        if (pend_x)
            sync::mbar_wait(&sm.bar_x, 0, &never);
    }

    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, ST_TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Kernel 2, compact form: the same recurrence in 113 KB of shared memory and
// 256 TMEM columns, so that two CTAs share an SM -- for calls with many
// (sequence, value head) pairs, where one CTA per SM leaves the state loads
// and the per-piece latencies exposed.  Differences from the kernel above:
// one 48 KB record buffer, loaded with W / Q for product 1 and then with
// K' / P for product 2; the Delta~ tiles overlay the state tiles (dead
// between the two products); D's TMEM columns take O2 in product 2; outputs
// are written at the end of their own piece; 256 threads (two per TMEM lane).
// ---------------------------------------------------------------------------
struct StSmemCompact {
    // S~^T hi / lo [v][k]; between product 1 and product 2 the first 32 KB
    // hold Delta~^T hi / lo [v][i]
    alignas(1024) unsigned char st[2][128 * 128 * 2];
    alignas(1024) unsigned char rec[REC_A_BYTES];        // [W^T hi | Q^T], W^T lo; then [K' | P^T] hi, lo
    alignas(16) float rec_s[REC_S_BYTES / 4];            // fo, gamma of the piece
    float fo[C];
    // products; copies of W / Q, K' / P, fo / gamma, and of the state at the start
    unsigned long long bar_m, bar_a, bar_b, bar_r, bar_x;
    uint32_t tmem_base;
    int failed;
};
static_assert(REC_A_BYTES == REC_B_BYTES, "one buffer holds either half of a record");

constexpr int SC_PARTS = 2;
constexpr int SC_THREADS = 128 * SC_PARTS;
constexpr uint32_t SC_TMEM_COLS = 256;
constexpr uint32_t SC_COL_S = 0;      // S~^T                         [v][k]   128 columns
constexpr uint32_t SC_COL_D = 128;    // -S~^T W^T; O2 in product 2   [v][i]    64
constexpr uint32_t SC_COL_O1 = 192;   // -S~^T Q^T                    [v][j]    64

__global__ void __launch_bounds__(SC_THREADS, 2) gdn_chunk_state_compact_kernel(const __grid_constant__ DecodeParams p,
                                                                               const unsigned char *__restrict__ ws)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    StSmemCompact &sm = *reinterpret_cast<StSmemCompact *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int v = tid & 127, part = tid >> 7;
    const int i = blockIdx.x / p.HV;
    const int hv = blockIdx.x - i * p.HV;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);

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
        for (int t = part; t < len; t += SC_PARTS)
            out[(bos + t) * p.o_tok + hv * p.o_head + v] = __float2bfloat16_rn(0.f);
        return;
    }
    if (len == 0)
        return;
    const int64_t eos = bos + len;
    float *const s_gmem = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head;
    auto rec_of = [&](int64_t b) { return ws + (b * p.HV + hv) * static_cast<int64_t>(REC_BYTES); };

    int64_t blk = bos / C;
    if (tid == 0) {
        sync::mbar_init(&sm.bar_m, 1);
        sync::mbar_init(&sm.bar_a, 1);
        sync::mbar_init(&sm.bar_b, 1);
        sync::mbar_init(&sm.bar_r, 1);
        sync::mbar_init(&sm.bar_x, 1);
        sm.failed = 0;
        sync::fence_barrier_init();
        // the state S [k][v] (64 KB, contiguous) into the state-tile region in
        // one bulk copy, beside the first piece's W / Q and fo / gamma
        sync::mbar_arrive_expect_state_tx(&sm.bar_x, K * V * 4);
        sync::bulk_load(sm.st, s_gmem, K * V * 4, &sm.bar_x);
        const unsigned char *r = rec_of(blk);
        sync::prefetch_l2(r + REC_UT, REC_FO - REC_UT);     // U^T of the first piece (read per thread)
        sync::mbar_arrive_expect_tx(&sm.bar_a, REC_A_BYTES);
        sync::bulk_load(sm.rec, r, REC_A_BYTES, &sm.bar_a);
        sync::mbar_arrive_expect_tx(&sm.bar_r, REC_S_BYTES);
        sync::bulk_load(sm.rec_s, r + REC_FO, REC_S_BYTES, &sm.bar_r);
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, SC_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, (warp & 3) * 32, 0);
    constexpr int KP = K / SC_PARTS, CP = C / SC_PARTS;
    const int kh = KP * part, ih = CP * part;

    uint32_t ph_m = 0, ph_a = 0, ph_b = 0, ph_r = 0, ph_x = 0;
    // copies issued and not yet waited for, with the parity their wait checks
    bool ok = true, pend_a = true, pend_b = false, pend_r = true, pend_x = true;
    uint32_t pa = 0, pb = 0, pr = 0;
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

    // column v of S (this thread's rows k) from the copied state into
    // registers; once every thread holds its part, into TMEM (lane v of
    // S~^T) and the S~^T hi / lo tiles over the same region
    wait_bar(&sm.bar_x, ph_x);
    if (ok) {
        pend_x = false;
        const float *raw = reinterpret_cast<const float *>(sm.st);
        float x[KP];
#pragma unroll
        for (int kk = 0; kk < KP; ++kk)
            x[kk] = raw[(kh + kk) * V + v];
        __syncthreads();
#pragma unroll
        for (int c = 0; c < KP; c += 16) {
            tc::tmem_st16(my_lane + SC_COL_S + kh + c, x + c);
            st_row8_hilo(sm.st[0], sm.st[1], v, kh + c, K, x + c);
            st_row8_hilo(sm.st[0], sm.st[1], v, kh + c + 8, K, x + c + 8);
        }
        tc::tmem_wait_st();
    }
    auto publish_smem = [&]() {
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    publish_smem();

    const unsigned char *wq_hi = sm.rec + REC_WQ_HI, *w_lo = sm.rec + REC_W_LO;
    const unsigned char *kp_hi = sm.rec, *kp_lo = sm.rec + (REC_KP_LO - REC_KP_HI);
    unsigned char *const dt_hi = sm.st[0], *const dt_lo = sm.st[0] + 128 * 64 * 2;

    float cs = 1.f;
    for (int64_t t = bos; t < eos && ok; ++blk) {
        const int64_t base = blk * C;
        const int r0 = static_cast<int>(t - base);
        const int r1 = static_cast<int>((eos < base + C ? eos : base + C) - base);
        const bool more = base + r1 < eos;
        const unsigned char *rec = rec_of(blk);
        if (more && tid == 0)           // the next piece's U^T, into L2 ahead of its per-thread reads
            sync::prefetch_l2(rec_of(blk + 1) + REC_UT, REC_FO - REC_UT);

        float u[CP];
        {
            const float4 *src = reinterpret_cast<const float4 *>(rec + REC_UT) + v * 16 + ih / 4;
#pragma unroll
            for (int m = 0; m < CP / 4; ++m) {
                const float4 x = __ldg(src + m);
                u[4 * m] = x.x;
                u[4 * m + 1] = x.y;
                u[4 * m + 2] = x.z;
                u[4 * m + 3] = x.w;
            }
        }

        // ---- product 1: [D | O1] = -S~^T [W hi; Q]^T, D -= S~hi^T W lo^T --
        wait_bar(&sm.bar_a, ph_a);
        if (!ok)
            break;
        pend_a = false;
        if (tid == 0)
            state_product1(tmem, SC_COL_D, sm.st[0], sm.st[1], wq_hi, w_lo, &sm.bar_m);
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;
        if (tid == 0) {               // K' and P of this piece into the buffer just read
            sync::mbar_arrive_expect_tx(&sm.bar_b, REC_B_BYTES);
            sync::bulk_load(sm.rec, rec + REC_KP_HI, REC_B_BYTES, &sm.bar_b);
        }
        pend_b = true;
        pb = ph_b;

        // ---- Delta~^T into its tiles (over the state tiles), D -> 0 --------
        wait_bar(&sm.bar_r, ph_r);
        if (!ok)
            break;
        pend_r = false;
        const float decay = expf(sm.rec_s[C + r1 - 1]);
        const float cn = cs * decay;
        const bool rescale = !(cn >= 0x1p-60f && cn <= 0x1p60f);
        const float dscale = rescale ? 1.f : __fdividef(1.f, cn);
        if (tid < C)
            sm.fo[tid] = sm.rec_s[tid];
#pragma unroll
        for (int cl = 0; cl < CP; cl += 16) {
            const int cb = ih + cl;
            float d[16];
            tc::tmem_ld16(my_lane + SC_COL_D + cb, d);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int ii = cb + e;
                d[e] = (ii >= r0 && ii < r1) ? fmaf(cs, d[e], u[cl + e]) * dscale : 0.f;
            }
            st_row8_hilo(dt_hi, dt_lo, v, cb, C, d);
            st_row8_hilo(dt_hi, dt_lo, v, cb + 8, C, d + 8);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                d[e] = 0.f;
            tc::tmem_st16(my_lane + SC_COL_D + cb, d);          // O2 accumulates from zero here
        }
        if (rescale) {
#pragma unroll 1
            for (int k0 = kh; k0 < kh + KP; k0 += 16) {
                float x[16];
                tc::tmem_ld16(my_lane + SC_COL_S + k0, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] *= cn;
                tc::tmem_st16(my_lane + SC_COL_S + k0, x);
            }
        }
        tc::tmem_wait_st();
        const float cs_new = rescale ? 1.f : cn;
        publish_smem();

        // ---- product 2: [S~^T | O2] += Delta~^T [K' | P^T] -----------------
        wait_bar(&sm.bar_b, ph_b);
        if (!ok)
            break;
        pend_b = false;
        if (tid == 0) {
            state_product2(tmem, SC_COL_S, dt_hi, dt_lo, kp_hi, kp_lo, &sm.bar_m);
            if (more) {
                sync::mbar_arrive_expect_tx(&sm.bar_r, REC_S_BYTES);
                sync::bulk_load(sm.rec_s, rec_of(blk + 1) + REC_FO, REC_S_BYTES, &sm.bar_r);
            }
        }
        pend_r = more;
        pr = ph_r;
        wait_bar(&sm.bar_m, ph_m);
        if (!ok)
            break;
        if (more && tid == 0) {       // W and Q of the next piece
            sync::mbar_arrive_expect_tx(&sm.bar_a, REC_A_BYTES);
            sync::bulk_load(sm.rec, rec_of(blk + 1), REC_A_BYTES, &sm.bar_a);
        }
        pend_a = more;
        pa = ph_a;

        // ---- outputs o_j = fo_j cs (S~0^T q_j) + cs' (Delta~^T P^T)_j --------
#pragma unroll
        for (int cl = 0; cl < CP; cl += 16) {
            const int cb = ih + cl;
            float o1[16], o2[16];
            tc::tmem_ld16(my_lane + SC_COL_O1 + cb, o1);
            tc::tmem_ld16(my_lane + SC_COL_D + cb, o2);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = cb + e;
                if (j >= r0 && j < r1)
                    out[(base + j) * p.o_tok + hv * p.o_head + v] =
                        __float2bfloat16_rn(fmaf(-sm.fo[j] * cs, o1[e], cs_new * o2[e]));
            }
        }

        // ---- the next piece's S~^T tiles (over the Delta~ tiles), or the
        // final write-back ----------------------------------------------------
        for (int k0 = kh; k0 < kh + KP; k0 += 16) {
            float x[16];
            tc::tmem_ld16(my_lane + SC_COL_S + k0, x);
            tc::tmem_wait_ld();
            if (more) {
                st_row8_hilo(sm.st[0], sm.st[1], v, k0, K, x);
                st_row8_hilo(sm.st[0], sm.st[1], v, k0 + 8, K, x + 8);
            } else if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    __stcs(s_gmem + (k0 + e) * V + v, cs_new * x[e]);
            }
        }
        cs = cs_new;
        t = base + r1;
        publish_smem();
    }

    if (pend_a || pend_b || pend_r || pend_x) {
        volatile int never = 0;
        if (pend_a)
            sync::mbar_wait(&sm.bar_a, pa, &never);
        if (pend_b)
            sync::mbar_wait(&sm.bar_b, pb, &never);
        if (pend_r)
            sync::mbar_wait(&sm.bar_r, pr, &never);
        if (pend_x)
            sync::mbar_wait(&sm.bar_x, 0, &never);
    }

    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, SC_TMEM_COLS);
}

}  // namespace split
}  // namespace gdn

// gdn_chunk_state_half.cuh -- the recurrence kernel of the split chunked
// schedule (GDN_SCHEDULE_CHUNKED_SPLIT) with each (sequence, value head)
// state divided between two CTAs by columns.
//
// The delta rule updates every column of the state on its own: with S the
// K x V state, S' = e^g (I - beta k k^T) S + beta k v^T acts on each column
// S[:, v] with the same matrix and adds beta v_v k to it, and an output
// column o_v reads only S[:, v].  In the chunk form (gdn_chunk_split.cuh:
// Delta = U - W S0, o = fo (Q S0) + P Delta, S' = e^gamma_last S0 + K'^T Delta)
// the columns v of Delta, S and o depend on nothing but the same columns of
// U and S0, so two CTAs can take state columns 0..63 and 64..127 of one
// (sequence, head) with no exchange.  With few, long sequences this doubles
// the CTAs on the sequential recurrence, and each one's per-piece work --
// the Delta tiles, the next piece's state tiles, the outputs -- halves.
//
// The products are taken transposed against the full-width kernel, so that
// every MMA keeps M = 128 with N = 64 (this CTA's columns): the record tiles,
// written as [k][i | j] and [i][k | j] operand images by the block kernel,
// are read as MN-major A operands, and the state and Delta~ tiles are the B
// operands.  Per piece:
//   product 1  [D | O1] = -[W hi; Q] [S~hi | S~lo]     (M = 128 rows i | j,
//              N = 128: the hi and lo column halves, summed when read) and
//              DL = -W lo S~hi (rows 64.. of its A operand run past W lo's
//              tile into the next one: lanes 64.. of DL are never read);
//   Delta~     rows i (TMEM lanes 0..63): (U + cs (D + DL)) / cs';
//   product 2a S~ += K'^T Delta~         (M = 128 rows k, 3 split products);
//   product 2b O2 = [.; P] Delta~        (its A operand starts 64 columns
//              into [K' | P^T], so lanes 64.. hold P Delta~; lanes 0.. are
//              never read);
//   outputs    rows j (TMEM lanes 64..127), during the next piece's product 1.
#pragma once

#include "gdn_chunk_split.cuh"

namespace gdn {
namespace split {

constexpr int SH_COLS = V / 2;                 // state columns per CTA
constexpr int SH_PARTS = 4;                    // worker threads per TMEM lane
constexpr int SH_WORKERS = 128 * SH_PARTS;
constexpr int SH_THREADS = SH_WORKERS + 32;    // + one issuer warp
constexpr int SH_ISSUER = SH_WORKERS;
constexpr int SH_CP = SH_COLS / SH_PARTS;      // 16 columns per worker thread
constexpr uint32_t SH_TMEM_COLS = 512;
constexpr uint32_t SH_COL_S = 0;               // S~             lanes k        64 columns
constexpr uint32_t SH_COL_DL = 64;             // -W lo S~hi     lanes i        64
constexpr uint32_t SH_COL_O2 = 128;            // P Delta~       lanes 64 + j   64
constexpr uint32_t SH_COL_DQ = 256;            // [D | O1], hi and lo halves: 128 per piece parity (2 x 128)

enum { SH_BAR_A, SH_BAR_B, SH_BAR_R, SH_BAR_D, SH_BAR_S, SH_BAR_O, SH_BAR_DR, SH_BAR_TR, SH_NBAR };

struct ShSmem {
    // [S~hi | S~lo] [k][v' | v'], the MN-major B operand of product 1 (32 KB:
    // 128 rows k, this CTA's 64 columns as hi parts, then as lo parts)
    alignas(1024) unsigned char st[128 * 128 * 2];
    alignas(1024) unsigned char rec_a[REC_A_BYTES];     // [W^T hi | Q^T], W^T lo of the piece
    alignas(1024) unsigned char rec_b[2][REC_B_BYTES];  // [K' | P^T] hi, lo by piece parity (follows rec_a)
    alignas(1024) unsigned char dt[2][C * SH_COLS * 2]; // Delta~ hi / lo [i][v'], MN-major B of product 2
    alignas(16) float ut[SH_COLS * C];                  // this CTA's rows of U^T [v'][i]
    alignas(16) float rec_s[REC_S_BYTES / 4];           // fo, gamma of the piece
    // mbarriers, by SH_BAR_*: the bulk copies of W / Q, K' / P and U / fo /
    // gamma; product 1, product 2a and product 2b done; every worker warp's
    // Delta~ tiles (and rescale), and its next state tiles, written
    unsigned long long bar[SH_NBAR];
    uint32_t tmem_base;
    int failed;
};
static_assert(offsetof(ShSmem, rec_b) == offsetof(ShSmem, rec_a) + REC_A_BYTES,
              "product 1's DL operand reads 1 KB past W lo into rec_b");

// One MN-major x MN-major product over SLICES 16-deep k-slices:
// D (+)= A B with A read from a [kdim][a_cols] tile (M = 128 consecutive
// columns from `a`) and B from a [kdim][b_cols] tile (N from the idesc).
// The descriptors of successive slices differ only in their start address
// field (address / 16, 14 bits: shared-memory addresses stay below 256 KB,
// so the additions never carry out of it).
template <uint32_t SLICES>
__device__ __forceinline__ void mma_mn_mn(uint32_t d, const unsigned char *a, uint32_t a_cols, const unsigned char *b,
                                          uint32_t b_cols, uint32_t idesc, bool accumulate)
{
    const uint32_t ak = (a_cols >> 3) * 128u, bk = (b_cols >> 3) * 128u;
    const uint64_t a0 = tc::mn_desc(tc::smem_u32(a), ak, 128u), b0 = tc::mn_desc(tc::smem_u32(b), bk, 128u);
#pragma unroll
    for (uint32_t s = 0; s < SLICES; ++s)
        tc::mma_bf16(d, a0 + s * ((2u * ak) >> 4), b0 + s * ((2u * bk) >> 4), idesc, (accumulate || s > 0) ? 1u : 0u);
}

// Worker thread (lane, part): TMEM lane 32 (warp % 4) + lane -- a state row k
// in the state phases, a token row i (lanes 0..63) or j (64..127) in the
// Delta and output phases -- and columns SH_CP part .. + SH_CP of this CTA's
// 64, with part = warp / 4.  Warps whose lanes are 0..63 form Delta~; the
// others write the previous piece's outputs meanwhile.
__global__ void __launch_bounds__(SH_THREADS, 1) gdn_chunk_state_half_kernel(const __grid_constant__ DecodeParams p,
                                                                             const unsigned char *__restrict__ ws)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    ShSmem &sm = *reinterpret_cast<ShSmem *>(smem_raw);

    pdl_prologue();

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const bool worker = tid < SH_WORKERS;
    const int row = (warp & 3) * 32 + (tid & 31);       // TMEM lane
    const int cb = SH_CP * (warp >> 2);                   // first of this thread's columns
    const bool out_warp = worker && (warp & 3) >= 2;
    const int pair = blockIdx.x >> 1, half = blockIdx.x & 1;
    const int i = pair / p.HV;
    const int hv = pair - i * p.HV;
    const int v0 = SH_COLS * half;                        // this CTA's state columns v0 .. v0 + 63
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);

    // ---- token range and slot (uniform over the CTA) -----------------
    int64_t bos;
    int len;
    if (p.cu_seqlens) {
        const int b0 = __ldg(p.cu_seqlens + i);
        const int e0 = __ldg(p.cu_seqlens + i + 1);
        if (b0 < 0 || e0 < b0 || e0 > p.T_tot) {
            if (tid == 0 && hv == 0 && half == 0)
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
        if (tid == 0 && hv == 0 && half == 0)
            report(p.status, GDN_DEV_BAD_SLOT);
        return;
    }
    if (slot < 0) {
        if (worker)
            for (int t = tid >> 6; t < len; t += SH_WORKERS / SH_COLS)
                out[(bos + t) * p.o_tok + hv * p.o_head + v0 + (tid & 63)] = __float2bfloat16_rn(0.f);
        return;
    }
    if (len == 0)
        return;
    const int64_t eos = bos + len;
    float *const s_gmem = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head;
    auto rec_of = [&](int64_t b) { return ws + (b * p.HV + hv) * static_cast<int64_t>(REC_BYTES); };
    const uint32_t UT_BYTES = SH_COLS * C * 4;
    const int64_t ut_off = REC_UT + static_cast<int64_t>(half) * UT_BYTES;
    // the parts of block b's record this CTA reads, into L2 ahead of their copies
    auto prefetch_piece = [&](int64_t b) {
        const unsigned char *r = rec_of(b);
        sync::prefetch_l2(r, REC_A_BYTES + REC_B_BYTES);
        sync::prefetch_l2(r + ut_off, UT_BYTES);
        sync::prefetch_l2(r + REC_FO, REC_S_BYTES);
    };

    // ---- set-up: barriers, TMEM, the first piece's copies in flight, this
    // thread's state row part into registers -----------------------------
    int64_t blk = bos / C;
    if (tid == SH_ISSUER) {
        for (int m = 0; m < SH_NBAR; ++m)
            sync::mbar_init(&sm.bar[m], m == SH_BAR_DR || m == SH_BAR_TR ? SH_WORKERS / 32 : 1);
        sm.failed = 0;
        sync::fence_barrier_init();
        const unsigned char *r = rec_of(blk);
        sync::mbar_arrive_expect_tx(&sm.bar[SH_BAR_A], REC_A_BYTES);
        sync::bulk_load(sm.rec_a, r, REC_A_BYTES, &sm.bar[SH_BAR_A]);
        sync::mbar_arrive_expect_tx(&sm.bar[SH_BAR_B], REC_B_BYTES);
        sync::bulk_load(sm.rec_b[0], r + REC_KP_HI, REC_B_BYTES, &sm.bar[SH_BAR_B]);
        // the first piece's U / fo / gamma: the wait every worker makes first
        // (the test copy of the library withholds this arrival)
        sync::mbar_arrive_expect_state_tx(&sm.bar[SH_BAR_R], UT_BYTES + REC_S_BYTES);
        sync::bulk_load(sm.ut, r + ut_off, UT_BYTES, &sm.bar[SH_BAR_R]);
        sync::bulk_load(sm.rec_s, r + REC_FO, REC_S_BYTES, &sm.bar[SH_BAR_R]);
        if ((blk + 1) * C < bos + len)
            prefetch_piece(blk + 1);
    }
    float x[SH_CP];
    if (worker) {
        const float4 *src = reinterpret_cast<const float4 *>(s_gmem + static_cast<int64_t>(row) * V + v0 + cb);
#pragma unroll
        for (int m = 0; m < SH_CP / 4; ++m) {
            const float4 f = __ldcs(src + m);
            x[4 * m] = f.x;
            x[4 * m + 1] = f.y;
            x[4 * m + 2] = f.z;
            x[4 * m + 3] = f.w;
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, SH_TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t my_lane = tc::tmem_addr(tmem, (warp & 3) * 32, 0);
    // Barrier m (B_*): bit m of `phase` is the parity this thread waits for
    // next.  The issuer also records, per copy / product barrier, whether it
    // has used it (bit m of `used`) and the parity of its last phase (bit m
    // of `last`), for the drain after a failure.
    enum { B_A = SH_BAR_A, B_B = SH_BAR_B, B_R = SH_BAR_R, B_D = SH_BAR_D, B_S = SH_BAR_S, B_O = SH_BAR_O,
           B_DR = SH_BAR_DR, B_TR = SH_BAR_TR };
    uint32_t phase = 0, used = (1u << B_A) | (1u << B_B) | (1u << B_R), last = 0;
    auto wait_one = [&](int m) {          // bounded, this thread only
        const bool w = sync::mbar_wait(&sm.bar[m], (phase >> m) & 1u, &sm.failed);
        phase ^= 1u << m;
        if (!w) {
            sm.failed = 1;
            report(p.status, GDN_DEV_TIMEOUT);
        }
        tc::fence_after_sync();
        return w;
    };
    auto note = [&](int m) {              // issuer: one more phase of barrier m used
        last ^= (used >> m) & 1u ? 1u << m : 0u;
        used |= 1u << m;
    };
    // a worker warp's shared-memory tiles and TMEM stores, handed to the issuer
    auto arrive = [&](int m) {
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if ((tid & 31) == 0)
            sync::mbar_arrive(&sm.bar[m]);
    };
    bool mine = true;
    if (worker) {          // S~ = S (cs = 1) into TMEM and the hi / lo tiles
        tc::tmem_st16(my_lane + SH_COL_S + cb, x);
        st_row8_hilo(sm.st, sm.st + 1024, row, cb, 2 * SH_COLS, x);
        st_row8_hilo(sm.st, sm.st + 1024, row, cb + 8, 2 * SH_COLS, x + 8);
        tc::tmem_wait_st();
        arrive(B_TR);
    }

    // A piece's outputs (rows j, lanes 64..127) are written while the next
    // piece's product 1 runs, or after the last piece: rows of block o_blk,
    // from [D | O1] buffer obuf, with fo_j, and the scales before (ocs) and
    // after (ocs_new) the piece.
    auto write_outputs = [&](int64_t o_blk, int obuf, float fo_j, float ocs, float ocs_new) {
        const bool w = wait_one(B_O);         // product 2b of that piece
        if (w) {
            const int64_t obase = o_blk * C;
            const int out_r0 = static_cast<int>((bos > obase ? bos : obase) - obase);
            const int out_r1 = static_cast<int>((eos < obase + C ? eos : obase + C) - obase);
            const uint32_t dq = SH_COL_DQ + 128u * obuf;
            float oh[SH_CP], ol[SH_CP], o2[SH_CP];
            tc::tmem_ld16(my_lane + dq + cb, oh);
            tc::tmem_ld16(my_lane + dq + SH_COLS + cb, ol);
            tc::tmem_ld16(my_lane + SH_COL_O2 + cb, o2);
            tc::tmem_wait_ld();
            const int j = row - C;
            if (j >= out_r0 && j < out_r1) {
                const float f1 = -fo_j * ocs;
                uint32_t pk[SH_CP / 2];
#pragma unroll
                for (int e = 0; e < SH_CP; e += 2) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(fmaf(f1, oh[e] + ol[e], ocs_new * o2[e]),
                                                                   fmaf(f1, oh[e + 1] + ol[e + 1], ocs_new * o2[e + 1]));
                    pk[e / 2] = *reinterpret_cast<const uint32_t *>(&h);
                }
                uint2 *dst = reinterpret_cast<uint2 *>(out + (obase + j) * p.o_tok + hv * p.o_head + v0 + cb);
#pragma unroll
                for (int m = 0; m < SH_CP / 4; ++m)
                    dst[m] = make_uint2(pk[2 * m], pk[2 * m + 1]);
            }
        }
        return w;
    };

    // The loop runs without CTA-wide barriers: workers hand their tiles to
    // the issuer through bar_dr / bar_tr, the issuer hands products back
    // through bar_d / bar_s / bar_o; a thread whose wait fails (or that sees
    // another one's failure) leaves the loop.
    float cs = 1.f, prev_cs = 1.f;       // the scale before this piece and before the last one
    float fo_j = 0.f;                    // output rows: fo of the piece whose outputs are pending
    int buf = 0;
    for (int64_t t = bos; t < eos; ++blk, buf ^= 1) {
        const int64_t base = blk * C;
        const int r0 = static_cast<int>(t - base);
        const int r1 = static_cast<int>((eos < base + C ? eos : base + C) - base);
        const bool more = base + r1 < eos;
        const uint32_t dq = SH_COL_DQ + 128u * buf;

        if (tid == SH_ISSUER) {
            // ---- product 1 (bar_d) once this piece's state tiles and W / Q are in
            mine = wait_one(B_TR) && wait_one(B_A);
            if (!mine)
                break;
            const uint32_t ID_DQ = tc::idesc_bf16_f32(128, 2 * SH_COLS, true, true, true);
            const uint32_t ID_DL = tc::idesc_bf16_f32(128, SH_COLS, true, true, true);
            mma_mn_mn<K / 16>(tmem + dq, sm.rec_a + REC_WQ_HI, WQ_COLS, sm.st, 2 * SH_COLS, ID_DQ, false);
            mma_mn_mn<K / 16>(tmem + SH_COL_DL, sm.rec_a + REC_W_LO, C, sm.st, 2 * SH_COLS, ID_DL, false);
            tc::mma_commit(&sm.bar[SH_BAR_D]);
            note(B_D);

            // ---- product 2a: S~ += K'^T Delta~ (bar_s); 2b: O2 = P Delta~
            // (bar_o), once every worker's Delta~ tiles and rescale are in
            mine = wait_one(B_DR) && wait_one(B_B);
            if (!mine)
                break;
            if (more) {
                // the next piece's copies, ahead of this piece's product 2:
                // product 1 is done and U / fo / gamma were read (both before
                // every worker's arrival on bar_dr); the other K' / P buffer was
                // last read by the previous piece's product 2b, issued before
                // this piece's product 1, whose completion bar_d reported; and
                // the piece after next into L2
                const unsigned char *rn = rec_of(blk + 1);
                sync::mbar_arrive_expect_tx(&sm.bar[SH_BAR_A], REC_A_BYTES);
                sync::bulk_load(sm.rec_a, rn, REC_A_BYTES, &sm.bar[SH_BAR_A]);
                sync::mbar_arrive_expect_tx(&sm.bar[SH_BAR_R], UT_BYTES + REC_S_BYTES);
                sync::bulk_load(sm.ut, rn + ut_off, UT_BYTES, &sm.bar[SH_BAR_R]);
                sync::bulk_load(sm.rec_s, rn + REC_FO, REC_S_BYTES, &sm.bar[SH_BAR_R]);
                sync::mbar_arrive_expect_tx(&sm.bar[SH_BAR_B], REC_B_BYTES);
                sync::bulk_load(sm.rec_b[buf ^ 1], rn + REC_KP_HI, REC_B_BYTES, &sm.bar[SH_BAR_B]);
                note(B_A);
                note(B_R);
                note(B_B);
                if ((blk + 2) * C < eos)
                    prefetch_piece(blk + 2);
            }
            const uint32_t ID = tc::idesc_bf16_f32(128, SH_COLS, false, true, true);
            const unsigned char *kp_hi = sm.rec_b[buf], *kp_lo = sm.rec_b[buf] + (REC_KP_LO - REC_KP_HI);
            mma_mn_mn<C / 16>(tmem + SH_COL_S, kp_hi, KP_COLS, sm.dt[0], SH_COLS, ID, true);
            mma_mn_mn<C / 16>(tmem + SH_COL_S, kp_hi, KP_COLS, sm.dt[1], SH_COLS, ID, true);
            mma_mn_mn<C / 16>(tmem + SH_COL_S, kp_lo, KP_COLS, sm.dt[0], SH_COLS, ID, true);
            tc::mma_commit(&sm.bar[SH_BAR_S]);
            note(B_S);
            mma_mn_mn<C / 16>(tmem + SH_COL_O2, kp_hi + 1024, KP_COLS, sm.dt[0], SH_COLS, ID, false);
            mma_mn_mn<C / 16>(tmem + SH_COL_O2, kp_hi + 1024, KP_COLS, sm.dt[1], SH_COLS, ID, true);
            mma_mn_mn<C / 16>(tmem + SH_COL_O2, kp_lo + 1024, KP_COLS, sm.dt[0], SH_COLS, ID, true);
            tc::mma_commit(&sm.bar[SH_BAR_O]);
            note(B_O);
        } else if (worker) {
            // ---- the piece's decay and scale (every worker: the rescale is shared)
            mine = wait_one(B_R);
            if (!mine)
                break;
            const float cn = cs * expf(sm.rec_s[C + r1 - 1]);     // e^gamma at the piece's last row
            const bool rescale = !(cn >= 0x1p-60f && cn <= 0x1p60f);
            const float dscale = rescale ? 1.f : __fdividef(1.f, cn);
            const float cs_new = rescale ? 1.f : cn;
            if (out_warp) {
                if (t > bos && !(mine = write_outputs(blk - 1, buf ^ 1, fo_j, prev_cs, cs)))
                    break;
                fo_j = sm.rec_s[row - C];
            } else {
                // ---- Delta~ rows i (thread: row i, columns cb..) ------------
                if (!(mine = wait_one(B_D)))
                    break;
                float dh[SH_CP], dl[SH_CP], dw[SH_CP];
                tc::tmem_ld16(my_lane + dq + cb, dh);
                tc::tmem_ld16(my_lane + dq + SH_COLS + cb, dl);
                tc::tmem_ld16(my_lane + SH_COL_DL + cb, dw);
                tc::tmem_wait_ld();
                const bool live = row >= r0 && row < r1;
#pragma unroll
                for (int e = 0; e < SH_CP; ++e)
                    dh[e] = live ? fmaf(cs, (dh[e] + dl[e]) + dw[e], sm.ut[(cb + e) * C + row]) * dscale : 0.f;
                st_row8_hilo(sm.dt[0], sm.dt[1], row, cb, SH_COLS, dh);
                st_row8_hilo(sm.dt[0], sm.dt[1], row, cb + 8, SH_COLS, dh + 8);
            }
            if (rescale) {      // S~ <- cs' S~ in TMEM; the scale returns to 1
                float y[SH_CP];
                tc::tmem_ld16(my_lane + SH_COL_S + cb, y);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < SH_CP; ++e)
                    y[e] *= cn;
                tc::tmem_st16(my_lane + SH_COL_S + cb, y);
                tc::tmem_wait_st();
            }
            arrive(B_DR);

            // ---- the next piece's state tiles, or the final write-back ----
            if (!(mine = wait_one(B_S)))
                break;
            float y[SH_CP];
            tc::tmem_ld16(my_lane + SH_COL_S + cb, y);
            tc::tmem_wait_ld();
            if (more) {
                st_row8_hilo(sm.st, sm.st + 1024, row, cb, 2 * SH_COLS, y);
                st_row8_hilo(sm.st, sm.st + 1024, row, cb + 8, 2 * SH_COLS, y + 8);
                arrive(B_TR);
            } else if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
                float4 *dst = reinterpret_cast<float4 *>(s_gmem + static_cast<int64_t>(row) * V + v0 + cb);
#pragma unroll
                for (int m = 0; m < SH_CP / 4; ++m)
                    __stcs(dst + m, make_float4(cs_new * y[4 * m], cs_new * y[4 * m + 1], cs_new * y[4 * m + 2],
                                                cs_new * y[4 * m + 3]));
            }
            prev_cs = cs;
            cs = cs_new;
        }
        t = base + r1;
    }
    if (mine && out_warp)
        mine = write_outputs(blk - 1, buf ^ 1, fo_j, prev_cs, cs);
    const bool ok = __syncthreads_and(mine) != 0;

    // after a failed wait, copies or products may still be in flight: let
    // them finish (bounded) before the shared and tensor memory is released
    // (a phase that has completed returns at once)
    if (!ok && tid == SH_ISSUER) {
        volatile int never = 0;
#pragma unroll 1
        for (int m = 0; m < 6; ++m)
            if ((used >> m) & 1u)
                sync::mbar_wait(&sm.bar[m], (last >> m) & 1u, &never);
    }

    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, SH_TMEM_COLS);
}

}  // namespace split
}  // namespace gdn

// gdn_decode_pipelined.cuh -- persistent, bulk-copy-pipelined sm_100a kernel
// of the fused sigmoid-gating Gated DeltaNet decode update (operation in
// include/gdn_decode.h; same arithmetic as gdn_decode_kernel.cuh), for bf16
// activations and the fused sigmoid gating.
//
// One CTA per SM walks a static list of (sequence, value head) units: unit
// u = blockIdx.x + n * gridDim.x.  A unit's whole fp32 state S (K x V =
// 128 x 128, 64 KB) is contiguous in the pool, so it moves between HBM and
// shared memory as plain bulk async copies (cp.async.bulk, no tensor map,
// no multicast) issued by one producer thread:
//
//   stage ring: STAGES x 64 KB of shared memory, one `full` and one `done`
//   mbarrier per stage.
//   producer (warp CONSUMER_WARPS, lane 0):
//       prologue: load units 0..STAGES-1;
//       for each unit j: wait done[j % STAGES]; bulk-store the updated S back
//       to its slot; once the store has read the stage, bulk-load unit
//       j + STAGES into it.
//   consumers (CONSUMER_WARPS warps = 4 column groups of 128 threads):
//       wait full[s]; move the group's [128 x 32] columns into registers
//       (thread (kg, vq): rows kg*8..kg*8+7, columns 4*vq..4*vq+3 of the
//       group); run the sequence's tokens exactly as the per-tile kernel does
//       (one pass for S^T k, S^T q, |k|^2, |q|^2, k.q; xor-shuffles; one
//       shared-memory exchange per token behind a 128-thread named barrier);
//       write S back into the stage; fence.proxy.async; arrive on done[s].
//
// Loads for the next STAGES-1 units are in flight while a unit is computed,
// and stores drain asynchronously, so the bytes in flight per SM are set by
// shared memory, not by registers.  Every mbarrier wait is bounded (by the
// global timer); on a timeout the CTA sets GDN_DEV_TIMEOUT, stops issuing
// copies, skips all remaining stores and waits (bounded) for the copies it
// already issued before it exits.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn_decode.h"
#include "gdn_decode_kernel.cuh"
#include "mbarrier_sm100.cuh"

namespace gdn {
namespace pipe {

using namespace gdn::sync;

constexpr int K = 128;
constexpr int V = 128;
constexpr int GROUP_COLS = 32;                       // columns per consumer group
constexpr int GROUPS = V / GROUP_COLS;               // 4
constexpr int GROUP_THREADS = 128;                   // 8 (columns/4) x 16 (row groups of 8)
constexpr int CONSUMER_WARPS = GROUPS * GROUP_THREADS / 32;   // 16
constexpr int THREADS = (CONSUMER_WARPS + 1) * 32;  // + one producer warp
constexpr int R = 8;                                 // rows per consumer thread
constexpr int XW = 2 * GROUP_COLS + 4;               // exchange floats per warp
constexpr uint32_t TILE_BYTES = K * V * 4;           // 65536
constexpr int CHUNKS = 4;                            // bulk copies per tile
constexpr uint32_t CHUNK_BYTES = TILE_BYTES / CHUNKS;

template <int STAGES>
struct Smem {
    float tile[STAGES][K * V];
    float xch[GROUPS][2][GROUP_THREADS / 32][XW];
    unsigned long long full[STAGES];
    unsigned long long done[STAGES];
    int failed;
};

using sync::bulk_commit;
using sync::bulk_load;
using sync::bulk_store;
using sync::bulk_wait_all;
using sync::bulk_wait_read_all;
using sync::fence_proxy_async;

__device__ __forceinline__ void group_sync(int group)
{
    asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "n"(GROUP_THREADS) : "memory");
}

// Barrier over one consumer group that also ANDs a predicate across it, so
// every thread of the group takes the same branch afterwards.
__device__ __forceinline__ bool group_all(int group, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(group + 1), "n"(GROUP_THREADS)
        : "memory");
    return r != 0;
}

// What a unit needs: its token range and slot, or why it is skipped.
struct Unit {
    int64_t bos;
    int len;
    int slot;
    int hv;
    int kind;  // 0 active, 1 padded (zero output), 2 nothing to do, 3 invalid
};

__device__ __forceinline__ Unit classify(const DecodeParams &p, int unit)
{
    Unit u;
    const int i = unit / p.HV;
    u.hv = unit - i * p.HV;
    u.slot = -1;
    u.bos = 0;
    u.len = 0;
    if (p.cu_seqlens) {
        const int b0 = __ldg(p.cu_seqlens + i);
        const int e0 = __ldg(p.cu_seqlens + i + 1);
        if (b0 < 0 || e0 < b0 || e0 > p.T_tot) {
            u.kind = 3;
            u.slot = -2;  // marks a seqlens fault
            return u;
        }
        u.bos = b0;
        u.len = e0 - b0;
    } else {
        u.bos = static_cast<int64_t>(i) * p.T_fixed;
        u.len = p.T_fixed;
    }
    const int slot = __ldg(p.indices + i);
    u.slot = slot;
    if (slot < -1 || slot >= p.num_slots)
        u.kind = 3;
    else if (slot == -1)
        u.kind = 1;
    else if (u.len == 0)
        u.kind = 2;
    else
        u.kind = 0;
    return u;
}

template <int STAGES>
__global__ void __launch_bounds__(THREADS, 1) gdn_decode_pipelined_kernel(const __grid_constant__ DecodeParams p)
{
    pdl_prologue();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem<STAGES> &sm = *reinterpret_cast<Smem<STAGES> *>(smem_raw);
    volatile int *failed = &sm.failed;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int units = p.N * p.HV;
    const int n_mine = blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const bool write_back = !(p.flags & GDN_NO_FINAL_WRITEBACK);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.done[s], CONSUMER_WARPS);
        }
        sm.failed = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == CONSUMER_WARPS) {
        // ------------------------------------------------------------------
        // producer
        // ------------------------------------------------------------------
        if (lane != 0)
            return;
        auto state_ptr = [&](const Unit &u) {
            return p.state + static_cast<int64_t>(u.slot) * p.s_slot + static_cast<int64_t>(u.hv) * p.s_head;
        };
        auto issue = [&](int j) {
            const int s = j % STAGES;
            const Unit u = classify(p, blockIdx.x + j * gridDim.x);
            if (u.kind == 0 && !*failed) {
                sync::mbar_arrive_expect_state_tx(&sm.full[s], TILE_BYTES);
                const float *src = state_ptr(u);
#pragma unroll
                for (int c = 0; c < CHUNKS; ++c)
                    bulk_load(&sm.tile[s][c * (CHUNK_BYTES / 4)], src + c * (CHUNK_BYTES / 4), CHUNK_BYTES,
                              &sm.full[s]);
            } else {
                mbar_arrive(&sm.full[s]);
            }
        };
        const int pro = n_mine < STAGES ? n_mine : STAGES;
        for (int j = 0; j < pro; ++j)
            issue(j);
        int issued = pro;
        for (int j = 0; j < n_mine; ++j) {
            const int s = j % STAGES;
            if (!mbar_wait(&sm.done[s], (j / STAGES) & 1, failed)) {
                *failed = 1;
                report(p.status, GDN_DEV_TIMEOUT);
                break;
            }
            const Unit u = classify(p, blockIdx.x + j * gridDim.x);
            const bool store = u.kind == 0 && write_back && !*failed;
            if (store) {
                bulk_store(state_ptr(u), sm.tile[s], TILE_BYTES);
                bulk_commit();
            }
            if (j + STAGES < n_mine) {
                if (store)
                    bulk_wait_read_all();
                issue(j + STAGES);
                issued = j + STAGES + 1;
            }
        }
        // Loads still in flight (only after a failure) must land before exit;
        // only the last STAGES issued loads can still be in flight.
        if (*failed) {
            volatile int never = 0;
            for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
                mbar_wait(&sm.full[j % STAGES], (j / STAGES) & 1, &never);
        }
        pdl_trigger();
        bulk_wait_all();
        return;
    }

    // ----------------------------------------------------------------------
    // consumers: group g owns columns g*32 .. g*32+31 of every tile
    // ----------------------------------------------------------------------
    const int g = warp / (GROUP_THREADS / 32);
    const int gtid = tid - g * GROUP_THREADS;
    const int gwarp = gtid >> 5;
    const int vq = gtid & 7;
    const int kg = gtid >> 3;
    const int row0 = kg * R;
    const int col0 = g * GROUP_COLS + vq * 4;
    const bool l2norm = (p.flags & GDN_L2NORM_QK) != 0;
    const bool write_inter = (p.flags & GDN_WRITE_INTERMEDIATE) != 0;
    // This schedule takes bf16 activations and bf16 a, b (the host checks).
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *a = static_cast<const __nv_bfloat16 *>(p.a);
    const __nv_bfloat16 *b = static_cast<const __nv_bfloat16 *>(p.b);
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);

    uint32_t tcount = 0;  // tokens this group has processed: picks the exchange buffer
    for (int j = 0; j < n_mine; ++j) {
        const int s = j % STAGES;
        const Unit u = classify(p, blockIdx.x + j * gridDim.x);
        bool ok = mbar_wait(&sm.full[s], (j / STAGES) & 1, failed);
        if (!ok) {
            *failed = 1;
            report(p.status, GDN_DEV_TIMEOUT);
        }
        ok = group_all(g, ok && !*failed);
        if (u.kind == 3) {
            if (tid == 0)
                report(p.status, u.slot == -2 ? GDN_DEV_BAD_SEQLENS : GDN_DEV_BAD_SLOT);
        } else if (u.kind == 1) {
            if (kg == 0)
                for (int t = 0; t < u.len; ++t)
                    *reinterpret_cast<uint2 *>(out + (u.bos + t) * p.o_tok + u.hv * p.o_head + col0) =
                        make_uint2(0u, 0u);
        } else if (u.kind == 0 && ok) {
            float *tile = sm.tile[s];
            float4 st[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                st[r] = *reinterpret_cast<const float4 *>(tile + (row0 + r) * V + col0);

            const int h = u.hv / p.G;
            const float neg_A = -expf(__ldg(p.A_log + u.hv * p.A_stride));
            const float dt_b = __ldg(p.dt_bias + u.hv * p.dt_stride);
            for (int t = 0; t < u.len; ++t) {
                const int64_t tok = u.bos + t;
                float kr[R], qr[R];
                unpack8(__ldg(reinterpret_cast<const uint4 *>(k + tok * p.k_tok + h * p.k_head + row0)), kr);
                unpack8(__ldg(reinterpret_cast<const uint4 *>(q + tok * p.q_tok + h * p.q_head + row0)), qr);
                const uint2 v_raw =
                    __ldg(reinterpret_cast<const uint2 *>(v + tok * p.v_tok + u.hv * p.v_head + col0));
                const float a_t = load_bf16(a + tok * p.a_tok + u.hv * p.a_head);
                const float b_t = load_bf16(b + tok * p.b_tok + u.hv * p.b_head);

                float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
                float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f;
                float skk = 0.f, sqq = 0.f, skq = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    u0 = fmaf(st[r].x, kr[r], u0); u1 = fmaf(st[r].y, kr[r], u1);
                    u2 = fmaf(st[r].z, kr[r], u2); u3 = fmaf(st[r].w, kr[r], u3);
                    w0 = fmaf(st[r].x, qr[r], w0); w1 = fmaf(st[r].y, qr[r], w1);
                    w2 = fmaf(st[r].z, qr[r], w2); w3 = fmaf(st[r].w, qr[r], w3);
                    skk = fmaf(kr[r], kr[r], skk);
                    sqq = fmaf(qr[r], qr[r], sqq);
                    skq = fmaf(kr[r], qr[r], skq);
                }
#pragma unroll
                for (int off = 8; off < 32; off <<= 1) {
                    u0 += __shfl_xor_sync(0xffffffffu, u0, off); u1 += __shfl_xor_sync(0xffffffffu, u1, off);
                    u2 += __shfl_xor_sync(0xffffffffu, u2, off); u3 += __shfl_xor_sync(0xffffffffu, u3, off);
                    w0 += __shfl_xor_sync(0xffffffffu, w0, off); w1 += __shfl_xor_sync(0xffffffffu, w1, off);
                    w2 += __shfl_xor_sync(0xffffffffu, w2, off); w3 += __shfl_xor_sync(0xffffffffu, w3, off);
                    skk += __shfl_xor_sync(0xffffffffu, skk, off);
                    sqq += __shfl_xor_sync(0xffffffffu, sqq, off);
                    skq += __shfl_xor_sync(0xffffffffu, skq, off);
                }
                float *xb = sm.xch[g][tcount & 1][0];
                ++tcount;
                if (lane < 8) {
                    *reinterpret_cast<float4 *>(xb + gwarp * XW + vq * 4) = make_float4(u0, u1, u2, u3);
                    *reinterpret_cast<float4 *>(xb + gwarp * XW + GROUP_COLS + vq * 4) =
                        make_float4(w0, w1, w2, w3);
                    if (lane == 0) {
                        xb[gwarp * XW + 2 * GROUP_COLS + 0] = skk;
                        xb[gwarp * XW + 2 * GROUP_COLS + 1] = sqq;
                        xb[gwarp * XW + 2 * GROUP_COLS + 2] = skq;
                    }
                }
                group_sync(g);
                float4 U = make_float4(0.f, 0.f, 0.f, 0.f), W = U;
                float SKK = 0.f, SQQ = 0.f, SKQ = 0.f;
#pragma unroll
                for (int wi = 0; wi < GROUP_THREADS / 32; ++wi) {
                    const float4 uu = *reinterpret_cast<const float4 *>(xb + wi * XW + vq * 4);
                    const float4 ww = *reinterpret_cast<const float4 *>(xb + wi * XW + GROUP_COLS + vq * 4);
                    U.x += uu.x; U.y += uu.y; U.z += uu.z; U.w += uu.w;
                    W.x += ww.x; W.y += ww.y; W.z += ww.z; W.w += ww.w;
                    SKK += xb[wi * XW + 2 * GROUP_COLS + 0];
                    SQQ += xb[wi * XW + 2 * GROUP_COLS + 1];
                    SKQ += xb[wi * XW + 2 * GROUP_COLS + 2];
                }

                const float rk = l2norm ? rsqrtf(SKK + 1e-6f) : 1.f;
                const float qs = (l2norm ? rsqrtf(SQQ + 1e-6f) : 1.f) * p.scale;
                const float x = a_t + dt_b;
                const float sp = x > 20.f ? x : log1pf(expf(x));
                const float decay = expf(neg_A * sp);
                const float beta = 1.f / (1.f + expf(-b_t));
                const float kq = SKQ * rk * qs;
                const float dku = decay * rk;
                const float dwq = decay * qs;
                const float d0 = beta * (bf16_lo(v_raw.x) - dku * U.x);
                const float d1 = beta * (bf16_hi(v_raw.x) - dku * U.y);
                const float d2 = beta * (bf16_lo(v_raw.y) - dku * U.z);
                const float d3 = beta * (bf16_hi(v_raw.y) - dku * U.w);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float kh = kr[r] * rk;
                    st[r].x = fmaf(kh, d0, decay * st[r].x);
                    st[r].y = fmaf(kh, d1, decay * st[r].y);
                    st[r].z = fmaf(kh, d2, decay * st[r].z);
                    st[r].w = fmaf(kh, d3, decay * st[r].w);
                }
                if (kg == 0) {
                    const float o0 = fmaf(kq, d0, dwq * W.x);
                    const float o1 = fmaf(kq, d1, dwq * W.y);
                    const float o2 = fmaf(kq, d2, dwq * W.z);
                    const float o3 = fmaf(kq, d3, dwq * W.w);
                    *reinterpret_cast<uint2 *>(out + tok * p.o_tok + u.hv * p.o_head + col0) =
                        make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
                }
                if (write_inter) {
                    float *ip = p.inter + tok * p.i_tok + u.hv * p.i_head + static_cast<int64_t>(row0) * V + col0;
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        __stcs(reinterpret_cast<float4 *>(ip + r * V), st[r]);
                }
            }
            if (write_back) {
#pragma unroll
                for (int r = 0; r < R; ++r)
                    *reinterpret_cast<float4 *>(tile + (row0 + r) * V + col0) = st[r];
                fence_proxy_async();
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.done[s]);
    }
}

}  // namespace pipe
}  // namespace gdn

// gdn_decode_kernel.cuh -- sm_100a kernels of the Gated DeltaNet decode /
// speculative-decode state update (the operation is stated in
// include/gdn_decode.h): the per-tile update kernel and the gating kernel.
//
// Work decomposition.  One CTA owns one (sequence i, value head hv, V-tile)
// unit: a [K, BV] slab of the fp32 state S = pool[slot_i, hv].  The slab is
// split over the CTA's threads as a (KG x VG) grid: thread (kg, vq) holds
// rows kg*R .. kg*R+R-1 (R = K/KG) and the four columns vq*4 .. vq*4+3, i.e.
// R float4 registers.  Each warp-wide load touches whole row segments of
// 64-256 bytes, so the state moves with 128-bit, fully coalesced streaming
// loads and stores, once per sequence; the slab stays in registers across
// all tokens of the sequence (the speculative-decode path).
//
// Per token the two contractions over K that the update needs -- u = S^T k
// and w = S^T q on the state before this token -- are done in ONE pass over
// the registers, together with |k|^2, |q|^2 and k.q (for the rsqrt
// normalisation, which is a per-token scalar and therefore commutes with the
// sums).  Partial sums are reduced with xor-shuffles inside the warp and,
// for multi-warp tiles, one shared-memory exchange across warps (one
// __syncthreads per token, double-buffered by token parity).  Then, with
// decay = exp(g):
//     delta = beta * (v - decay * u * rk)                (S^T k^ on the decayed S)
//     o     = decay * w * qs + (k^ . q^) * delta         (= S'^T q^ after the update)
//     S'    = decay * S + k^ delta^T
// which is the update of the header rearranged so that S is read once.  The
// registers hold S / cs for a per-CTA scale cs that absorbs the decays, so
// the update costs one FMA per element (see the token loop).
//
// Template parameters: the activation element type TAct (q, k, v, out:
// bf16 or fp32) and GIVEN_GATES (false: decay and beta come from A_log, a,
// b, dt_bias -- the fused sigmoid gating; true: from per-token g and beta
// arrays -- the recurrence of the unfused pair).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn_decode.h"

namespace gdn {

struct DecodeParams {
    const void *q, *k, *v;      // TAct
    const void *a, *b;          // fused: a, b; given gates: g (fp32), beta
    const float *A_log, *dt_bias;
    float *state;
    const int32_t *indices;
    const int32_t *cu_seqlens;  // nullptr: fixed length T_fixed
    void *out;                  // TAct
    float *inter;               // nullptr unless GDN_WRITE_INTERMEDIATE
    uint32_t *status;           // nullptr: device errors are not reported
    // strides in elements
    int64_t q_tok, q_head, k_tok, k_head, v_tok, v_head;
    int64_t a_tok, a_head, b_tok, b_head, o_tok, o_head;
    int64_t A_stride, dt_stride;
    int64_t s_slot, s_head, i_tok, i_head;
    int32_t N, T_fixed, T_tot, HV, G, num_slots;
    int32_t a_f32, b_f32;       // element type of a / b (fused) or g / beta (given): 1 = fp32, 0 = bf16
    float scale;
    uint32_t flags;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 u, float *f)
{
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
    f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
    f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ float load_bf16(const __nv_bfloat16 *p)
{
    const unsigned short bits = __ldg(reinterpret_cast<const unsigned short *>(p));
    return __uint_as_float(static_cast<uint32_t>(bits) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

// A scalar gate input stored as fp32 or bf16: fetch its raw bits now, widen
// them when the value is needed (so the load stays in flight meanwhile).
__device__ __forceinline__ uint32_t gate_raw(const void *base, int64_t idx, int32_t is_f32)
{
    return is_f32 ? __ldg(static_cast<const unsigned int *>(base) + idx)
                  : static_cast<uint32_t>(__ldg(static_cast<const unsigned short *>(base) + idx));
}

__device__ __forceinline__ float gate_value(uint32_t raw, int32_t is_f32)
{
    return __uint_as_float(is_f32 ? raw : raw << 16);
}

// Element-type traits of the activations.
template <typename T>
struct Act;

template <>
struct Act<__nv_bfloat16> {
    static constexpr int PER16 = 8;   // elements per 16-byte load
    using Raw4 = uint2;               // four elements
    __device__ static void unpack16(const uint4 u, float *f) { unpack8(u, f); }
    __device__ static float4 unpack4(const uint2 r)
    {
        return make_float4(bf16_lo(r.x), bf16_hi(r.x), bf16_lo(r.y), bf16_hi(r.y));
    }
    __device__ static void store4(__nv_bfloat16 *p, float a, float b, float c, float d)
    {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
    }
};

template <>
struct Act<float> {
    static constexpr int PER16 = 4;
    using Raw4 = float4;
    __device__ static void unpack16(const uint4 u, float *f)
    {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    __device__ static float4 unpack4(const float4 r) { return r; }
    __device__ static void store4(float *p, float a, float b, float c, float d)
    {
        *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
    }
};

// Programmatic dependent launch.  pdl_prologue: wait until the previous
// kernel on the stream has completed (and its writes are visible) before
// touching any input.  pdl_trigger: this CTA's main work is done -- once
// every CTA of the grid has triggered or exited, the next kernel may be
// scheduled (it still waits for this grid to complete before it reads).
// Triggering late keeps the next grid's CTAs from occupying SM slots while
// this grid still needs them.  Both are no-ops when the grid was launched
// without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_prologue() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void report(uint32_t *status, uint32_t bit)
{
    if (status)
        atomicOr(status, bit);
}

template <int K, int V, int BV, int KG>
struct TileShape {
    static constexpr int VG = BV / 4;            // threads across the tile's columns
    static constexpr int THREADS = VG * KG;
    static constexpr int WARPS = THREADS / 32;
    static constexpr int R = K / KG;             // state rows per thread
    static constexpr int NV = V / BV;            // V-tiles per head
    static constexpr int XW = 2 * BV + 4;        // exchange floats per warp: u, w, |k|^2, |q|^2, k.q
    static_assert(BV % 4 == 0 && V % BV == 0, "V must split into BV-wide tiles");
    static_assert(VG <= 32 && 32 % VG == 0, "a warp must hold whole k-groups");
    static_assert(THREADS % 32 == 0 && THREADS <= 1024, "whole warps");
    static_assert(K % KG == 0 && R % 8 == 0, "q/k rows are loaded 16 bytes at a time");
};

template <int K, int V, int BV, int KG, typename TAct, bool GIVEN_GATES>
__global__ void __launch_bounds__(TileShape<K, V, BV, KG>::THREADS)
gdn_decode_kernel(const __grid_constant__ DecodeParams p)
{
    using TS = TileShape<K, V, BV, KG>;
    using A = Act<TAct>;
    constexpr int VG = TS::VG, WARPS = TS::WARPS, R = TS::R, NV = TS::NV, XW = TS::XW;
    constexpr int QK_LOADS = R / A::PER16;

    __shared__ __align__(16) float xch[2][WARPS > 1 ? WARPS : 1][WARPS > 1 ? XW : 4];

    pdl_prologue();

    const TAct *q = static_cast<const TAct *>(p.q);
    const TAct *k = static_cast<const TAct *>(p.k);
    const TAct *v = static_cast<const TAct *>(p.v);
    TAct *out = static_cast<TAct *>(p.out);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int vq = tid % VG;
    const int kg = tid / VG;
    const int row0 = kg * R;

    int unit = blockIdx.x;
    const int vt = unit % NV;
    unit /= NV;
    const int hv = unit % p.HV;
    const int i = unit / p.HV;
    const int col0 = vt * BV + vq * 4;

    // ---- token range and slot of sequence i -------------------------
    int64_t bos;
    int len;
    if (p.cu_seqlens) {
        const int b0 = __ldg(p.cu_seqlens + i);
        const int e0 = __ldg(p.cu_seqlens + i + 1);
        if (b0 < 0 || e0 < b0 || e0 > p.T_tot) {
            if (tid == 0)
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
        if (tid == 0)
            report(p.status, GDN_DEV_BAD_SLOT);
        return;
    }
    if (slot < 0) {
        // Padded sequence: zero output rows of this tile, no state access.
        if (kg == 0)
            for (int t = 0; t < len; ++t)
                A::store4(out + (bos + t) * p.o_tok + hv * p.o_head + col0, 0.f, 0.f, 0.f, 0.f);
        return;
    }
    if (len == 0)
        return;

    // ---- state slab -> registers (128-bit, streamed once) ------------
    float *const s_ptr = p.state + static_cast<int64_t>(slot) * p.s_slot + hv * p.s_head +
                         static_cast<int64_t>(row0) * V + col0;
    float4 s[R];
#pragma unroll
    for (int j = 0; j < R; ++j)
        s[j] = __ldcs(reinterpret_cast<const float4 *>(s_ptr + j * V));

    const int h = hv / p.G;
    float neg_A = 0.f, dt_b = 0.f;
    if constexpr (!GIVEN_GATES) {
        neg_A = -expf(__ldg(p.A_log + hv * p.A_stride));
        dt_b = __ldg(p.dt_bias + hv * p.dt_stride);
    }
    const bool l2norm = (p.flags & GDN_L2NORM_QK) != 0;
    const bool write_inter = (p.flags & GDN_WRITE_INTERMEDIATE) != 0;

    // Token inputs are software-pipelined: the raw words of token t+1 are
    // in flight while token t is computed.
    uint4 k_nx[QK_LOADS], q_nx[QK_LOADS];
    typename A::Raw4 v_nx;
    uint32_t a_nx, b_nx;
    auto fetch = [&](int64_t tok) {
        const uint4 *kp = reinterpret_cast<const uint4 *>(k + tok * p.k_tok + h * p.k_head + row0);
        const uint4 *qp = reinterpret_cast<const uint4 *>(q + tok * p.q_tok + h * p.q_head + row0);
#pragma unroll
        for (int c = 0; c < QK_LOADS; ++c) {
            k_nx[c] = __ldg(kp + c);
            q_nx[c] = __ldg(qp + c);
        }
        v_nx = __ldg(reinterpret_cast<const typename A::Raw4 *>(v + tok * p.v_tok + hv * p.v_head + col0));
        a_nx = gate_raw(p.a, tok * p.a_tok + hv * p.a_head, p.a_f32);
        b_nx = gate_raw(p.b, tok * p.b_tok + hv * p.b_head, p.b_f32);
    };
    fetch(bos);

    // The registers hold the state divided by a per-CTA scale cs (S = cs * s),
    // so that a token's decay multiplies cs instead of every element: the
    // update becomes s += k (rk / cs') delta^T with cs' = cs decay, one FMA
    // per element.  When cs' leaves [2^-60, 2^60] the decay is applied to
    // the elements instead and cs returns to 1, so s never overflows and
    // 1 / cs' stays finite (this also covers decays that underflow to 0).
    float cs = 1.f;

    for (int t = 0; t < len; ++t) {
        const int64_t tok = bos + t;

        // ---- inputs: this thread's R rows of q and k, 4 columns of v
        float kr[R], qr[R];
#pragma unroll
        for (int c = 0; c < QK_LOADS; ++c) {
            A::unpack16(k_nx[c], kr + A::PER16 * c);
            A::unpack16(q_nx[c], qr + A::PER16 * c);
        }
        const float4 v_t = A::unpack4(v_nx);
        const float a_t = gate_value(a_nx, p.a_f32);   // a, or g with given gates
        const float b_t = gate_value(b_nx, p.b_f32);   // b, or beta with given gates
        if (t + 1 < len)
            fetch(tok + 1);

        // ---- partial S^T k, S^T q, |k|^2, |q|^2, k.q over my rows ----
        float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
        float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f;
        float skk = 0.f, sqq = 0.f, skq = 0.f;
#pragma unroll
        for (int j = 0; j < R; ++j) {
            u0 = fmaf(s[j].x, kr[j], u0); u1 = fmaf(s[j].y, kr[j], u1);
            u2 = fmaf(s[j].z, kr[j], u2); u3 = fmaf(s[j].w, kr[j], u3);
            w0 = fmaf(s[j].x, qr[j], w0); w1 = fmaf(s[j].y, qr[j], w1);
            w2 = fmaf(s[j].z, qr[j], w2); w3 = fmaf(s[j].w, qr[j], w3);
            skk = fmaf(kr[j], kr[j], skk);
            sqq = fmaf(qr[j], qr[j], sqq);
            skq = fmaf(kr[j], qr[j], skq);
        }
        // lanes that differ only in their k-group hold the same columns
#pragma unroll
        for (int off = VG; off < 32; off <<= 1) {
            u0 += __shfl_xor_sync(0xffffffffu, u0, off); u1 += __shfl_xor_sync(0xffffffffu, u1, off);
            u2 += __shfl_xor_sync(0xffffffffu, u2, off); u3 += __shfl_xor_sync(0xffffffffu, u3, off);
            w0 += __shfl_xor_sync(0xffffffffu, w0, off); w1 += __shfl_xor_sync(0xffffffffu, w1, off);
            w2 += __shfl_xor_sync(0xffffffffu, w2, off); w3 += __shfl_xor_sync(0xffffffffu, w3, off);
            skk += __shfl_xor_sync(0xffffffffu, skk, off);
            sqq += __shfl_xor_sync(0xffffffffu, sqq, off);
            skq += __shfl_xor_sync(0xffffffffu, skq, off);
        }
        float4 U, W;
        float SKK, SQQ, SKQ;
        if constexpr (WARPS == 1) {
            // the whole tile lives in one warp: the shuffles already summed all rows
            U = make_float4(u0, u1, u2, u3);
            W = make_float4(w0, w1, w2, w3);
            SKK = skk; SQQ = sqq; SKQ = skq;
        } else {
            const int buf = t & 1;
            if (lane < VG) {
                *reinterpret_cast<float4 *>(&xch[buf][warp][vq * 4]) = make_float4(u0, u1, u2, u3);
                *reinterpret_cast<float4 *>(&xch[buf][warp][BV + vq * 4]) = make_float4(w0, w1, w2, w3);
                if (lane == 0) {
                    xch[buf][warp][2 * BV + 0] = skk;
                    xch[buf][warp][2 * BV + 1] = sqq;
                    xch[buf][warp][2 * BV + 2] = skq;
                }
            }
            __syncthreads();
            U = make_float4(0.f, 0.f, 0.f, 0.f);
            W = U;
            SKK = 0.f; SQQ = 0.f; SKQ = 0.f;
#pragma unroll
            for (int wi = 0; wi < WARPS; ++wi) {
                const float4 uu = *reinterpret_cast<const float4 *>(&xch[buf][wi][vq * 4]);
                const float4 ww = *reinterpret_cast<const float4 *>(&xch[buf][wi][BV + vq * 4]);
                U.x += uu.x; U.y += uu.y; U.z += uu.z; U.w += uu.w;
                W.x += ww.x; W.y += ww.y; W.z += ww.z; W.w += ww.w;
                SKK += xch[buf][wi][2 * BV + 0];
                SQQ += xch[buf][wi][2 * BV + 1];
                SKQ += xch[buf][wi][2 * BV + 2];
            }
        }

        // ---- gates and norms (scalars, computed by every thread) ----
        const float rk = l2norm ? rsqrtf(SKK + 1e-6f) : 1.f;
        const float qs = (l2norm ? rsqrtf(SQQ + 1e-6f) : 1.f) * p.scale;
        float decay, beta;
        if constexpr (GIVEN_GATES) {
            decay = expf(a_t);
            beta = b_t;
        } else {
            const float x = a_t + dt_b;
            const float sp = x > 20.f ? x : log1pf(expf(x));
            decay = expf(neg_A * sp);
            beta = __fdividef(1.f, 1.f + expf(-b_t));   // 0 for b = -inf
        }
        const float kq = SKQ * rk * qs;

        // ---- delta and output ----------------------------------
        const float cn = cs * decay;        // scale of the decayed state
        const float dku = cn * rk;
        const float dwq = cn * qs;
        const float d0 = beta * (v_t.x - dku * U.x);
        const float d1 = beta * (v_t.y - dku * U.y);
        const float d2 = beta * (v_t.z - dku * U.z);
        const float d3 = beta * (v_t.w - dku * U.w);

        // ---- S <- decay S + k^ delta^T -----------------------------
        if (cn >= 0x1p-60f && cn <= 0x1p60f) {
            // s <- s + k (rk / cs') delta^T; the scale becomes cs'
            const float f = rk * __fdividef(1.f, cn);
            const float e0 = d0 * f, e1 = d1 * f, e2 = d2 * f, e3 = d3 * f;
#pragma unroll
            for (int j = 0; j < R; ++j) {
                s[j].x = fmaf(kr[j], e0, s[j].x);
                s[j].y = fmaf(kr[j], e1, s[j].y);
                s[j].z = fmaf(kr[j], e2, s[j].z);
                s[j].w = fmaf(kr[j], e3, s[j].w);
            }
            cs = cn;
        } else {
            // apply the scale to the elements: s <- cs' s + k^ delta^T, cs = 1
#pragma unroll
            for (int j = 0; j < R; ++j) {
                const float kh = kr[j] * rk;
                s[j].x = fmaf(kh, d0, cn * s[j].x);
                s[j].y = fmaf(kh, d1, cn * s[j].y);
                s[j].z = fmaf(kh, d2, cn * s[j].z);
                s[j].w = fmaf(kh, d3, cn * s[j].w);
            }
            cs = 1.f;
        }

        if (kg == 0)
            A::store4(out + tok * p.o_tok + hv * p.o_head + col0, fmaf(kq, d0, dwq * W.x),
                      fmaf(kq, d1, dwq * W.y), fmaf(kq, d2, dwq * W.z), fmaf(kq, d3, dwq * W.w));

        // ---- optional per-token state ------------------------------
        if (write_inter) {
            float *ip = p.inter + tok * p.i_tok + hv * p.i_head + static_cast<int64_t>(row0) * V + col0;
#pragma unroll
            for (int j = 0; j < R; ++j)
                __stcs(reinterpret_cast<float4 *>(ip + j * V), make_float4(cs * s[j].x, cs * s[j].y, cs * s[j].z, cs * s[j].w));
        }
    }

    pdl_trigger();

    // ---- write the slab back in place ------------------------------
    if (!(p.flags & GDN_NO_FINAL_WRITEBACK)) {
#pragma unroll
        for (int j = 0; j < R; ++j)
            __stcs(reinterpret_cast<float4 *>(s_ptr + j * V), make_float4(cs * s[j].x, cs * s[j].y, cs * s[j].z, cs * s[j].w));
    }
}

// ---------------------------------------------------------------------------
// The gating step alone (the first kernel of the unfused pair):
//     g[t,hv]    = -exp(A_log[hv]) * softplus(a[t,hv] + dt_bias[hv])   (fp32)
//     beta[t,hv] = sigmoid(b[t,hv])                                    (fp32 or bf16)
// One thread per (token, value head), grid-stride over T_tot * HV.
// ---------------------------------------------------------------------------
struct GatingParams {
    const void *a, *b;
    const float *A_log, *dt_bias;
    float *g;
    void *beta;
    int64_t a_tok, a_head, b_tok, b_head, g_tok, g_head, beta_tok, beta_head, A_stride, dt_stride;
    int64_t n;                  // T_tot * HV
    int32_t HV, a_f32, b_f32, beta_f32;
};

__global__ void __launch_bounds__(256) gdn_gating_kernel(const __grid_constant__ GatingParams p)
{
    pdl_prologue();
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < p.n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t tok = e / p.HV;
        const int hv = static_cast<int>(e - tok * p.HV);
        const float a_t = gate_value(gate_raw(p.a, tok * p.a_tok + hv * p.a_head, p.a_f32), p.a_f32);
        const float b_t = gate_value(gate_raw(p.b, tok * p.b_tok + hv * p.b_head, p.b_f32), p.b_f32);
        const float x = a_t + __ldg(p.dt_bias + hv * p.dt_stride);
        const float sp = x > 20.f ? x : log1pf(expf(x));
        p.g[tok * p.g_tok + hv * p.g_head] = -expf(__ldg(p.A_log + hv * p.A_stride)) * sp;
        const float beta = 1.f / (1.f + expf(-b_t));
        if (p.beta_f32)
            static_cast<float *>(p.beta)[tok * p.beta_tok + hv * p.beta_head] = beta;
        else
            static_cast<__nv_bfloat16 *>(p.beta)[tok * p.beta_tok + hv * p.beta_head] = __float2bfloat16_rn(beta);
    }
    pdl_trigger();
}

}  // namespace gdn

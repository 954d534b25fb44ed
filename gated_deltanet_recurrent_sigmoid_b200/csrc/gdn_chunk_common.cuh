// gdn_chunk_common.cuh -- helpers shared by the chunked sm_100a kernels
// (gdn_chunk_local.cuh, gdn_chunk_split.cuh): the bf16 hi / lo split of fp32
// operands, 16-byte row stores into K-major operand tiles, and the issue of
// a product over several 16-column k-slices.
//
// Precision.  Operands that are not exact bf16 values (the state, T, R,
// Delta, K', P, W) are split into a bf16 high part plus a bf16 low part; a
// product is taken as hi*hi + hi*lo + lo*hi with fp32 accumulators in tensor
// memory, which keeps ~16 mantissa bits per operand (relative error ~2^-16
// per term), so the state stays well within 1e-4 of the fp32 recurrence over
// thousands of tokens.  Raw bf16 q, k, v rows are exact operands.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_sm100.cuh"

namespace gdn {
namespace chunk {

// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi).
__device__ __forceinline__ void split2(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// The hi and lo parts of two values at once, packed as bf16 pairs (x0 in the
// low half): the paired conversion rounds each value to nearest even, exactly
// as split2 does one at a time, in half the instructions.
__device__ __forceinline__ void split2x2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Eight consecutive columns c0..c0+7 (c0 % 8 == 0) of row r: one 16-byte store
// of their hi or lo parts into a K-major tile whose rows have `cols` columns.
__device__ __forceinline__ void st_row8(unsigned char *tile, uint32_t r, uint32_t c0, uint32_t cols, const float *x,
                                        bool lo_part)
{
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        uint32_t hi, lo;
        split2x2(x[2 * e], x[2 * e + 1], hi, lo);
        w[e] = lo_part ? lo : hi;
    }
    *reinterpret_cast<uint4 *>(tile + tc::kmajor_offset(r, c0, cols)) = make_uint4(w[0], w[1], w[2], w[3]);
}

// The same eight columns of row r into a hi tile and a lo tile of the same
// layout at once (one split per pair of elements, two 16-byte stores).
__device__ __forceinline__ void st_row8_hilo(unsigned char *hi_tile, unsigned char *lo_tile, uint32_t r, uint32_t c0,
                                             uint32_t cols, const float *x)
{
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        split2x2(x[2 * e], x[2 * e + 1], wh[e], wl[e]);
    const uint32_t off = tc::kmajor_offset(r, c0, cols);
    *reinterpret_cast<uint4 *>(hi_tile + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
}

// Issue a product over `slices` 16-column k-slices: D (+)= A * B^T, both
// operands K-major tiles (A: `a_cols` columns, B: `b_cols` columns).
__device__ __forceinline__ void mma_tiles(uint32_t d, const unsigned char *a, uint32_t a_cols, const unsigned char *b,
                                          uint32_t b_cols, uint32_t slices, uint32_t idesc, bool accumulate)
{
#pragma unroll 1
    for (uint32_t s = 0; s < slices; ++s)
        tc::mma_bf16(d, tc::kslice_desc(a, a_cols, s), tc::kslice_desc(b, b_cols, s), idesc,
                     (accumulate || s > 0) ? 1u : 0u);
}

}  // namespace chunk
}  // namespace gdn

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

// Eight consecutive columns c0..c0+7 (c0 % 8 == 0) of row r: one 16-byte store
// of their hi or lo parts into a K-major tile whose rows have `cols` columns.
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

// The same eight columns of row r into a hi tile and a lo tile of the same
// layout at once (one split per element, two 16-byte stores).
__device__ __forceinline__ void st_row8_hilo(unsigned char *hi_tile, unsigned char *lo_tile, uint32_t r, uint32_t c0,
                                             uint32_t cols, const float *x)
{
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat16 h0, l0, h1, l1;
        split2(x[2 * e], h0, l0);
        split2(x[2 * e + 1], h1, l1);
        wh[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        wl[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
    }
    const uint32_t off = tc::kmajor_offset(r, c0, cols);
    *reinterpret_cast<uint4 *>(hi_tile + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
}

// Issue a product over `slices` 16-column k-slices: D (+)= A * B^T, both
// operands K-major tiles (A: `a_cols` columns, B: `b_cols` columns).
__device__ __forceinline__ void mma_tiles(uint32_t d, const unsigned char *a, uint32_t a_cols, const unsigned char *b,
                                          uint32_t b_cols, uint32_t slices, uint32_t idesc, bool accumulate)
{
    for (uint32_t s = 0; s < slices; ++s)
        tc::mma_bf16(d, tc::kslice_desc(a, a_cols, s), tc::kslice_desc(b, b_cols, s), idesc,
                     (accumulate || s > 0) ? 1u : 0u);
}

}  // namespace chunk
}  // namespace gdn

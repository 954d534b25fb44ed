// tc_sm100.cuh -- thin wrappers over the sm_100a 5th-generation tensor-core
// instructions (tcgen05) used by the chunked kernel: tensor-memory (TMEM)
// allocation, shared-memory matrix descriptors, the bf16 MMA with an fp32
// accumulator in TMEM, its completion signal, and TMEM <-> register moves.
//
// Operand layout used throughout ("K-major, no swizzle"): an R x C tile of
// bf16 (C = the contraction dimension, contiguous) is stored as 8 x 8 core
// matrices of 128 contiguous bytes; element (r, c) lives at byte
//     (r / 8) * SBO + (c / 8) * 128 + (r % 8) * 16 + (c % 8) * 2,
// with SBO = (C / 8) * 128 (the next 8-row group) and LBO = 128 (the next
// 8-column chunk).  One MMA consumes 16 columns (two chunks): the
// descriptor for columns [16 s, 16 s + 16) starts at byte 256 s.
//
// MMA semantics: D[m][n] (+)= sum_c A[m][c] * B[n][c], A: M x 16 k-slice, B:
// N x 16 k-slice, D in TMEM.  For M = 128, D[m][n] sits in TMEM lane m,
// column n.  All of this follows the PTX ISA's tcgen05 chapter; the field
// positions of the descriptors are those of CUTLASS's UMMA::SmemDescriptor
// and UMMA::InstrDescriptor.
#pragma once

#include <stdint.h>

namespace gdn {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (r, c) in a K-major, unswizzled bf16 tile whose
// contraction dimension has `cols` elements.
__host__ __device__ constexpr uint32_t kmajor_offset(uint32_t r, uint32_t c, uint32_t cols)
{
    return (r >> 3) * (cols >> 3) * 128u + (c >> 3) * 128u + (r & 7u) * 16u + (c & 7u) * 2u;
}

// Shared-memory matrix descriptor: start address, leading byte offset (LBO,
// between the two 8-column chunks of one MMA), stride byte offset (SBO,
// between 8-row groups), version 1, no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;  // descriptor version for sm_100
    return d;                               // base offset 0, layout type 0 (no swizzle)
}

// Descriptor of the k-slice s (columns [16 s, 16 s + 16)) of a K-major tile.
__device__ __forceinline__ uint64_t kslice_desc(const void *tile, uint32_t cols, uint32_t s)
{
    return smem_desc(smem_u32(tile) + s * 256u, 128u, (cols >> 3) * 128u);
}

// Descriptor of an operand stored MN-major (16-byte rows of 8 consecutive
// M / N elements at one K index, 8 such rows per core matrix): `k_stride` is
// the byte distance between core matrices along K, `mn_stride` along M / N.
// As for K-major operands, the leading byte offset carries the K-direction
// stride and the stride byte offset the M / N-direction one (checked by the
// one-tile probe).
__device__ __forceinline__ uint64_t mn_desc(uint32_t saddr, uint32_t k_stride, uint32_t mn_stride)
{
    return smem_desc(saddr, k_stride, mn_stride);
}

// Instruction descriptor: bf16 x bf16 -> fp32, A and B K-major, optional
// negation of A.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool negate_a = false,
                                                      bool a_mn_major = false, bool b_mn_major = false)
{
    return (1u << 4)                           // D format: fp32
           | (1u << 7)                         // A format: bf16
           | (1u << 10)                        // B format: bf16
           | ((negate_a ? 1u : 0u) << 13)      // negate A
           | ((a_mn_major ? 1u : 0u) << 15)    // A major-ness: 1 = MN-major
           | ((b_mn_major ? 1u : 0u) << 16)    // B major-ness: 1 = MN-major
           | ((N >> 3) << 17)                  // N / 8
           | ((M >> 4) << 24);                 // M / 16
}

// One MMA, issued by a single thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        :
        : "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// Arrive (once) on an mbarrier when every MMA this thread issued so far is done.
__device__ __forceinline__ void mma_commit(unsigned long long *mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(mbar))
                 : "memory");
}

// TMEM allocation: executed by one whole warp; the base address is written
// to shared memory.  `ncols` is a power of two >= 32.
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit columns of this thread's TMEM lane (the warp's 32
// lanes are its sub-partition: warp w % 4 owns lanes 32 (w % 4) .. + 31).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the
// tensor cores (async proxy); follow with a barrier before the MMA issue.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col)
{
    return base + (lane << 16) + col;
}

}  // namespace tc
}  // namespace gdn

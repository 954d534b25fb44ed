// tc_gemm_probe.cu -- TEST INFRASTRUCTURE: one tensor-core tile product
// D = A * B^T (bf16 in, fp32 out) through the product's tcgen05 wrappers, so
// the GPU tests can check descriptors, TMEM layout, MMA issue, commit and
// TMEM loads against a plain matrix product before any kernel relies on them.
//
// One CTA of 128 threads.  A: M x K, B: N x K, D: M x N, all row-major in
// global memory; M in {64, 128}, N in {16..256, step 16}, K in {16..128, step 16}.
// With `twice`, the same products are accumulated a second time (D = 2 A B^T);
// with `negate_a`, A is negated by the instruction descriptor.
#include <cuda_bf16.h>
#include <stdint.h>

#include "mbarrier_sm100.cuh"
#include "tc_sm100.cuh"

namespace {

using namespace gdn;

__global__ void __launch_bounds__(128, 1)
tc_gemm_probe_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int M, int N, int K, int negate_a,
                     int twice, int *status)
{
    extern __shared__ __align__(1024) unsigned char smem[];
    __nv_bfloat16 *sA = reinterpret_cast<__nv_bfloat16 *>(smem);                     // up to 128 x 128
    __nv_bfloat16 *sB = reinterpret_cast<__nv_bfloat16 *>(smem + 128 * 128 * 2);     // up to 256 x 128
    unsigned long long *mbar = reinterpret_cast<unsigned long long *>(smem + 128 * 128 * 2 + 256 * 128 * 2);
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    volatile int *failed = reinterpret_cast<volatile int *>(tmem_base_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < M * K; e += blockDim.x) {
        const int r = e / K, c = e % K;
        *reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<unsigned char *>(sA) + tc::kmajor_offset(r, c, K)) =
            A[e];
    }
    for (int e = tid; e < N * K; e += blockDim.x) {
        const int r = e / K, c = e % K;
        *reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<unsigned char *>(sB) + tc::kmajor_offset(r, c, K)) =
            B[e];
    }
    if (tid == 0) {
        sync::mbar_init(mbar, 1);
        *failed = 0;
        sync::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_slot, 256);
        tc::tmem_relinquish();
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base_slot;

    if (tid == 0) {
        const uint32_t idesc = tc::idesc_bf16_f32(M, N, negate_a != 0);
        for (int rep = 0; rep < (twice ? 2 : 1); ++rep)
            for (int s = 0; s < K / 16; ++s)
                tc::mma_bf16(tmem, tc::kslice_desc(sA, K, s), tc::kslice_desc(sB, K, s), idesc,
                             (rep > 0 || s > 0) ? 1u : 0u);
        tc::mma_commit(mbar);
    }
    __syncwarp();
    const bool ok = sync::mbar_wait(mbar, 0, failed);
    if (!ok) {
        *failed = 1;
        if (lane == 0)
            atomicOr(status, 1);
    }
    tc::fence_after_sync();
    if (ok) {
        // M = 128: row m in lane m.  M = 64: row m in lane (m % 16) + 32 (m / 16).
        const int row = (M == 128) ? (warp * 32 + lane) : (lane < 16 ? warp * 16 + lane : -1);
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, warp * 32, c0), v);
            tc::tmem_wait_ld();
            if (row >= 0)
                for (int i = 0; i < 16; ++i)
                    D[row * N + c0 + i] = v[i];
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, 256);
}


// Byte offset of element (r, c) of an R x C operand stored MN-major without
// swizzle: 16-byte rows of 8 consecutive MN (r) elements at one K (c) index,
// 8 such rows (8 K indices) per 128-byte core matrix; core matrices adjacent
// along MN (128 bytes apart), then along K ((R / 8) * 128 bytes apart).
__host__ __device__ constexpr uint32_t mnmajor_offset(uint32_t r, uint32_t c, uint32_t rows)
{
    return (c >> 3) * (rows >> 3) * 128u + (r >> 3) * 128u + (c & 7u) * 16u + (r & 7u) * 2u;
}

// The same product with A and / or B given MN-major.  `swap` selects which
// descriptor field carries which stride for an MN-major operand: 0 puts the
// stride between core matrices along MN in LBO and the one along K in SBO,
// 1 the other way round.
__global__ void __launch_bounds__(128, 1)
tc_gemm_probe_mn_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int M, int N, int K, int a_mn,
                        int b_mn, int swap, int *status)
{
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *sA = smem;                           // 32 KB
    unsigned char *sB = smem + 32768;                   // 32 KB (N <= 128)
    unsigned long long *mbar = reinterpret_cast<unsigned long long *>(smem + 131072 - 64);
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    volatile int *failed = reinterpret_cast<volatile int *>(tmem_base_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < M * K; e += blockDim.x) {
        const int r = e / K, c = e % K;
        const uint32_t off = a_mn ? mnmajor_offset(r, c, M) : tc::kmajor_offset(r, c, K);
        *reinterpret_cast<__nv_bfloat16 *>(sA + off) = A[e];
    }
    for (int e = tid; e < N * K; e += blockDim.x) {
        const int r = e / K, c = e % K;
        const uint32_t off = b_mn ? mnmajor_offset(r, c, N) : tc::kmajor_offset(r, c, K);
        *reinterpret_cast<__nv_bfloat16 *>(sB + off) = B[e];
    }
    if (tid == 0) {
        sync::mbar_init(mbar, 1);
        *failed = 0;
        sync::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base_slot, 256);
        tc::tmem_relinquish();
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base_slot;

    if (tid == 0) {
        const uint32_t idesc = tc::idesc_bf16_f32(M, N) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
        for (int s = 0; s < K / 16; ++s) {
            // K-major: the k-slice starts 256 bytes on; MN-major: two K groups on
            const uint32_t a_mn_s = (M / 8) * 128, b_mn_s = (N / 8) * 128;
            const uint64_t ad = a_mn ? tc::smem_desc(tc::smem_u32(sA) + s * 2 * a_mn_s, swap ? a_mn_s : 128u,
                                                     swap ? 128u : a_mn_s)
                                     : tc::kslice_desc(sA, K, s);
            const uint64_t bd = b_mn ? tc::smem_desc(tc::smem_u32(sB) + s * 2 * b_mn_s, swap ? b_mn_s : 128u,
                                                     swap ? 128u : b_mn_s)
                                     : tc::kslice_desc(sB, K, s);
            tc::mma_bf16(tmem, ad, bd, idesc, s > 0 ? 1u : 0u);
        }
        tc::mma_commit(mbar);
    }
    __syncwarp();
    const bool ok = sync::mbar_wait(mbar, 0, failed);
    if (!ok) {
        *failed = 1;
        if (lane == 0)
            atomicOr(status, 1);
    }
    tc::fence_after_sync();
    if (ok) {
        const int row = (M == 128) ? (warp * 32 + lane) : (lane < 16 ? warp * 16 + lane : -1);
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, warp * 32, c0), v);
            tc::tmem_wait_ld();
            if (row >= 0)
                for (int i = 0; i < 16; ++i)
                    D[row * N + c0 + i] = v[i];
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0)
        tc::tmem_dealloc(tmem, 256);
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int tc_gemm_probe(const void *A, const void *B, float *D, int M,
                                                                   int N, int K, int negate_a, int twice,
                                                                   int *status, void *stream)
{
    if ((M != 64 && M != 128) || N < 16 || N > 256 || N % 16 || K < 16 || K > 128 || K % 16)
        return -1;
    const size_t smem = 128 * 128 * 2 + 256 * 128 * 2 + 64;
    cudaFuncSetAttribute(tc_gemm_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    tc_gemm_probe_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B), D, M, N, K, negate_a, twice,
        status);
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

// M, N in {64, 128}, K in {64, 128}: every read of either descriptor
// variant stays inside the kernel's 128 KB of shared memory.
extern "C" __attribute__((visibility("default"))) int tc_gemm_probe_mn(const void *A, const void *B, float *D, int M,
                                                                      int N, int K, int a_mn, int b_mn, int swap,
                                                                      int *status, void *stream)
{
    if ((M != 64 && M != 128) || (N != 64 && N != 128) || (K != 64 && K != 128))
        return -1;
    const size_t smem = 131072;
    cudaFuncSetAttribute(tc_gemm_probe_mn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    tc_gemm_probe_mn_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B), D, M, N, K, a_mn, b_mn, swap,
        status);
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

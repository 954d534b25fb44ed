// gdn_decode_api.cu -- host side of the C ABI declared in include/gdn_decode.h:
// argument validation, parameter marshalling and the kernel launch.
//
// Every check runs on the host before anything is enqueued, and none of
// them touches device memory or calls the CUDA runtime (only the optional
// GDN_CHECK_INDICES copies the index arrays back).  This file holds no step
// of the update's arithmetic; the kernel does all of it.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "gdn_decode.h"
#include "gdn_decode_kernel.cuh"
#include "gdn_chunk_split.cuh"
#include "gdn_chunk_state_half.cuh"
#include "gdn_chunk_local.cuh"
#include "gdn_decode_pipelined.cuh"

namespace {

constexpr int kHeadK = 128;
constexpr int kHeadV = 128;
// GDN_SCHEDULE_AUTO, for calls the chunked kernels are built for, by the
// mean sequence length L = T_tot / N and the (sequence, value head) pair
// count P = N * HV (measured B200 crossovers, lengths spread over
// [L/2, 3L/2]):
//   - the split kernels (with a large enough caller workspace) from L >= 80
//     while two state CTAs per pair fit one wave (2 P <= the SM count), from
//     L >= 144 when P < 128, L >= 192 when P < 256, L >= 512 when P < 512,
//     never beyond: only few, long sequences gain from computing every
//     block's products in parallel first.  The on-chip kernel's time steps
//     with the longest sequence's chunk count (~13 us a chunk), the split
//     schedule's grows by ~3 us a piece from ~22 us (device-timed graphs of
//     24 calls: 8 pairs at L = 84, 25.5 vs 28.0 us; 64 pairs at L = 94, 29.5
//     vs 40.0, at 70, 26.4 vs 28.0; 80 pairs at 131, 46.0 vs 44.1, at 177,
//     53.2 vs 59.2; 120 pairs at 135, 48.9 vs 46.9, at 147, 53.6 vs 59.5;
//     back-to-back calls: 32 sequences at L = 506, 255 vs 261 us; 64
//     sequences: the on-chip kernel is 4-10 % faster at every length up to
//     2,085, 128 sequences 16-20 %);
//   - the on-chip chunked kernel from L >= 20 when P < 64, L >= 14 when
//     P < 512, L >= 13 beyond (its one-CTA chain costs ~20 us, so with few
//     pairs the per-token kernel wins longer: 1 sequence 28.7 vs 22.5 us at
//     L = 32, 8: 26.6 vs 21.4 at 19; 1024 sequences 513 vs 539 us at 11.9,
//     663 vs 550 at 16);
//   - the per-token kernel otherwise.
bool split_pays(int64_t pairs, int64_t T_tot, int64_t N, int sms)
{
    if (2 * pairs <= sms)
        return T_tot >= 80 * N;
    if (pairs < 128)
        return T_tot >= 144 * N;
    if (pairs < 256)
        return T_tot >= 192 * N;
    if (pairs < 512)
        return T_tot >= 512 * N;
    return false;
}
int64_t chunked_min_mean_tokens(int64_t pairs) { return pairs < 64 ? 20 : (pairs < 512 ? 14 : 13); }
// The split schedule's state kernel in its compact form (two CTAs per SM)
// from this many (sequence, value head) pairs per SM, for sequences of at
// most this many tokens on average (measured on B200: 0.89-0.92x the time of
// the full form on the varlen sweeps of 256-1024 sequences, mean ~33 tokens;
// 1.06x on 64 sequences of ~480 tokens, where the full form's deeper
// prefetching wins).
constexpr int64_t kSplitCompactMinUnitsPerSm = 2;
constexpr int64_t kSplitCompactMaxMeanTokens = 128;

int64_t elem_size(int32_t dtype)
{
    switch (dtype) {
    case GDN_DTYPE_BF16: return 2;
    case GDN_DTYPE_F32: return 4;
    case GDN_DTYPE_I32: return 4;
    default: return 0;
    }
}

bool aligned(const void *p, uintptr_t bytes) { return (reinterpret_cast<uintptr_t>(p) % bytes) == 0; }

// Byte range a descriptor can reach: [lo, hi).  Empty when any dim is 0.
struct Span {
    uintptr_t lo = 0, hi = 0;
    bool empty() const { return hi <= lo; }
};

Span span_of(const gdn_tensor *t)
{
    Span s;
    if (!t || !t->data)
        return s;
    int64_t last = 0;
    for (int d = 0; d < t->ndim; ++d) {
        if (t->shape[d] == 0)
            return s;
        last += (t->shape[d] - 1) * t->stride[d];
    }
    s.lo = reinterpret_cast<uintptr_t>(t->data);
    s.hi = s.lo + static_cast<uintptr_t>((last + 1) * elem_size(t->dtype));
    return s;
}

bool overlap(const Span &x, const Span &y)
{
    if (x.empty() || y.empty())
        return false;
    return x.lo < y.hi && y.lo < x.hi;
}

// Basic descriptor sanity: rank, non-negative shape and strides, and a data
// pointer unless the tensor has no elements.  `dtype2` is a second accepted
// element type (0: none).
int check_desc(const gdn_tensor *t, int32_t dtype, int32_t dtype2 = 0)
{
    if (!t)
        return GDN_ERR_NULL_ARG;
    if (t->dtype != dtype && (dtype2 == 0 || t->dtype != dtype2))
        return GDN_ERR_DTYPE;
    if (t->ndim < 1 || t->ndim > 4)
        return GDN_ERR_SHAPE;
    bool empty = false;
    for (int d = 0; d < t->ndim; ++d) {
        if (t->shape[d] < 0 || t->stride[d] < 0)
            return GDN_ERR_SHAPE;
        empty = empty || t->shape[d] == 0;
    }
    if (!t->data && !empty)
        return GDN_ERR_NULL_ARG;
    return GDN_OK;
}

// Token layout of an activation whose trailing `trail` dims are per token.
// Varlen: leading dims [T_tot] or [1, T_tot].  Fixed length: [N, T], which
// must flatten to one token dimension.
struct TokenLayout {
    int64_t T_tot = 0;   // tokens
    int64_t T = 0;       // tokens per sequence (fixed-length mode)
    int64_t tok = 0;     // stride between consecutive tokens, in elements
};

int token_layout(const gdn_tensor *t, int trail, bool varlen, int64_t N, TokenLayout *L)
{
    const int lead = t->ndim - trail;
    if (varlen) {
        if (lead == 1) {
            L->T_tot = t->shape[0];
            L->tok = t->stride[0];
        } else if (lead == 2 && t->shape[0] == 1) {
            L->T_tot = t->shape[1];
            L->tok = t->stride[1];
        } else {
            return GDN_ERR_SHAPE;
        }
        L->T = -1;
        return GDN_OK;
    }
    if (lead != 2 || t->shape[0] != N)
        return GDN_ERR_SHAPE;
    const int64_t T = t->shape[1];
    L->T = T;
    L->T_tot = N * T;
    if (T == 0 || N == 0)
        L->tok = 0;  // no tokens: the stride is never used
    else if (T == 1)
        L->tok = t->stride[0];
    else if (N == 1)
        L->tok = t->stride[1];
    else if (t->stride[0] != T * t->stride[1])
        return GDN_ERR_SHAPE;
    else
        L->tok = t->stride[1];
    return GDN_OK;
}

// The stride of a dim matters only when the dim has more than one entry.
bool stride_ok(int64_t extent, int64_t stride, int64_t multiple)
{
    return extent <= 1 || stride % multiple == 0;
}

#define GDN_TRY(expr)              \
    do {                           \
        const int rc_ = (expr);    \
        if (rc_ != GDN_OK)         \
            return rc_;            \
    } while (0)

// Workspace bytes of the split schedule for T_tot tokens and HV value heads
// (both >= 0), saturating at UINT64_MAX instead of wrapping for sizes no
// device could hold.
uint64_t split_workspace_bytes(int64_t T_tot, int64_t HV)
{
    const uint64_t blocks = static_cast<uint64_t>((T_tot + gdn::split::C - 1) / gdn::split::C);
    uint64_t recs = 0, bytes = 0;
    if (__builtin_mul_overflow(blocks, static_cast<uint64_t>(HV), &recs) ||
        __builtin_mul_overflow(recs, static_cast<uint64_t>(gdn::split::REC_BYTES), &bytes))
        return UINT64_MAX;
    return bytes;
}

// One-time set-up per device (shared-memory opt-ins, SM counts), safe when
// several host threads make their first call on a device at once: the first
// caller runs `init` under the lock; the flag is published with release
// order after everything `init` wrote, so a thread that sees it set also
// sees those writes.  A failed `init` leaves the flag clear (the next call
// tries again).
struct PerDevice {
    static constexpr int kMaxDevices = 64;
    std::mutex lock;
    std::atomic<bool> ready[kMaxDevices] = {};
};

template <typename Init>
cudaError_t once_per_device(PerDevice &pd, int dev, Init &&init)
{
    if (dev < 0 || dev >= PerDevice::kMaxDevices)
        return cudaErrorInvalidDevice;
    if (pd.ready[dev].load(std::memory_order_acquire))
        return cudaSuccess;
    std::lock_guard<std::mutex> guard(pd.lock);
    if (pd.ready[dev].load(std::memory_order_relaxed))
        return cudaSuccess;
    const cudaError_t err = init();
    if (err == cudaSuccess)
        pd.ready[dev].store(true, std::memory_order_release);
    return err;
}

// Streaming multiprocessors of the current device (read once per device).
cudaError_t current_sm_count(int *sms)
{
    static PerDevice once;
    static int count[PerDevice::kMaxDevices];      // written once per device, inside `once`
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess)
        err = once_per_device(once, dev, [&]() {
            return cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
        });
    if (err == cudaSuccess)
        *sms = count[dev];
    return err;
}

// Host-side index check (GDN_CHECK_INDICES).
int check_indices_on_host(const int32_t *d_idx, const int32_t *d_cu, int64_t N, int64_t num_slots,
                          int64_t T_tot, cudaStream_t stream)
{
    std::vector<int32_t> idx(static_cast<size_t>(N));
    std::vector<int32_t> cu(d_cu ? static_cast<size_t>(N + 1) : 0);
    if (cudaMemcpyAsync(idx.data(), d_idx, sizeof(int32_t) * N, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (d_cu && cudaMemcpyAsync(cu.data(), d_cu, sizeof(int32_t) * (N + 1), cudaMemcpyDeviceToHost, stream) !=
                    cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    std::vector<uint8_t> seen(static_cast<size_t>(num_slots), 0);
    for (int64_t i = 0; i < N; ++i) {
        const int32_t s = idx[i];
        if (s < -1 || s >= num_slots)
            return GDN_ERR_INDICES;
        if (s >= 0) {
            if (seen[s])
                return GDN_ERR_INDICES;
            seen[s] = 1;
        }
    }
    if (d_cu) {
        if (cu[0] < 0)
            return GDN_ERR_INDICES;
        for (int64_t i = 0; i < N; ++i)
            if (cu[i + 1] < cu[i])
                return GDN_ERR_INDICES;
        if (cu[N] > T_tot)
            return GDN_ERR_INDICES;
    }
    return GDN_OK;
}

// Launch with or without the programmatic-stream-serialization attribute.
template <typename Kernel, typename... Args>
cudaError_t launch_ex(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                      const Args &...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BV, int KG, typename TAct, bool GIVEN>
cudaError_t launch(const gdn::DecodeParams &p, int64_t units, cudaStream_t stream, bool pdl)
{
    using TS = gdn::TileShape<kHeadK, kHeadV, BV, KG>;
    const dim3 grid(static_cast<unsigned>(units * TS::NV));
    return launch_ex(gdn::gdn_decode_kernel<kHeadK, kHeadV, BV, KG, TAct, GIVEN>, grid, dim3(TS::THREADS), 0,
                     stream, pdl, p);
}

// Split chunked schedule: the block kernel over ceil(T_tot / 64) x HV CTAs,
// then a state kernel over the (sequence, value head) pairs: two CTAs per
// pair (half the state columns each) while they fit one wave, the compact
// form for many short sequences, else the full-width form.  The state
// kernel always uses programmatic dependent launch behind the block kernel
// (it waits for the block kernel's completion before reading anything).
cudaError_t launch_split(const gdn::DecodeParams &p, unsigned char *ws, int64_t units, cudaStream_t stream,
                         bool pdl, bool l2norm)
{
    static PerDevice once;
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess)
        err = current_sm_count(&sms);
    if (err != cudaSuccess)
        return err;
    const size_t smem_wy = sizeof(gdn::split::WySmem), smem_st = sizeof(gdn::split::StSmem);
    err = once_per_device(once, dev, [&]() {
        cudaError_t e = cudaFuncSetAttribute(gdn::split::gdn_chunk_wy_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_wy));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::split::gdn_chunk_wy_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_wy));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::split::gdn_chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem_st));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::split::gdn_chunk_state_compact_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(sizeof(gdn::split::StSmemCompact)));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::split::gdn_chunk_state_half_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(sizeof(gdn::split::ShSmem)));
        // the largest shared-memory carveout, so that four block-kernel CTAs
        // (two compact state-kernel CTAs) fit on an SM
        for (int l2 = 0; l2 < 2 && e == cudaSuccess; ++l2)
            e = cudaFuncSetAttribute(l2 ? gdn::split::gdn_chunk_wy_kernel<true> : gdn::split::gdn_chunk_wy_kernel<false>,
                                     cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::split::gdn_chunk_state_compact_kernel,
                                     cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        return e;
    });
    if (err != cudaSuccess)
        return err;
    const int64_t blocks = (static_cast<int64_t>(p.T_tot) + gdn::split::C - 1) / gdn::split::C * p.HV;
    err = launch_ex(l2norm ? gdn::split::gdn_chunk_wy_kernel<true> : gdn::split::gdn_chunk_wy_kernel<false>,
                    dim3(static_cast<unsigned>(blocks)), dim3(gdn::split::THREADS), smem_wy, stream, pdl, p, ws);
    if (err != cudaSuccess)
        return err;
    // Few (sequence, head) pairs: two CTAs per pair, each on half the state
    // columns, as long as they fit one wave; many pairs: the compact state
    // kernel (two CTAs per SM); otherwise the full-width kernel.
    if (2 * units <= sms)
        return launch_ex(gdn::split::gdn_chunk_state_half_kernel, dim3(static_cast<unsigned>(2 * units)),
                         dim3(gdn::split::SH_THREADS), sizeof(gdn::split::ShSmem), stream, true, p,
                         static_cast<const unsigned char *>(ws));
    if (units >= kSplitCompactMinUnitsPerSm * sms &&
        static_cast<int64_t>(p.T_tot) <= kSplitCompactMaxMeanTokens * p.N)
        return launch_ex(gdn::split::gdn_chunk_state_compact_kernel, dim3(static_cast<unsigned>(units)),
                         dim3(gdn::split::SC_THREADS), sizeof(gdn::split::StSmemCompact), stream, true, p,
                         static_cast<const unsigned char *>(ws));
    return launch_ex(gdn::split::gdn_chunk_state_kernel, dim3(static_cast<unsigned>(units)),
                     dim3(gdn::split::ST_THREADS), smem_st, stream, true, p,
                     static_cast<const unsigned char *>(ws));
}

// Chunked schedule: one 256-thread CTA per (sequence, value head), two per
// SM, every chunk product on chip (gdn_chunk_local.cuh).
cudaError_t launch_chunked(const gdn::DecodeParams &p, int64_t units, cudaStream_t stream, bool pdl, bool l2norm)
{
    static PerDevice once;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    const size_t smem = sizeof(gdn::local::Smem);
    err = once_per_device(once, dev, [&]() {
        cudaError_t e = cudaSuccess;
        for (int l2 = 0; l2 < 2 && e == cudaSuccess; ++l2) {
            auto kern = l2 ? gdn::local::gdn_chunk_local_kernel<true> : gdn::local::gdn_chunk_local_kernel<false>;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            // the largest shared-memory carveout, so that two CTAs fit on an SM
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        }
        return e;
    });
    if (err != cudaSuccess)
        return err;
    return launch_ex(l2norm ? gdn::local::gdn_chunk_local_kernel<true> : gdn::local::gdn_chunk_local_kernel<false>,
                     dim3(static_cast<unsigned>(units)), dim3(gdn::local::THREADS), smem, stream, pdl, p);
}

// The tile table: (V-tile width, rows per thread) -> (BV, KG = K / rows).
template <typename TAct, bool GIVEN>
cudaError_t launch_tile(const gdn::DecodeParams &p, int64_t units, cudaStream_t stream, bool pdl, int tile_v,
                        int tile_rows)
{
    switch (tile_v * 100 + tile_rows) {
    case 808: return launch<8, 16, TAct, GIVEN>(p, units, stream, pdl);
    case 1616: return launch<16, 8, TAct, GIVEN>(p, units, stream, pdl);
    case 3216: return launch<32, 8, TAct, GIVEN>(p, units, stream, pdl);
    case 3232: return launch<32, 4, TAct, GIVEN>(p, units, stream, pdl);
    case 6416: return launch<64, 8, TAct, GIVEN>(p, units, stream, pdl);
    default: return launch<64, 4, TAct, GIVEN>(p, units, stream, pdl);
    }
}

constexpr int kPipeStages = 3;

cudaError_t launch_pipelined(const gdn::DecodeParams &p, int64_t units, cudaStream_t stream, bool pdl)
{
    // per device, once: the dynamic shared memory opt-in and the SM count
    // that sizes the persistent grid
    static PerDevice once;
    static int sms[PerDevice::kMaxDevices];           // written once per device, inside `once`
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    const size_t smem = sizeof(gdn::pipe::Smem<kPipeStages>);
    err = once_per_device(once, dev, [&]() {
        cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn::pipe::gdn_decode_pipelined_kernel<kPipeStages>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        return e;
    });
    if (err != cudaSuccess)
        return err;
    const int64_t grid = units < sms[dev] ? units : sms[dev];
    return launch_ex(gdn::pipe::gdn_decode_pipelined_kernel<kPipeStages>, dim3(static_cast<unsigned>(grid)),
                     dim3(gdn::pipe::THREADS), smem, stream, pdl, p);
}

// Everything one update call needs; the fused and the given-gate entry
// points differ only in where decay and beta come from.
struct UpdateArgs {
    const gdn_tensor *q, *k, *v, *out;
    bool given_gates;
    const gdn_tensor *gate_a, *gate_b;   // fused: a, b; given: g, beta
    const gdn_tensor *A_log, *dt_bias;   // fused only
    const gdn_tensor *state_pool, *state_indices, *cu_seqlens;
    float scale;
    uint32_t flags;
    const gdn_extra *extra;
};

int run_update(const UpdateArgs &c)
{
    const gdn_tensor *q = c.q, *k = c.k, *v = c.v, *out = c.out, *ga = c.gate_a, *gb = c.gate_b;
    const gdn_tensor *A_log = c.A_log, *dt_bias = c.dt_bias, *state_pool = c.state_pool;
    const gdn_tensor *state_indices = c.state_indices, *cu_seqlens = c.cu_seqlens;
    const gdn_extra *extra = c.extra;
    const uint32_t flags = c.flags;

    // ---- scalars and flags
    const uint32_t known =
        GDN_L2NORM_QK | GDN_WRITE_INTERMEDIATE | GDN_NO_FINAL_WRITEBACK | GDN_CHECK_INDICES | GDN_LAUNCH_PDL;
    if ((flags & ~known) != 0 || !std::isfinite(c.scale) || !(c.scale > 0.f))
        return GDN_ERR_ARG;
    int schedule = extra ? extra->schedule : GDN_SCHEDULE_AUTO;
    if (schedule != GDN_SCHEDULE_AUTO && schedule != GDN_SCHEDULE_PER_TILE && schedule != GDN_SCHEDULE_PIPELINED &&
        schedule != GDN_SCHEDULE_CHUNKED && schedule != GDN_SCHEDULE_CHUNKED_SPLIT)
        return GDN_ERR_ARG;
    if (extra && extra->reserved != 0)
        return GDN_ERR_ARG;
    const bool want_inter = (flags & GDN_WRITE_INTERMEDIATE) != 0;
    const gdn_tensor *inter = extra ? extra->intermediate_states : nullptr;
    if (want_inter && !inter)
        return GDN_ERR_NULL_ARG;

    // ---- descriptors and dtypes
    GDN_TRY(check_desc(q, GDN_DTYPE_BF16, GDN_DTYPE_F32));
    const int32_t act = q->dtype;
    GDN_TRY(check_desc(k, act));
    GDN_TRY(check_desc(v, act));
    GDN_TRY(check_desc(out, act));
    if (c.given_gates) {
        GDN_TRY(check_desc(ga, GDN_DTYPE_F32));
        GDN_TRY(check_desc(gb, GDN_DTYPE_BF16, GDN_DTYPE_F32));
    } else {
        GDN_TRY(check_desc(ga, GDN_DTYPE_BF16, GDN_DTYPE_F32));
        GDN_TRY(check_desc(gb, GDN_DTYPE_BF16, GDN_DTYPE_F32));
        GDN_TRY(check_desc(A_log, GDN_DTYPE_F32));
        GDN_TRY(check_desc(dt_bias, GDN_DTYPE_F32));
    }
    GDN_TRY(check_desc(state_pool, GDN_DTYPE_F32));
    GDN_TRY(check_desc(state_indices, GDN_DTYPE_I32));
    if (cu_seqlens)
        GDN_TRY(check_desc(cu_seqlens, GDN_DTYPE_I32));
    if (want_inter)
        GDN_TRY(check_desc(inter, GDN_DTYPE_F32));
    const bool varlen = cu_seqlens != nullptr;
    const int64_t act_size = elem_size(act);

    // ---- shapes
    if (state_indices->ndim != 1 || q->ndim < 3 || q->ndim > 4)
        return GDN_ERR_SHAPE;
    const int64_t N = state_indices->shape[0];
    const int64_t H = q->shape[q->ndim - 2], K = q->shape[q->ndim - 1];
    if (v->ndim != q->ndim)
        return GDN_ERR_SHAPE;
    const int64_t HV = v->shape[v->ndim - 2], V = v->shape[v->ndim - 1];
    if (H <= 0 || HV <= 0 || HV % H != 0 || K <= 0 || V <= 0)
        return GDN_ERR_SHAPE;

    TokenLayout Lq, Lk, Lv, La, Lb, Lo;
    GDN_TRY(token_layout(q, 2, varlen, N, &Lq));
    GDN_TRY(token_layout(k, 2, varlen, N, &Lk));
    GDN_TRY(token_layout(v, 2, varlen, N, &Lv));
    GDN_TRY(token_layout(out, 2, varlen, N, &Lo));
    if (ga->ndim != q->ndim - 1 || gb->ndim != q->ndim - 1 || out->ndim != q->ndim || k->ndim != q->ndim)
        return GDN_ERR_SHAPE;
    GDN_TRY(token_layout(ga, 1, varlen, N, &La));
    GDN_TRY(token_layout(gb, 1, varlen, N, &Lb));
    const int64_t T_tot = Lq.T_tot;
    if (Lk.T_tot != T_tot || Lv.T_tot != T_tot || Lo.T_tot != T_tot || La.T_tot != T_tot || Lb.T_tot != T_tot)
        return GDN_ERR_SHAPE;
    if (k->shape[k->ndim - 2] != H || k->shape[k->ndim - 1] != K)
        return GDN_ERR_SHAPE;
    if (out->shape[out->ndim - 2] != HV || out->shape[out->ndim - 1] != V)
        return GDN_ERR_SHAPE;
    if (ga->shape[ga->ndim - 1] != HV || gb->shape[gb->ndim - 1] != HV)
        return GDN_ERR_SHAPE;
    if (!c.given_gates &&
        (A_log->ndim != 1 || A_log->shape[0] != HV || dt_bias->ndim != 1 || dt_bias->shape[0] != HV))
        return GDN_ERR_SHAPE;
    if (state_pool->ndim != 4 || state_pool->shape[1] != HV || state_pool->shape[2] != K ||
        state_pool->shape[3] != V)
        return GDN_ERR_SHAPE;
    const int64_t num_slots = state_pool->shape[0];
    if (varlen && (cu_seqlens->ndim != 1 || cu_seqlens->shape[0] != N + 1))
        return GDN_ERR_SHAPE;
    if (want_inter && (inter->ndim != 4 || inter->shape[0] != T_tot || inter->shape[1] != HV ||
                       inter->shape[2] != K || inter->shape[3] != V))
        return GDN_ERR_SHAPE;
    if (N > INT32_MAX || T_tot > INT32_MAX || num_slots > INT32_MAX || HV > INT32_MAX ||
        (!varlen && Lq.T > INT32_MAX))
        return GDN_ERR_SHAPE;

    // ---- contiguity and alignment: q/k rows are read 16 bytes at a time,
    // v/out 4 elements at a time, the state 16 bytes at a time
    if (q->stride[q->ndim - 1] != 1 || k->stride[k->ndim - 1] != 1 || v->stride[v->ndim - 1] != 1 ||
        out->stride[out->ndim - 1] != 1)
        return GDN_ERR_SHAPE;
    if (state_pool->stride[3] != 1 || state_pool->stride[2] != V)
        return GDN_ERR_SHAPE;
    if (want_inter && (inter->stride[3] != 1 || inter->stride[2] != V))
        return GDN_ERR_SHAPE;
    if (state_indices->stride[0] != 1 && N > 1)
        return GDN_ERR_SHAPE;
    if (varlen && cu_seqlens->stride[0] != 1)
        return GDN_ERR_SHAPE;
    const int64_t qk_mult = 16 / act_size;
    for (const gdn_tensor *t : {q, k}) {
        if (!aligned(t->data, 16) || !stride_ok(T_tot, t == q ? Lq.tok : Lk.tok, qk_mult) ||
            !stride_ok(H, t->stride[t->ndim - 2], qk_mult))
            return GDN_ERR_ALIGN;
    }
    for (const gdn_tensor *t : {v, out}) {
        if (!aligned(t->data, static_cast<uintptr_t>(4 * act_size)) || !stride_ok(T_tot, t == v ? Lv.tok : Lo.tok, 4) ||
            !stride_ok(HV, t->stride[t->ndim - 2], 4))
            return GDN_ERR_ALIGN;
    }
    if (!aligned(ga->data, elem_size(ga->dtype)) || !aligned(gb->data, elem_size(gb->dtype)) ||
        !aligned(state_indices->data, 4) || (varlen && !aligned(cu_seqlens->data, 4)))
        return GDN_ERR_ALIGN;
    if (!c.given_gates && (!aligned(A_log->data, 4) || !aligned(dt_bias->data, 4)))
        return GDN_ERR_ALIGN;
    if (!aligned(state_pool->data, 16) || !stride_ok(num_slots, state_pool->stride[0], 4) ||
        !stride_ok(HV, state_pool->stride[1], 4))
        return GDN_ERR_ALIGN;
    if (want_inter && (!aligned(inter->data, 16) || !stride_ok(T_tot, inter->stride[0], 4) ||
                       !stride_ok(HV, inter->stride[1], 4)))
        return GDN_ERR_ALIGN;
    if (extra && extra->device_status && !aligned(extra->device_status, 4))
        return GDN_ERR_ALIGN;

    // ---- aliasing: nothing written may overlap anything else
    {
        const Span s_out = span_of(out), s_pool = span_of(state_pool), s_inter = want_inter ? span_of(inter) : Span{};
        const gdn_tensor *inputs[] = {q, k, v, ga, gb, c.given_gates ? nullptr : A_log,
                                      c.given_gates ? nullptr : dt_bias, state_indices, cu_seqlens};
        for (const gdn_tensor *t : inputs) {
            if (!t)
                continue;
            const Span s = span_of(t);
            if (overlap(s, s_out) || overlap(s, s_pool) || overlap(s, s_inter))
                return GDN_ERR_ALIAS;
        }
        if (overlap(s_out, s_pool) || overlap(s_out, s_inter) || overlap(s_pool, s_inter))
            return GDN_ERR_ALIAS;
        if (extra && extra->device_status) {
            Span st;
            st.lo = reinterpret_cast<uintptr_t>(extra->device_status);
            st.hi = st.lo + sizeof(uint32_t);
            if (overlap(st, s_out) || overlap(st, s_pool) || overlap(st, s_inter))
                return GDN_ERR_ALIAS;
        }
    }

    // ---- the caller's workspace (used by the split chunked schedule only):
    // a given workspace must be aligned and overlap no tensor of the call
    void *const ws = extra ? extra->workspace : nullptr;
    const uint64_t ws_bytes = extra ? extra->workspace_bytes : 0;
    if (ws) {
        if (!aligned(ws, 256))
            return GDN_ERR_ALIGN;
        Span sw;
        sw.lo = reinterpret_cast<uintptr_t>(ws);
        sw.hi = sw.lo + static_cast<uintptr_t>(ws_bytes);
        const gdn_tensor *all[] = {q, k, v, ga, gb, c.given_gates ? nullptr : A_log, c.given_gates ? nullptr : dt_bias,
                                   state_indices, cu_seqlens, out, state_pool, want_inter ? inter : nullptr};
        for (const gdn_tensor *t : all)
            if (t && overlap(sw, span_of(t)))
                return GDN_ERR_ALIAS;
        if (extra->device_status) {
            Span st;
            st.lo = reinterpret_cast<uintptr_t>(extra->device_status);
            st.hi = st.lo + sizeof(uint32_t);
            if (overlap(sw, st))
                return GDN_ERR_ALIAS;
        }
    }
    const bool ws_fits = ws && ws_bytes >= split_workspace_bytes(T_tot, HV);
    if (schedule == GDN_SCHEDULE_CHUNKED_SPLIT && !ws)
        return GDN_ERR_NULL_ARG;
    if (schedule == GDN_SCHEDULE_CHUNKED_SPLIT && !ws_fits)
        return GDN_ERR_ARG;

    // ---- supported configurations and the library's choices
    if (K != kHeadK || V != kHeadV)
        return GDN_ERR_UNSUPPORTED;
    // Single-token decode is a pure stream of state bytes: the widest tile
    // with the most rows per thread keeps the most bytes in flight per
    // register (64 x 32).  With several tokens per sequence the work per
    // state byte grows with the length and the per-token dependency chain
    // (reduction over K, then the update) sets the time: one-warp tiles need
    // no block barrier -- 32 x 32 when there are many (sequence, head)
    // pairs, 16 x 16 (twice the CTAs, shorter chains) when there are few,
    // and 8 x 8 (8 rows x 4 columns a thread, 16 V-tiles per head) for at
    // most 64 pairs, where the GPU is nearly idle and only the chain length
    // counts (measured: 1 sequence of ~29 tokens 17.7 vs 19.7 us, 8 sequences
    // 37.6 vs 39.2 us; with 64 sequences 8 x 8 is slower, 151 vs 113 us).
    const bool one_token = T_tot == N && !want_inter;
    const int64_t pairs = N * HV;
    int tile_v, tile_rows;
    if (one_token) {
        tile_v = 64;
        tile_rows = 32;
    } else if (pairs >= 2048) {
        tile_v = 32;
        tile_rows = 32;
    } else if (pairs <= 64) {
        tile_v = 8;
        tile_rows = 8;
    } else {
        tile_v = 16;
        tile_rows = 16;
    }
    if (act == GDN_DTYPE_F32) {
        // fp32 q/k rows double the prefetch registers: 16 rows per thread
        // keep every fp32 tile free of spills
        tile_v = one_token ? 32 : 16;
        tile_rows = 16;
    }
    if (extra && extra->tile_v) {
        tile_v = extra->tile_v;
        tile_rows = extra->tile_rows ? extra->tile_rows : 16;
    } else if (extra && extra->tile_rows) {
        tile_rows = extra->tile_rows;
    }
    const bool tile_ok = (tile_v == 8 && tile_rows == 8) || (tile_v == 16 && tile_rows == 16) ||
                         (tile_v == 32 && (tile_rows == 16 || tile_rows == 32)) ||
                         (tile_v == 64 && (tile_rows == 16 || tile_rows == 32));
    if (!tile_ok)
        return GDN_ERR_UNSUPPORTED;
    // The library's schedule (thresholds above): the split kernels for few,
    // long sequences, the on-chip chunked kernel from a dozen or so tokens per
    // sequence on average, else the per-tile kernel.
    const bool v_rows_16b =
        aligned(v->data, 16) && stride_ok(T_tot, Lv.tok, 8) && stride_ok(HV, v->stride[v->ndim - 2], 8);
    if (schedule == GDN_SCHEDULE_AUTO && !(extra && (extra->tile_v || extra->tile_rows)) &&
        act == GDN_DTYPE_BF16 && !c.given_gates && !want_inter && v_rows_16b && N > 0) {
        int sms = 0;
        if (ws_fits && current_sm_count(&sms) != cudaSuccess)
            return GDN_ERR_CUDA;
        if (ws_fits && split_pays(N * HV, T_tot, N, sms))
            schedule = GDN_SCHEDULE_CHUNKED_SPLIT;
        else if (T_tot >= chunked_min_mean_tokens(N * HV) * N)
            schedule = GDN_SCHEDULE_CHUNKED;
    }
    // The pipelined schedule is built for bf16 activations and fused bf16
    // gates; the chunked one for bf16 activations, fused gates and no
    // per-token states.
    if (schedule == GDN_SCHEDULE_PIPELINED &&
        (act != GDN_DTYPE_BF16 || c.given_gates || ga->dtype != GDN_DTYPE_BF16 || gb->dtype != GDN_DTYPE_BF16))
        return GDN_ERR_UNSUPPORTED;
    const bool chunked = schedule == GDN_SCHEDULE_CHUNKED || schedule == GDN_SCHEDULE_CHUNKED_SPLIT;
    if (chunked && (act != GDN_DTYPE_BF16 || c.given_gates || want_inter))
        return GDN_ERR_UNSUPPORTED;
    // the chunked kernels read v rows 16 bytes at a time, like q and k
    if (chunked && !v_rows_16b)
        return GDN_ERR_ALIGN;
    const int64_t units = N * HV;
    if (units * (kHeadV / tile_v) > INT32_MAX)
        return GDN_ERR_SHAPE;

    if (N == 0 || T_tot == 0)
        return GDN_OK;

    cudaStream_t stream = extra ? static_cast<cudaStream_t>(extra->stream) : nullptr;
    if (flags & GDN_CHECK_INDICES)
        GDN_TRY(check_indices_on_host(static_cast<const int32_t *>(state_indices->data),
                                      varlen ? static_cast<const int32_t *>(cu_seqlens->data) : nullptr, N,
                                      num_slots, T_tot, stream));

    // ---- parameters
    gdn::DecodeParams p;
    std::memset(&p, 0, sizeof p);
    p.q = q->data;
    p.k = k->data;
    p.v = v->data;
    p.a = ga->data;
    p.b = gb->data;
    p.A_log = c.given_gates ? nullptr : static_cast<const float *>(A_log->data);
    p.dt_bias = c.given_gates ? nullptr : static_cast<const float *>(dt_bias->data);
    p.state = static_cast<float *>(state_pool->data);
    p.indices = static_cast<const int32_t *>(state_indices->data);
    p.cu_seqlens = varlen ? static_cast<const int32_t *>(cu_seqlens->data) : nullptr;
    p.out = out->data;
    p.inter = want_inter ? static_cast<float *>(inter->data) : nullptr;
    p.status = extra ? extra->device_status : nullptr;
    p.q_tok = Lq.tok;
    p.q_head = q->stride[q->ndim - 2];
    p.k_tok = Lk.tok;
    p.k_head = k->stride[k->ndim - 2];
    p.v_tok = Lv.tok;
    p.v_head = v->stride[v->ndim - 2];
    p.o_tok = Lo.tok;
    p.o_head = out->stride[out->ndim - 2];
    p.a_tok = La.tok;
    p.a_head = ga->stride[ga->ndim - 1];
    p.b_tok = Lb.tok;
    p.b_head = gb->stride[gb->ndim - 1];
    p.A_stride = c.given_gates ? 0 : A_log->stride[0];
    p.dt_stride = c.given_gates ? 0 : dt_bias->stride[0];
    p.s_slot = state_pool->stride[0];
    p.s_head = state_pool->stride[1];
    p.i_tok = want_inter ? inter->stride[0] : 0;
    p.i_head = want_inter ? inter->stride[1] : 0;
    p.N = static_cast<int32_t>(N);
    p.T_fixed = varlen ? 0 : static_cast<int32_t>(Lq.T);
    p.T_tot = static_cast<int32_t>(T_tot);
    p.HV = static_cast<int32_t>(HV);
    p.G = static_cast<int32_t>(HV / H);
    p.num_slots = static_cast<int32_t>(num_slots);
    p.a_f32 = ga->dtype == GDN_DTYPE_F32;
    p.b_f32 = gb->dtype == GDN_DTYPE_F32;
    p.scale = c.scale;
    p.flags = flags;

    const bool pdl = (flags & GDN_LAUNCH_PDL) != 0;
    cudaError_t err;
    if (schedule == GDN_SCHEDULE_PIPELINED)
        err = launch_pipelined(p, units, stream, pdl);
    else if (schedule == GDN_SCHEDULE_CHUNKED)
        err = launch_chunked(p, units, stream, pdl, (flags & GDN_L2NORM_QK) != 0);
    else if (schedule == GDN_SCHEDULE_CHUNKED_SPLIT)
        err = launch_split(p, static_cast<unsigned char *>(ws), units, stream, pdl, (flags & GDN_L2NORM_QK) != 0);
    else if (act == GDN_DTYPE_BF16)
        err = c.given_gates ? launch_tile<__nv_bfloat16, true>(p, units, stream, pdl, tile_v, tile_rows)
                            : launch_tile<__nv_bfloat16, false>(p, units, stream, pdl, tile_v, tile_rows);
    else
        err = c.given_gates ? launch_tile<float, true>(p, units, stream, pdl, tile_v, tile_rows)
                            : launch_tile<float, false>(p, units, stream, pdl, tile_v, tile_rows);
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

GDN_API int gdn_version(void) { return GDN_DECODE_ABI_VERSION; }

GDN_API uint64_t gdn_static_scratch_bytes(void) { return GDN_STATIC_SCRATCH_BYTES; }

GDN_API uint64_t gdn_chunked_workspace_bytes(int64_t T_tot, int64_t HV)
{
    if (T_tot <= 0 || HV <= 0)
        return 0;
    return split_workspace_bytes(T_tot, HV);
}

GDN_API const char *gdn_status_string(int status)
{
    switch (status) {
    case GDN_OK: return "GDN_OK: success";
    case GDN_ERR_NULL_ARG: return "GDN_ERR_NULL_ARG: a required tensor or pointer is NULL";
    case GDN_ERR_DTYPE: return "GDN_ERR_DTYPE: a tensor has the wrong dtype";
    case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE: a tensor has the wrong rank, shape or strides";
    case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN: a pointer or stride breaks an alignment rule";
    case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS: a written tensor overlaps another tensor";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: head size, tile or schedule not built for this call";
    case GDN_ERR_ARG: return "GDN_ERR_ARG: bad scalar argument or flag";
    case GDN_ERR_INDICES: return "GDN_ERR_INDICES: bad or repeated state index, or bad cu_seqlens";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: the CUDA runtime refused the launch or copy";
    case GDN_ERR_SCRATCH:
        return "GDN_ERR_SCRATCH: the call needs more scratch than the library's static array holds "
               "(gdn_decode_update_static_scratch: T_tot x HV too large)";
    default: return "unknown gdn status";
    }
}

GDN_API int gdn_decode_update(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                              const gdn_tensor *a, const gdn_tensor *b, const gdn_tensor *A_log,
                              const gdn_tensor *dt_bias, const gdn_tensor *state_pool,
                              const gdn_tensor *state_indices, const gdn_tensor *cu_seqlens,
                              const gdn_tensor *out, float scale, uint32_t flags, const gdn_extra *extra)
{
    UpdateArgs c{q, k, v, out, false, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, scale, flags, extra};
    return run_update(c);
}

GDN_API int gdn_recurrent_update(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                                 const gdn_tensor *g, const gdn_tensor *beta, const gdn_tensor *state_pool,
                                 const gdn_tensor *state_indices, const gdn_tensor *cu_seqlens,
                                 const gdn_tensor *out, float scale, uint32_t flags, const gdn_extra *extra)
{
    UpdateArgs c{q, k, v, out, true, g, beta, nullptr, nullptr, state_pool, state_indices, cu_seqlens, scale, flags,
                 extra};
    return run_update(c);
}

GDN_API int gdn_gating(const gdn_tensor *A_log, const gdn_tensor *a, const gdn_tensor *dt_bias,
                       const gdn_tensor *b, const gdn_tensor *g, const gdn_tensor *beta, const gdn_extra *extra)
{
    GDN_TRY(check_desc(A_log, GDN_DTYPE_F32));
    GDN_TRY(check_desc(dt_bias, GDN_DTYPE_F32));
    GDN_TRY(check_desc(a, GDN_DTYPE_BF16, GDN_DTYPE_F32));
    GDN_TRY(check_desc(b, GDN_DTYPE_BF16, GDN_DTYPE_F32));
    GDN_TRY(check_desc(g, GDN_DTYPE_F32));
    GDN_TRY(check_desc(beta, GDN_DTYPE_BF16, GDN_DTYPE_F32));
    if (extra && (extra->schedule != 0 || extra->reserved != 0))
        return GDN_ERR_ARG;
    // a, b, g, beta: the same shape [T_tot, HV] (any leading dims that
    // flatten to tokens are passed as rank 2 here)
    const gdn_tensor *pt[] = {a, b, g, beta};
    for (const gdn_tensor *t : pt)
        if (t->ndim != 2 || t->shape[0] != a->shape[0] || t->shape[1] != a->shape[1])
            return GDN_ERR_SHAPE;
    const int64_t T_tot = a->shape[0], HV = a->shape[1];
    if (HV <= 0 || HV > INT32_MAX || A_log->ndim != 1 || A_log->shape[0] != HV || dt_bias->ndim != 1 ||
        dt_bias->shape[0] != HV)
        return GDN_ERR_SHAPE;
    for (const gdn_tensor *t : {A_log, dt_bias, a, b, g, beta})
        if (!aligned(t->data, elem_size(t->dtype)))
            return GDN_ERR_ALIGN;
    const Span sg = span_of(g), sb = span_of(beta);
    if (overlap(sg, sb))
        return GDN_ERR_ALIAS;
    for (const gdn_tensor *t : {A_log, dt_bias, a, b}) {
        const Span s = span_of(t);
        if (overlap(s, sg) || overlap(s, sb))
            return GDN_ERR_ALIAS;
    }
    if (T_tot == 0)
        return GDN_OK;

    gdn::GatingParams p;
    std::memset(&p, 0, sizeof p);
    p.a = a->data;
    p.b = b->data;
    p.A_log = static_cast<const float *>(A_log->data);
    p.dt_bias = static_cast<const float *>(dt_bias->data);
    p.g = static_cast<float *>(g->data);
    p.beta = beta->data;
    p.a_tok = a->stride[0];
    p.a_head = a->stride[1];
    p.b_tok = b->stride[0];
    p.b_head = b->stride[1];
    p.g_tok = g->stride[0];
    p.g_head = g->stride[1];
    p.beta_tok = beta->stride[0];
    p.beta_head = beta->stride[1];
    p.A_stride = A_log->stride[0];
    p.dt_stride = dt_bias->stride[0];
    p.n = T_tot * HV;
    p.HV = static_cast<int32_t>(HV);
    p.a_f32 = a->dtype == GDN_DTYPE_F32;
    p.b_f32 = b->dtype == GDN_DTYPE_F32;
    p.beta_f32 = beta->dtype == GDN_DTYPE_F32;
    cudaStream_t stream = extra ? static_cast<cudaStream_t>(extra->stream) : nullptr;
    const int64_t blocks = (p.n + 255) / 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks < 4096 ? blocks : 4096));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, gdn::gdn_gating_kernel, p);
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Scratch that needs no allocation: a fixed device array inside the library.
//
// gdn_decode_update_static_scratch serves callers that cannot allocate device
// memory themselves (see include/gdn_decode.h).  Its scratch is this file-scope
// array, created with the library's module on every GPU that loads the
// library and held until the process exits.  On the host the name
// `g_static_scratch` is only a stand-in for the device symbol, never a device
// address: the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_static_scratch on the current device.  The address
// belongs to the module the CUDA runtime loaded into the device's current
// context, and a context that is torn down and created again (e.g. after
// cudaDeviceReset) loads the module afresh, possibly elsewhere: so every call
// outside stream capture looks the address up again (a host-side table
// lookup once the module is loaded) and records it; a call made while its
// stream is capturing uses the address recorded by the last call on this
// device outside capture (capture must not load modules).  Returns nullptr
// (and the CUDA error in *err) on failure.
void *static_scratch_address(cudaStream_t stream, cudaError_t *err)
{
    static std::mutex lock;
    static void *addr[PerDevice::kMaxDevices];
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess)
        return nullptr;
    if (dev < 0 || dev >= PerDevice::kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    // the legacy stream cannot be queried while another stream captures
    // (an error): treat that as capturing
    const bool capturing = cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
    std::lock_guard<std::mutex> guard(lock);
    if (!capturing || !addr[dev]) {
        void *ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (*err != cudaSuccess)
            return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

GDN_API int gdn_decode_update_static_scratch(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                                             const gdn_tensor *a, const gdn_tensor *b, const gdn_tensor *A_log,
                                             const gdn_tensor *dt_bias, const gdn_tensor *state_pool,
                                             const gdn_tensor *state_indices, const gdn_tensor *cu_seqlens,
                                             const gdn_tensor *out, float scale, uint32_t flags,
                                             const gdn_extra *extra)
{
    if (!v)
        return GDN_ERR_NULL_ARG;
    if (extra && (extra->workspace || extra->workspace_bytes ||
                  (extra->schedule != GDN_SCHEDULE_AUTO && extra->schedule != GDN_SCHEDULE_CHUNKED_SPLIT)))
        return GDN_ERR_ARG;
    // size check first: T_tot = all leading dims of v, HV = its second-to-last.
    // Each dim is checked before it enters a product, so hostile shapes cannot
    // overflow it (T_tot <= INT32_MAX^2 fits in int64_t).
    if (v->ndim < 2 || v->ndim > 4)
        return GDN_ERR_SHAPE;
    int64_t T_tot = 1;
    for (int d = 0; d < v->ndim - 2; ++d) {
        if (v->shape[d] < 0 || v->shape[d] > INT32_MAX || (d > 0 && T_tot > INT32_MAX))
            return GDN_ERR_SHAPE;
        T_tot *= v->shape[d];
    }
    const int64_t HV = v->shape[v->ndim - 2];
    if (T_tot > INT32_MAX || HV < 0 || HV > INT32_MAX)
        return GDN_ERR_SHAPE;
    if (T_tot > 0 && HV > 0 && split_workspace_bytes(T_tot, HV) > GDN_STATIC_SCRATCH_BYTES)
        return GDN_ERR_SCRATCH;
    cudaError_t err = cudaSuccess;
    void *scratch = static_scratch_address(extra ? static_cast<cudaStream_t>(extra->stream) : nullptr, &err);
    if (!scratch)
        return GDN_ERR_CUDA;
    gdn_extra x;
    std::memset(&x, 0, sizeof x);
    if (extra)
        x = *extra;
    x.schedule = GDN_SCHEDULE_CHUNKED_SPLIT;
    x.workspace = scratch;
    x.workspace_bytes = GDN_STATIC_SCRATCH_BYTES;
    return gdn_decode_update(q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out, scale, flags,
                             &x);
}

GDN_API int gdn_host_step_issue(const gdn_host_step *s)
{
    if (!s || !s->extra || !s->host_in || !s->dev_in || !s->dev_out || !s->host_out || !s->ev_h2d ||
        !s->ev_ran || !s->ev_d2h)
        return GDN_ERR_NULL_ARG;
    cudaStream_t compute = static_cast<cudaStream_t>(s->extra->stream);
    cudaStream_t cin = static_cast<cudaStream_t>(s->copy_in_stream);
    cudaStream_t cout = static_cast<cudaStream_t>(s->copy_out_stream);
    cudaEvent_t h2d = static_cast<cudaEvent_t>(s->ev_h2d), ran = static_cast<cudaEvent_t>(s->ev_ran),
                d2h = static_cast<cudaEvent_t>(s->ev_d2h);
    cudaError_t err = cudaSuccess;
    if (s->reused)
        err = cudaStreamWaitEvent(cin, ran, 0);
    if (err == cudaSuccess && s->in_bytes)
        err = cudaMemcpyAsync(s->dev_in, s->host_in, s->in_bytes, cudaMemcpyHostToDevice, cin);
    if (err == cudaSuccess)
        err = cudaEventRecord(h2d, cin);
    if (err == cudaSuccess)
        err = cudaStreamWaitEvent(compute, h2d, 0);
    if (err == cudaSuccess && s->reused)
        err = cudaStreamWaitEvent(compute, d2h, 0);
    if (err != cudaSuccess)
        return GDN_ERR_CUDA;
    const int status = gdn_decode_update(s->q, s->k, s->v, s->a, s->b, s->A_log, s->dt_bias, s->state_pool,
                                         s->state_indices, s->cu_seqlens, s->out, s->scale, s->flags, s->extra);
    if (status != GDN_OK)
        return status;
    err = cudaEventRecord(ran, compute);
    if (err == cudaSuccess)
        err = cudaStreamWaitEvent(cout, ran, 0);
    if (err == cudaSuccess && s->out_bytes)
        err = cudaMemcpyAsync(s->host_out, s->dev_out, s->out_bytes, cudaMemcpyDeviceToHost, cout);
    if (err == cudaSuccess)
        err = cudaEventRecord(d2h, cout);
    return err == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"

// Shared device helpers for libqkq (sm_100a): PTX wrappers for the bulk-copy
// (TMA, non-tensor) + mbarrier pipeline with time-bounded waits, and constants.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qkq {

// status bits (mirror include/qkq.h)
constexpr int ST_NONFINITE = 1;
constexpr int ST_SCALE_OVERFLOW = 2;
constexpr int ST_POS_RANGE = 4;
constexpr int ST_TIMEOUT = 8;
constexpr int ST_EMPTY_STREAM = 16;
constexpr int ST_BOUNDS = 32;  // bounds-checking build only: an index check failed

// Bounds-checking build (compiled with -DQKQ_BOUNDS_CHECK, a debug library): index checks on
// the transform's copies and stores.  A failed check ORs ST_BOUNDS into the status and the
// access is skipped — never a trap, so a wrong index shows as a status bit on the host and
// the context stays usable.  In the normal build the checks compile to nothing.
#ifdef QKQ_BOUNDS_CHECK
#define QKQ_IN_BOUNDS(cond, flags) ((cond) ? true : ((flags) |= ST_BOUNDS, false))
#else
#define QKQ_IN_BOUNDS(cond, flags) true
#endif

constexpr int ROPE_HALF = 0;
constexpr int ROPE_INTERLEAVED = 1;

constexpr int MODE_HADAMARD = 0;
constexpr int MODE_PAIRWISE = 1;
constexpr int MODE_PAIRWISE_HADAMARD = 2;
constexpr int MODE_BLOCK_HADAMARD = 3;
constexpr int MODE_ROPE_ONLY = 4;

constexpr unsigned FULL_MASK = 0xffffffffu;

// A wait on an mbarrier gives up after this long (the copies it waits for take
// microseconds; only a fault elsewhere could make it run out).
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy ones (a stage is read with ld.shared, then refilled by a bulk copy).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// One bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16),
// completing `bytes` of the barrier's transaction count.  No multicast.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// One arrival on the barrier (a consumer telling the producer that a stage is free).
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the barrier phase `parity` to complete; returns false if it did not
// within limit_ns (the caller then records ST_TIMEOUT and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns = WAIT_LIMIT_NS)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Programmatic dependent launch: a kernel launched with the programmatic-serialisation
// attribute may start while the kernel before it in the stream is still running; it waits
// here, before its first read of anything that kernel may have written, until that kernel
// has completed and its writes are visible (a no-op when launched without the attribute).
// Signalling lets the next such kernel in the stream be launched early in the same way.
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kern` with programmatic stream serialisation (the launch above the kernel's
// wait_prior_grid).  Every kernel launched this way calls wait_prior_grid() before it
// reads or writes global memory.
template <typename... Params, typename... Args>
cudaError_t launch_after_prior(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t stream, Args &&...args)
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
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// max(|acc|, |x|) with NaN propagation; the sign of the result is not meaningful.
__device__ __forceinline__ float max_abs_nan(float acc, float x)
{
    float r;
    asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(acc), "f"(x));
    return r;
}

__device__ __forceinline__ int64_t clamp_pos(int m, int max_pos, int &flags)
{
    if (m < 0 || m >= max_pos) {
        flags |= ST_POS_RANGE;
        m = m < 0 ? 0 : max_pos - 1;
    }
    return m;
}

}  // namespace qkq

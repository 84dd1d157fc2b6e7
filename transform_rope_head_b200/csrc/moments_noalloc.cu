// qkq_accumulate_moments_noalloc: the calibration moment accumulation for callers
// that cannot allocate device memory.
//
// Some callers have no allocator to hand at the point where they accumulate
// calibration moments: an inference-runtime plugin whose per-batch enqueue step is
// not allowed to allocate, or a serving engine that has reserved all free HBM for its
// own pool and forbids ad-hoc allocations.  qkq_accumulate_moments needs a scratch
// workspace for its per-CTA partial sums; this variant takes that scratch from a
// fixed array compiled into the library instead, so the caller passes only its
// inputs and its accumulator.
//
// The scratch is a file-scope __device__ array of QKQ_NOALLOC_SCRATCH_BYTES (2 MiB)
// that every GPU loading the library holds until the process exits.  A call needs
// 2 x d_h/2 x 5 doubles of partial sums per CTA; this variant runs at most as many CTAs
// as fit the array (409 at d_h = 128, 819 at d_h = 64; a B200 runs 296, the same grid
// as the workspace entry point), so every size that entry point accepts fits.  Host code cannot
// use the array's name as a device address, so the first call on each device looks
// the address up with cudaGetSymbolAddress (with that device current) and caches it.
// All calls share the array: two calls whose kernels overlap on the GPU (different
// streams, or different host threads on the same device) race on it and must be
// serialised by the caller.  The partial sums are overwritten in full by every call,
// so nothing in the array has to start at zero.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qkq.h"
#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t QKQ_NOALLOC_SCRATCH_BYTES = 2u << 20;

__device__ __align__(256) double g_moment_partials[QKQ_NOALLOC_SCRATCH_BYTES / sizeof(double)];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch[kMaxDevices];

// Device address of the scratch array on the current device (looked up once per device).
int scratch_on_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QKQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moment_partials) != cudaSuccess || p == nullptr)
            return QKQ_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return QKQ_OK;
}

bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int qkq_accumulate_moments_noalloc(const void *q_bf16, const void *k_bf16,
                                              const int32_t *pos, int64_t T, int Hq, int Hkv,
                                              int d_h, int rope_style, const float *cos_tab,
                                              const float *sin_tab, int max_pos, double *moments,
                                              int *status, qkq_stream_t stream)
{
    const int pairs = rope_style & ~QKQ_ROPE_SPLIT_TABLE;
    if (pairs != QKQ_ROPE_HALF && pairs != QKQ_ROPE_INTERLEAVED) return QKQ_ERR_ARG;
    if (T < 0 || (d_h != 64 && d_h != 128) || max_pos < 1 || Hq < 1 || Hkv < 1)
        return QKQ_ERR_SHAPE;
    if (T == 0) return QKQ_OK;
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !moments) return QKQ_ERR_ARG;
    if (!aligned_to(q_bf16, 16) || !aligned_to(k_bf16, 16) || !aligned_to(cos_tab, 16) ||
        !aligned_to(sin_tab, 16) || !aligned_to(pos, 4) || !aligned_to(moments, 8) ||
        !aligned_to(status, 4))
        return QKQ_ERR_ALIGN;
    // the partial sums take 2 x d_h/2 x 5 doubles per CTA: run at most as many CTAs as fit
    const int fit = static_cast<int>(QKQ_NOALLOC_SCRATCH_BYTES / qkq::moments_partial_bytes(1, d_h));
    const int max_ctas = fit < qkq::MOM_MAX_CTAS ? fit : qkq::MOM_MAX_CTAS;
    if (qkq::moments_partial_bytes(max_ctas, d_h) > QKQ_NOALLOC_SCRATCH_BYTES) return QKQ_ERR_WORKSPACE;
    int dev = 0;
    qkq::DeviceInfo info;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&info.smem_per_block_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return QKQ_ERR_CUDA;
    if (info.cc_major != 10 || info.cc_minor != 0) return QKQ_ERR_UNSUPPORTED;
    info.ordinal = dev;
    void *scratch = nullptr;
    int rc = scratch_on_current_device(&scratch);
    if (rc) return rc;
    qkq::MomentsParams mp{};
    mp.q = static_cast<const uint16_t *>(q_bf16);
    mp.k = static_cast<const uint16_t *>(k_bf16);
    mp.pos = pos;
    mp.T = T;
    mp.Hq = Hq;
    mp.Hkv = Hkv;
    mp.cos_t = cos_tab;
    mp.sin_t = sin_tab;
    mp.max_pos = max_pos;
    mp.split = (rope_style & QKQ_ROPE_SPLIT_TABLE) != 0;
    mp.partials = static_cast<double *>(scratch);
    mp.status = status;
    int ctas = 0;
    cudaError_t e;
    if (d_h == 64)
        e = pairs == QKQ_ROPE_HALF
                ? qkq::moments_partial_launch<64, qkq::ROPE_HALF>(mp, info, max_ctas, &ctas, stream)
                : qkq::moments_partial_launch<64, qkq::ROPE_INTERLEAVED>(mp, info, max_ctas, &ctas, stream);
    else
        e = pairs == QKQ_ROPE_HALF
                ? qkq::moments_partial_launch<128, qkq::ROPE_HALF>(mp, info, max_ctas, &ctas, stream)
                : qkq::moments_partial_launch<128, qkq::ROPE_INTERLEAVED>(mp, info, max_ctas, &ctas, stream);
    if (e != cudaSuccess) return e == cudaErrorInvalidConfiguration ? QKQ_ERR_UNSUPPORTED : QKQ_ERR_CUDA;
    if (qkq::moments_final_launch(mp.partials, ctas, T * Hq, T * Hkv, d_h / 2, moments, stream) !=
        cudaSuccess)
        return QKQ_ERR_CUDA;
    return QKQ_OK;
}

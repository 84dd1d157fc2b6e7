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
// that every GPU loading the library holds until the process exits.  Host code cannot
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
    if (rope_style != QKQ_ROPE_HALF && rope_style != QKQ_ROPE_INTERLEAVED) return QKQ_ERR_ARG;
    if (T < 0 || (d_h != 64 && d_h != 128) || max_pos < 1 || Hq < 1 || Hkv < 1)
        return QKQ_ERR_SHAPE;
    if (T == 0) return QKQ_OK;
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !moments) return QKQ_ERR_ARG;
    if (!aligned_to(q_bf16, 16) || !aligned_to(k_bf16, 16) || !aligned_to(cos_tab, 16) ||
        !aligned_to(sin_tab, 16) || !aligned_to(pos, 4) || !aligned_to(moments, 8) ||
        !aligned_to(status, 4))
        return QKQ_ERR_ALIGN;
    const int P = d_h / 2;
    const int bq = qkq::moments_blocks(T * Hq), bk = qkq::moments_blocks(T * Hkv);
    const size_t need = static_cast<size_t>(bq + bk) * P * 5 * sizeof(double);
    if (need > QKQ_NOALLOC_SCRATCH_BYTES) return QKQ_ERR_WORKSPACE;  // split the batch
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return QKQ_ERR_CUDA;
    if (major != 10 || minor != 0) return QKQ_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    int rc = scratch_on_current_device(&scratch);
    if (rc) return rc;
    double *wq = static_cast<double *>(scratch);
    double *wk = wq + static_cast<size_t>(bq) * P * 5;
    qkq::MomentsParams mq{static_cast<const uint16_t *>(q_bf16), pos, T, Hq, cos_tab, sin_tab,
                          max_pos, wq, status};
    qkq::MomentsParams mk{static_cast<const uint16_t *>(k_bf16), pos, T, Hkv, cos_tab, sin_tab,
                          max_pos, wk, status};
    auto run = [&](const qkq::MomentsParams &mp, int blocks) -> cudaError_t {
        if (d_h == 64)
            return rope_style == QKQ_ROPE_HALF
                       ? qkq::moments_partial_launch<64, qkq::ROPE_HALF>(mp, blocks, stream)
                       : qkq::moments_partial_launch<64, qkq::ROPE_INTERLEAVED>(mp, blocks, stream);
        return rope_style == QKQ_ROPE_HALF
                   ? qkq::moments_partial_launch<128, qkq::ROPE_HALF>(mp, blocks, stream)
                   : qkq::moments_partial_launch<128, qkq::ROPE_INTERLEAVED>(mp, blocks, stream);
    };
    if (run(mq, bq) != cudaSuccess || run(mk, bk) != cudaSuccess) return QKQ_ERR_CUDA;
    if (qkq::moments_final_launch(wq, bq, T * Hq, wk, bk, T * Hkv, P, moments, stream) !=
        cudaSuccess)
        return QKQ_ERR_CUDA;
    return QKQ_OK;
}

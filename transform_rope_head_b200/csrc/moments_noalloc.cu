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
// The scratch is a file-scope __device__ array of QKQ_NOALLOC_SCRATCH_BYTES (5 MiB) that
// every GPU loading the library holds until the process exits.  It holds the partial sums
// of the largest grid the moments kernel ever runs (MOM_MAX_CTAS CTAs of 2 x d_h/2 x 5
// doubles at d_h = 128), so this variant launches exactly the grid of the workspace entry
// point and its results are bit for bit the same; the partial sums depend on the grid, not
// on the number of tokens, so every batch fits.  Host code cannot use the array's name as a
// device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it for the process.  All calls
// share the array: two calls whose kernels overlap on the GPU (different streams, or
// different host threads on the same device) race on it and must be serialised by the
// caller.  The partial sums are overwritten in full by every call, so nothing in the array
// has to start at zero.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qkq.h"
#include "common.cuh"
#include "internal.h"

namespace {

// the partials of MOM_MAX_CTAS CTAs at d_h = 128: 1024 x 2 x 64 x 5 doubles = 5 MiB
constexpr size_t QKQ_NOALLOC_SCRATCH_BYTES = size_t(qkq::MOM_MAX_CTAS) * 2 * 64 * 5 * sizeof(double);

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
    const qkq::NvtxRange nvtx_range("qkq_accumulate_moments_noalloc");
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
    // the workspace entry point's grid limit; its partial sums must fit the array (they
    // always do at this size: the guard keeps the two in step if either changes)
    const int max_ctas = qkq::MOM_MAX_CTAS;
    if (qkq::moments_partial_bytes(max_ctas, d_h) > QKQ_NOALLOC_SCRATCH_BYTES) return QKQ_ERR_WORKSPACE;
    qkq::DeviceInfo info;
    int rc = qkq::current_device(&info);
    if (rc) return rc;
    void *scratch = nullptr;
    rc = scratch_on_current_device(&scratch);
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

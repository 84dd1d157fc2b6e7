// C ABI of libqkq (declared in include/qkq.h): argument checks, launch-limit
// lookup per device, and dispatch to the kernels.  Host code only; it allocates
// nothing and synchronises nothing.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/qkq.h"
#include "common.cuh"
#include "internal.h"

namespace {

using qkq::DeviceInfo;

using qkq::NvtxRange;

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices];

}  // namespace

namespace qkq {

// Launch limits of the current device (queried once per device).
int current_device(DeviceInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QKQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_dev_ok[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                   dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_per_block_optin,
                                   cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) !=
                cudaSuccess)
            return QKQ_ERR_CUDA;
        d.ordinal = dev;
        g_dev[dev] = d;
        g_dev_ok[dev] = true;
    }
    *out = g_dev[dev];
    if (out->cc_major != 10 || out->cc_minor != 0) return QKQ_ERR_UNSUPPORTED;  // built for sm_100a
    return QKQ_OK;
}

}  // namespace qkq

namespace {

using qkq::current_device;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// rope_style = pair layout | optional QKQ_ROPE_SPLIT_TABLE
bool split_table(int rope_style) { return (rope_style & QKQ_ROPE_SPLIT_TABLE) != 0; }
bool half_pairs(int rope_style) { return (rope_style & ~QKQ_ROPE_SPLIT_TABLE) == QKQ_ROPE_HALF; }

int check_dims(int64_t T, int d_h, int rope_style, int max_pos)
{
    const int pairs = rope_style & ~QKQ_ROPE_SPLIT_TABLE;
    if (pairs != QKQ_ROPE_HALF && pairs != QKQ_ROPE_INTERLEAVED) return QKQ_ERR_ARG;
    if (T < 0 || (d_h != 64 && d_h != 128) || max_pos < 1) return QKQ_ERR_SHAPE;
    return QKQ_OK;
}

// w_k = theta^(-2k/d_h) in fp64, or the caller's inverse frequency
double inv_freq(int k, int d_h, double theta, const double *inv_freq_host)
{
    return inv_freq_host != nullptr
               ? inv_freq_host[k]
               : pow(theta, -(2.0 * static_cast<double>(k)) / static_cast<double>(d_h));
}

int check_mode(int mode, int b, int group, int d_h, const float *phi)
{
    if (mode < QKQ_MODE_HADAMARD || mode > QKQ_MODE_ROPE_ONLY) return QKQ_ERR_ARG;
    if ((mode == QKQ_MODE_PAIRWISE || mode == QKQ_MODE_PAIRWISE_HADAMARD) && phi == nullptr)
        return QKQ_ERR_ARG;
    if (mode == QKQ_MODE_BLOCK_HADAMARD && (!is_pow2(b) || b < 2 || b > d_h)) return QKQ_ERR_SHAPE;
    if ((group != 32 && group != 64 && group != 128) || d_h % group != 0) return QKQ_ERR_SHAPE;
    return QKQ_OK;
}

float mixing_kappa(int mode, int b, int d_h)
{
    int n = 1;
    if (mode == QKQ_MODE_HADAMARD || mode == QKQ_MODE_PAIRWISE_HADAMARD) n = d_h;
    if (mode == QKQ_MODE_BLOCK_HADAMARD) n = b;
    return static_cast<float>(1.0 / sqrt(static_cast<double>(n)));
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return QKQ_OK;
    if (e == cudaErrorInvalidConfiguration) return QKQ_ERR_UNSUPPORTED;
    return QKQ_ERR_CUDA;
}

size_t moments_ws(int64_t T, int Hq, int Hkv, int d_h)
{
    if (T <= 0 || Hq < 1 || Hkv < 1 || (d_h != 64 && d_h != 128)) return 0;
    return qkq::moments_partial_bytes(qkq::moments_max_ctas(T), d_h);
}

size_t dequant_ws(int64_t T, int Hkv)
{
    if (T <= 0 || Hkv < 1) return 0;
    return static_cast<size_t>(qkq::dequant_max_ctas(T)) * 6 * sizeof(double);
}

// qkq_transform_quantize and its Q/K/V form (v_bf16 == nullptr: no value rows).
int transform_call(const void *q_bf16, const void *k_bf16, const void *v_bf16, const int32_t *pos,
                   int64_t T, int Hq, int Hkv, int d_h, int rope_style, const float *cos_tab,
                   const float *sin_tab, int max_pos, const float *phi, int mode, int b,
                   int group, void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                   uint8_t *v_codes, void *v_scales_f16, float *k_transformed_f32,
                   float *v_transformed_f32, double *stats, void *workspace,
                   size_t workspace_bytes, int *status, qkq_stream_t stream)
{
    int rc = check_dims(T, d_h, rope_style, max_pos);
    if (rc) return rc;
    rc = check_mode(mode, b, group, d_h, phi);
    if (rc) return rc;
    if (Hq < 1 || Hkv < 1) return QKQ_ERR_SHAPE;
    if (stats != nullptr && !aligned(stats, 8)) return QKQ_ERR_ALIGN;
    if (T == 0) {  // nothing to do (empty tensors may have null pointers)
        if (stats == nullptr) return QKQ_OK;
        DeviceInfo dev0;
        const int rc0 = current_device(&dev0);
        if (rc0) return rc0;
        return from_cuda(cudaMemsetAsync(stats, 0, 6 * sizeof(double), stream));
    }
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !q_out_bf16 || !k_codes ||
        !k_scales_f16)
        return QKQ_ERR_ARG;
    if (stats != nullptr) {
        if (!aligned(workspace, 16)) return QKQ_ERR_ALIGN;
        if (workspace == nullptr || workspace_bytes < dequant_ws(T, Hkv)) return QKQ_ERR_WORKSPACE;
    }
    if (!aligned(q_bf16, 16) || !aligned(k_bf16, 16) || !aligned(q_out_bf16, 16) ||
        !aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(k_transformed_f32, 16) ||
        !aligned(k_codes, 4) || !aligned(k_scales_f16, 2) || !aligned(pos, 4) ||
        !aligned(status, 4) || !aligned(phi, 4))
        return QKQ_ERR_ALIGN;
    if (v_bf16 != nullptr &&
        (!aligned(v_bf16, 16) || !aligned(v_codes, 4) || !aligned(v_scales_f16, 2) ||
         !aligned(v_transformed_f32, 16)))
        return QKQ_ERR_ALIGN;
    const size_t qb = static_cast<size_t>(T) * Hq * d_h * 2;
    if (q_out_bf16 != q_bf16 && overlaps(q_out_bf16, qb, q_bf16, qb)) return QKQ_ERR_ARG;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    qkq::TransformParams p{};
    p.q = static_cast<const uint16_t *>(q_bf16);
    p.k = static_cast<const uint16_t *>(k_bf16);
    p.pos = pos;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.cos_t = cos_tab;
    p.sin_t = sin_tab;
    p.max_pos = max_pos;
    p.split = split_table(rope_style);
    p.phi = phi;
    p.kappa = mixing_kappa(mode, b, d_h);
    p.q_out = static_cast<uint16_t *>(q_out_bf16);
    p.k_codes = k_codes;
    p.k_scales = static_cast<uint16_t *>(k_scales_f16);
    p.k_f32 = k_transformed_f32;
    p.v = static_cast<const uint16_t *>(v_bf16);
    p.v_codes = v_bf16 ? v_codes : nullptr;
    p.v_scales = v_bf16 ? static_cast<uint16_t *>(v_scales_f16) : nullptr;
    p.v_f32 = v_bf16 ? v_transformed_f32 : nullptr;
    p.kappa_v = static_cast<float>(1.0 / sqrt(static_cast<double>(d_h)));
    p.stat_partials = stats != nullptr ? static_cast<double *>(workspace) : nullptr;
    p.status = status;
    cudaError_t e;
    int ctas = 0;
    if (d_h == 64)
        e = half_pairs(rope_style)
                ? qkq::transform_quant_launch<64, qkq::ROPE_HALF>(p, mode, b, group, dev, stream, &ctas)
                : qkq::transform_quant_launch<64, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, stream, &ctas);
    else
        e = half_pairs(rope_style)
                ? qkq::transform_quant_launch<128, qkq::ROPE_HALF>(p, mode, b, group, dev, stream, &ctas)
                : qkq::transform_quant_launch<128, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, stream, &ctas);
    if (e != cudaSuccess || stats == nullptr) return from_cuda(e);
    return from_cuda(qkq::dequant_final_launch(p.stat_partials, ctas, stats, stream));
}

}  // namespace

extern "C" {

int qkq_version(void) { return 200; }

const char *qkq_error_string(int code)
{
    switch (code) {
    case QKQ_OK: return "ok";
    case QKQ_ERR_ARG: return "invalid argument (null pointer or bad enum value)";
    case QKQ_ERR_SHAPE: return "unsupported or inconsistent sizes";
    case QKQ_ERR_ALIGN: return "pointer not aligned as required";
    case QKQ_ERR_CUDA: return "CUDA runtime error";
    case QKQ_ERR_UNSUPPORTED: return "unsupported configuration or device (needs sm_100)";
    case QKQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown error";
    }
}

const char *qkq_status_string(int s)
{
    static const char *bit_names[6] = {"nonfinite", "scale_overflow", "pos_range", "timeout",
                                       "empty_stream", "bounds"};
    static char names[64][96];  // every combination of the six bits, built once
    static std::once_flag once;
    std::call_once(once, [] {
        for (int v = 0; v < 64; ++v) {
            char *out = names[v];
            out[0] = 0;
            if (v == 0) strcpy(out, "ok");
            for (int b = 0; b < 6; ++b)
                if (v & (1 << b)) {
                    if (out[0]) strcat(out, "|");
                    strcat(out, bit_names[b]);
                }
        }
    });
    return (s >= 0 && s < 64) ? names[s] : "unknown status bits";
}

int qkq_rope_table(float *cos_host, float *sin_host, int max_pos, int d_h, double theta,
                   const double *inv_freq_host)
{
    if (cos_host == nullptr || sin_host == nullptr) return QKQ_ERR_ARG;
    if (max_pos < 1 || d_h < 2 || (d_h & 1)) return QKQ_ERR_SHAPE;
    if (inv_freq_host == nullptr && !(theta > 0.0)) return QKQ_ERR_SHAPE;
    const int P = d_h / 2;
    for (int k = 0; k < P; ++k) {
        const double w = inv_freq(k, d_h, theta, inv_freq_host);
        for (int m = 0; m < max_pos; ++m) {
            const double ang = static_cast<double>(m) * w;
            cos_host[static_cast<int64_t>(m) * P + k] = static_cast<float>(cos(ang));
            sin_host[static_cast<int64_t>(m) * P + k] = static_cast<float>(sin(ang));
        }
    }
    return QKQ_OK;
}

size_t qkq_rope_table_rows(int max_pos, int split)
{
    if (max_pos < 1) return 0;
    if (!split) return static_cast<size_t>(max_pos);
    return QKQ_ROPE_SPLIT_LOW + (static_cast<size_t>(max_pos) + QKQ_ROPE_SPLIT_LOW - 1) / QKQ_ROPE_SPLIT_LOW;
}

int qkq_rope_table_split(float *cos_host, float *sin_host, int max_pos, int d_h, double theta,
                         const double *inv_freq_host)
{
    if (cos_host == nullptr || sin_host == nullptr) return QKQ_ERR_ARG;
    if (max_pos < 1 || d_h < 2 || (d_h & 1)) return QKQ_ERR_SHAPE;
    if (inv_freq_host == nullptr && !(theta > 0.0)) return QKQ_ERR_SHAPE;
    const int P = d_h / 2;
    const int64_t rows = static_cast<int64_t>(qkq_rope_table_rows(max_pos, 1));
    for (int k = 0; k < P; ++k) {
        const double w = inv_freq(k, d_h, theta, inv_freq_host);
        for (int64_t r = 0; r < rows; ++r) {
            // low rows: l * w_k; high rows: (64 h) * w_k
            const double m = r < QKQ_ROPE_SPLIT_LOW
                                 ? static_cast<double>(r)
                                 : static_cast<double>((r - QKQ_ROPE_SPLIT_LOW) * QKQ_ROPE_SPLIT_LOW);
            const double ang = m * w;
            cos_host[r * P + k] = static_cast<float>(cos(ang));
            sin_host[r * P + k] = static_cast<float>(sin(ang));
        }
    }
    return QKQ_OK;
}

int qkq_transform_quantize(const void *q_bf16, const void *k_bf16, const int32_t *pos, int64_t T,
                           int Hq, int Hkv, int d_h, int rope_style, const float *cos_tab,
                           const float *sin_tab, int max_pos, const float *phi, int mode, int b,
                           int group, void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                           float *k_transformed_f32, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_transform_quantize");
    return transform_call(q_bf16, k_bf16, nullptr, pos, T, Hq, Hkv, d_h, rope_style, cos_tab,
                          sin_tab, max_pos, phi, mode, b, group, q_out_bf16, k_codes,
                          k_scales_f16, nullptr, nullptr, k_transformed_f32, nullptr, nullptr,
                          nullptr, 0, status, stream);
}

int qkq_transform_quantize_stats(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                                 int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                                 const float *cos_tab, const float *sin_tab, int max_pos,
                                 const float *phi, int mode, int b, int group, void *q_out_bf16,
                                 uint8_t *k_codes, void *k_scales_f16, double *stats,
                                 void *workspace, size_t workspace_bytes, int *status,
                                 qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_transform_quantize_stats");
    if (stats == nullptr) return QKQ_ERR_ARG;
    return transform_call(q_bf16, k_bf16, nullptr, pos, T, Hq, Hkv, d_h, rope_style, cos_tab,
                          sin_tab, max_pos, phi, mode, b, group, q_out_bf16, k_codes,
                          k_scales_f16, nullptr, nullptr, nullptr, nullptr, stats, workspace,
                          workspace_bytes, status, stream);
}

int qkq_transform_quantize_calibrate(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                                     int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                                     const float *cos_tab, const float *sin_tab, int max_pos,
                                     const float *phi, int mode, int b, int group,
                                     void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                                     double *moments, void *workspace, size_t workspace_bytes,
                                     int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_transform_quantize_calibrate");
    int rc = check_dims(T, d_h, rope_style, max_pos);
    if (rc) return rc;
    rc = check_mode(mode, b, group, d_h, phi);
    if (rc) return rc;
    if (Hq < 1 || Hkv < 1) return QKQ_ERR_SHAPE;
    if (moments == nullptr) return QKQ_ERR_ARG;
    if (!aligned(moments, 8)) return QKQ_ERR_ALIGN;
    if (T == 0) return QKQ_OK;
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !q_out_bf16 || !k_codes ||
        !k_scales_f16)
        return QKQ_ERR_ARG;
    if (!aligned(q_bf16, 16) || !aligned(k_bf16, 16) || !aligned(q_out_bf16, 16) ||
        !aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(k_codes, 4) ||
        !aligned(k_scales_f16, 2) || !aligned(pos, 4) || !aligned(status, 4) ||
        !aligned(phi, 4) || !aligned(workspace, 16))
        return QKQ_ERR_ALIGN;
    // Q~ is written while the moment warps read Q: no in-place output here
    const size_t qb = static_cast<size_t>(T) * Hq * d_h * 2;
    if (overlaps(q_out_bf16, qb, q_bf16, qb)) return QKQ_ERR_ARG;
    if (workspace == nullptr || workspace_bytes < moments_ws(T, Hq, Hkv, d_h)) return QKQ_ERR_WORKSPACE;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    qkq::TransformParams p{};
    p.q = static_cast<const uint16_t *>(q_bf16);
    p.k = static_cast<const uint16_t *>(k_bf16);
    p.pos = pos;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.cos_t = cos_tab;
    p.sin_t = sin_tab;
    p.max_pos = max_pos;
    p.split = split_table(rope_style);
    p.phi = phi;
    p.kappa = mixing_kappa(mode, b, d_h);
    p.q_out = static_cast<uint16_t *>(q_out_bf16);
    p.k_codes = k_codes;
    p.k_scales = static_cast<uint16_t *>(k_scales_f16);
    p.status = status;
    double *partials = static_cast<double *>(workspace);
    int ctas = 0;
    cudaError_t e;
    if (d_h == 64)
        e = half_pairs(rope_style)
                ? qkq::transform_calib_launch<64, qkq::ROPE_HALF>(p, mode, b, group, dev, partials, qkq::MOM_MAX_CTAS, &ctas, stream)
                : qkq::transform_calib_launch<64, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, partials, qkq::MOM_MAX_CTAS, &ctas, stream);
    else
        e = half_pairs(rope_style)
                ? qkq::transform_calib_launch<128, qkq::ROPE_HALF>(p, mode, b, group, dev, partials, qkq::MOM_MAX_CTAS, &ctas, stream)
                : qkq::transform_calib_launch<128, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, partials, qkq::MOM_MAX_CTAS, &ctas, stream);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(qkq::moments_final_launch(partials, ctas, T * Hq, T * Hkv, d_h / 2, moments, stream));
}

int qkq_transform_quantize_qkv(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                               const int32_t *pos, int64_t T, int Hq, int Hkv, int d_h,
                               int rope_style, const float *cos_tab, const float *sin_tab,
                               int max_pos, const float *phi, int mode, int b, int group,
                               void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                               uint8_t *v_codes, void *v_scales_f16, float *k_transformed_f32,
                               float *v_transformed_f32, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_transform_quantize_qkv");
    if (T > 0 && (!v_bf16 || !v_codes || !v_scales_f16)) return QKQ_ERR_ARG;
    return transform_call(q_bf16, k_bf16, v_bf16, pos, T, Hq, Hkv, d_h, rope_style, cos_tab,
                          sin_tab, max_pos, phi, mode, b, group, q_out_bf16, k_codes,
                          k_scales_f16, v_codes, v_scales_f16, k_transformed_f32,
                          v_transformed_f32, nullptr, nullptr, 0, status, stream);
}

int qkq_transform_quantize_tc(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                              int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                              const float *cos_tab, const float *sin_tab, int max_pos,
                              const float *phi, int mode, int b, int group, void *q_out_bf16,
                              uint8_t *k_codes, void *k_scales_f16, float *k_transformed_f32,
                              int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_transform_quantize_tc");
    int rc = check_dims(T, d_h, rope_style, max_pos);
    if (rc) return rc;
    rc = check_mode(mode, b, group, d_h, phi);
    if (rc) return rc;
    if (mode != QKQ_MODE_HADAMARD && mode != QKQ_MODE_PAIRWISE_HADAMARD &&
        mode != QKQ_MODE_BLOCK_HADAMARD)
        return QKQ_ERR_UNSUPPORTED;
    if (split_table(rope_style)) return QKQ_ERR_UNSUPPORTED;
    if (Hq < 1 || Hkv < 1) return QKQ_ERR_SHAPE;
    if (T == 0) return QKQ_OK;
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !q_out_bf16 || !k_codes ||
        !k_scales_f16)
        return QKQ_ERR_ARG;
    if (!aligned(q_bf16, 16) || !aligned(k_bf16, 16) || !aligned(q_out_bf16, 16) ||
        !aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(k_transformed_f32, 16) ||
        !aligned(k_codes, 4) || !aligned(k_scales_f16, 2) || !aligned(pos, 4) ||
        !aligned(status, 4) || !aligned(phi, 4))
        return QKQ_ERR_ALIGN;
    const size_t qb = static_cast<size_t>(T) * Hq * d_h * 2;
    if (overlaps(q_out_bf16, qb, q_bf16, qb)) return QKQ_ERR_ARG;  // rows are read after others are written
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    qkq::TransformParams p{};
    p.q = static_cast<const uint16_t *>(q_bf16);
    p.k = static_cast<const uint16_t *>(k_bf16);
    p.pos = pos;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.cos_t = cos_tab;
    p.sin_t = sin_tab;
    p.max_pos = max_pos;
    p.split = false;
    p.phi = phi;
    p.kappa = mixing_kappa(mode, b, d_h);
    p.q_out = static_cast<uint16_t *>(q_out_bf16);
    p.k_codes = k_codes;
    p.k_scales = static_cast<uint16_t *>(k_scales_f16);
    p.k_f32 = k_transformed_f32;
    p.status = status;
    cudaError_t e;
    if (d_h == 64)
        e = half_pairs(rope_style)
                ? qkq::transform_quant_tc_launch<64, qkq::ROPE_HALF>(p, mode, b, group, dev, stream)
                : qkq::transform_quant_tc_launch<64, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, stream);
    else
        e = half_pairs(rope_style)
                ? qkq::transform_quant_tc_launch<128, qkq::ROPE_HALF>(p, mode, b, group, dev, stream)
                : qkq::transform_quant_tc_launch<128, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, stream);
    return from_cuda(e);
}

namespace {

// Shared checks and parameters of the two consumer entry points; *rc < 0 on error, 1 when
// there is nothing to do.  q_align: the alignment the kernel's query loads need.
qkq::ScoresParams scores_params(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                                const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h,
                                int group, float *scores, int *status, size_t q_align,
                                DeviceInfo *dev, int *rc)
{
    qkq::ScoresParams p{};
    *rc = 0;
    if (Tq < 0 || Tk < 0 || Tq > 65535 || (d_h != 64 && d_h != 128)) { *rc = QKQ_ERR_SHAPE; return p; }
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) { *rc = QKQ_ERR_SHAPE; return p; }
    if ((group != 32 && group != 64 && group != 128) || d_h % group != 0) { *rc = QKQ_ERR_SHAPE; return p; }
    const int qpk = Hq / Hkv;
    if (qpk != 1 && qpk != 2 && qpk != 3 && qpk != 4 && qpk != 6 && qpk != 8) {
        *rc = QKQ_ERR_UNSUPPORTED;
        return p;
    }
    if (Tq == 0 || Tk == 0) { *rc = 1; return p; }
    if (!q_bf16 || !k_codes || !k_scales_f16 || !scores) { *rc = QKQ_ERR_ARG; return p; }
    if (!aligned(q_bf16, q_align) || !aligned(k_codes, 16) || !aligned(k_scales_f16, 2) ||
        !aligned(scores, 4) || (status && !aligned(status, 4))) {
        *rc = QKQ_ERR_ALIGN;
        return p;
    }
    *rc = current_device(dev);
    if (*rc) return p;
    if (Hkv > 65535) { *rc = QKQ_ERR_SHAPE; return p; }
    p.q = static_cast<const uint16_t *>(q_bf16);
    p.Tq = Tq;
    p.k_codes = k_codes;
    p.k_scales = static_cast<const uint16_t *>(k_scales_f16);
    p.Tk = Tk;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.scores = scores;
    p.status = status;
    return p;
}

}  // namespace

int qkq_attention_scores(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                         const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h, int group,
                         float *scores, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_attention_scores");
    DeviceInfo dev;
    int rc;
    const qkq::ScoresParams p = scores_params(q_bf16, Tq, k_codes, k_scales_f16, Tk, Hq, Hkv, d_h,
                                              group, scores, nullptr, 2, &dev, &rc);
    if (rc) return rc < 0 ? rc : QKQ_OK;
    return from_cuda(qkq::attention_scores_launch(p, d_h, group, stream));
}

int qkq_attention_scores_tc(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                            const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h,
                            int group, float *scores, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_attention_scores_tc");
    DeviceInfo dev;
    int rc;
    const qkq::ScoresParams p = scores_params(q_bf16, Tq, k_codes, k_scales_f16, Tk, Hq, Hkv, d_h,
                                              group, scores, status, 16, &dev, &rc);
    if (rc) return rc < 0 ? rc : QKQ_OK;
    return from_cuda(qkq::attention_scores_tc_launch(p, d_h, group, dev, stream));
}

int qkq_attention_scores_mma(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                             const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h,
                             int group, float *scores, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_attention_scores_mma");
    DeviceInfo dev;
    int rc;
    const qkq::ScoresParams p = scores_params(q_bf16, Tq, k_codes, k_scales_f16, Tk, Hq, Hkv, d_h,
                                              group, scores, nullptr, 2, &dev, &rc);
    if (rc) return rc < 0 ? rc : QKQ_OK;
    if (Tk * Hkv > 0xffffffffll) return QKQ_ERR_SHAPE;  // 32-bit cache row indices
    return from_cuda(qkq::attention_scores_mma_launch(p, dev, d_h, group, stream));
}

int qkq_selftest_bounded_wait(unsigned long long limit_ns, int *status, qkq_stream_t stream)
{
    if (status == nullptr) return QKQ_ERR_ARG;
    if (!aligned(status, 4)) return QKQ_ERR_ALIGN;
    if (limit_ns == 0 || limit_ns > 100000000ull) return QKQ_ERR_ARG;  // at most 100 ms
    DeviceInfo dev;
    const int rc = current_device(&dev);
    if (rc) return rc;
    return from_cuda(qkq::bounded_wait_selftest_launch(limit_ns, status, stream));
}

size_t qkq_moments_workspace_bytes(int64_t T, int Hq, int Hkv, int d_h)
{
    return moments_ws(T, Hq, Hkv, d_h);
}

int qkq_accumulate_moments(const void *q_bf16, const void *k_bf16, const int32_t *pos, int64_t T,
                           int Hq, int Hkv, int d_h, int rope_style, const float *cos_tab,
                           const float *sin_tab, int max_pos, double *moments, void *workspace,
                           size_t workspace_bytes, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_accumulate_moments");
    int rc = check_dims(T, d_h, rope_style, max_pos);
    if (rc) return rc;
    if (Hq < 1 || Hkv < 1) return QKQ_ERR_SHAPE;
    if (T == 0) return QKQ_OK;
    if (!q_bf16 || !k_bf16 || !pos || !cos_tab || !sin_tab || !moments) return QKQ_ERR_ARG;
    if (!aligned(q_bf16, 16) || !aligned(k_bf16, 16) || !aligned(cos_tab, 16) ||
        !aligned(sin_tab, 16) || !aligned(pos, 4) || !aligned(moments, 8) ||
        !aligned(workspace, 16) || !aligned(status, 4))
        return QKQ_ERR_ALIGN;
    const size_t need = moments_ws(T, Hq, Hkv, d_h);
    if (workspace == nullptr || workspace_bytes < need) return QKQ_ERR_WORKSPACE;
    DeviceInfo dev;
    rc = current_device(&dev);
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
    mp.split = split_table(rope_style);
    mp.partials = static_cast<double *>(workspace);
    mp.status = status;
    int ctas = 0;
    cudaError_t e;
    if (d_h == 64)
        e = half_pairs(rope_style)
                ? qkq::moments_partial_launch<64, qkq::ROPE_HALF>(mp, dev, qkq::MOM_MAX_CTAS, &ctas, stream)
                : qkq::moments_partial_launch<64, qkq::ROPE_INTERLEAVED>(mp, dev, qkq::MOM_MAX_CTAS, &ctas, stream);
    else
        e = half_pairs(rope_style)
                ? qkq::moments_partial_launch<128, qkq::ROPE_HALF>(mp, dev, qkq::MOM_MAX_CTAS, &ctas, stream)
                : qkq::moments_partial_launch<128, qkq::ROPE_INTERLEAVED>(mp, dev, qkq::MOM_MAX_CTAS, &ctas, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = qkq::moments_final_launch(mp.partials, ctas, T * Hq, T * Hkv, d_h / 2, moments, stream);
    return from_cuda(e);
}

int qkq_solve_angles(const double *moments, int d_h, int estimator, float *phi,
                     double *min_maxvar, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_solve_angles");
    if (!moments || !phi) return QKQ_ERR_ARG;
    if (estimator < QKQ_EST_POOLED || estimator > QKQ_EST_BALANCED) return QKQ_ERR_ARG;
    if (d_h != 64 && d_h != 128) return QKQ_ERR_SHAPE;
    if (!aligned(moments, 8) || !aligned(phi, 4) || !aligned(min_maxvar, 8) || !aligned(status, 4))
        return QKQ_ERR_ALIGN;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return from_cuda(
        qkq::solve_angles_launch(moments, d_h / 2, estimator, phi, min_maxvar, status, stream));
}

size_t qkq_dequant_error_workspace_bytes(int64_t T, int Hkv, int d_h, int group)
{
    (void)d_h;
    (void)group;
    return dequant_ws(T, Hkv);
}

int qkq_dequant_error(const float *k_transformed_f32, const uint8_t *k_codes,
                      const void *k_scales_f16, int64_t T, int Hkv, int d_h, int group,
                      double *stats, void *workspace, size_t workspace_bytes, int *status,
                      qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_dequant_error");
    if (T < 0 || Hkv < 1 || (d_h != 64 && d_h != 128)) return QKQ_ERR_SHAPE;
    if ((group != 32 && group != 64 && group != 128) || d_h % group != 0) return QKQ_ERR_SHAPE;
    if (!stats) return QKQ_ERR_ARG;
    if (T > 0 && (!k_transformed_f32 || !k_codes || !k_scales_f16)) return QKQ_ERR_ARG;
    if (!aligned(k_transformed_f32, 16) || !aligned(k_codes, 4) || !aligned(k_scales_f16, 2) ||
        !aligned(stats, 8) || !aligned(workspace, 16) || !aligned(status, 4))
        return QKQ_ERR_ALIGN;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    if (T == 0) return from_cuda(cudaMemsetAsync(stats, 0, 6 * sizeof(double), stream));
    const size_t need = dequant_ws(T, Hkv);
    if (workspace == nullptr || workspace_bytes < need) return QKQ_ERR_WORKSPACE;
    qkq::DequantF32Params p{};
    p.k_f32 = k_transformed_f32;
    p.k_codes = k_codes;
    p.k_scales = static_cast<const uint16_t *>(k_scales_f16);
    p.T = T;
    p.Hkv = Hkv;
    p.partials = static_cast<double *>(workspace);
    p.status = status;
    int ctas = 0;
    const cudaError_t e = qkq::dequant_f32_partial_launch(p, d_h, group, dev,
                                                          qkq::dequant_max_ctas(T), &ctas, stream);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(qkq::dequant_final_launch(p.partials, ctas, stats, stream));
}

int qkq_dequant_summary(const double *stats_host, double *summary_host)
{
    if (stats_host == nullptr || summary_host == nullptr) return QKQ_ERR_ARG;
    const double err2 = stats_host[0], ref2 = stats_host[1], n = stats_host[5];
    summary_host[0] = n > 0.0 ? stats_host[2] / n : 0.0;
    summary_host[1] = ref2 > 0.0 ? sqrt(err2 / ref2) : (err2 > 0.0 ? INFINITY : 0.0);
    summary_host[2] = n > 0.0 ? stats_host[3] / n : 0.0;
    summary_host[3] = stats_host[4];
    return QKQ_OK;
}

int qkq_dequant_error_recompute(const void *k_bf16, const int32_t *pos, int64_t T, int Hkv,
                                int d_h, int rope_style, const float *cos_tab,
                                const float *sin_tab, int max_pos, const float *phi, int mode,
                                int b, int group, const uint8_t *k_codes,
                                const void *k_scales_f16, double *stats, void *workspace,
                                size_t workspace_bytes, int *status, qkq_stream_t stream)
{
    const NvtxRange nvtx_range("qkq_dequant_error_recompute");
    int rc = check_dims(T, d_h, rope_style, max_pos);
    if (rc) return rc;
    rc = check_mode(mode, b, group, d_h, phi);
    if (rc) return rc;
    if (Hkv < 1) return QKQ_ERR_SHAPE;
    if (!k_bf16 || !pos || !cos_tab || !sin_tab || !k_codes || !k_scales_f16 || !stats)
        return QKQ_ERR_ARG;
    if (!aligned(k_bf16, 16) || !aligned(cos_tab, 16) || !aligned(sin_tab, 16) ||
        !aligned(k_codes, 16) || !aligned(k_scales_f16, 2) || !aligned(pos, 4) ||
        !aligned(stats, 8) || !aligned(workspace, 16) || !aligned(status, 4) || !aligned(phi, 4))
        return QKQ_ERR_ALIGN;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    if (T == 0) return from_cuda(cudaMemsetAsync(stats, 0, 6 * sizeof(double), stream));
    const size_t need = dequant_ws(T, Hkv);
    if (workspace == nullptr || workspace_bytes < need) return QKQ_ERR_WORKSPACE;
    qkq::DequantParams p{};
    p.k = static_cast<const uint16_t *>(k_bf16);
    p.pos = pos;
    p.T = T;
    p.Hkv = Hkv;
    p.cos_t = cos_tab;
    p.sin_t = sin_tab;
    p.max_pos = max_pos;
    p.split = split_table(rope_style);
    p.phi = phi;
    p.kappa = mixing_kappa(mode, b, d_h);
    p.k_codes = k_codes;
    p.k_scales = static_cast<const uint16_t *>(k_scales_f16);
    p.partials = static_cast<double *>(workspace);
    p.status = status;
    int ctas = 0;
    cudaError_t e;
    if (d_h == 64)
        e = half_pairs(rope_style)
                ? qkq::dequant_partial_launch<64, qkq::ROPE_HALF>(p, mode, b, group, dev, &ctas, stream)
                : qkq::dequant_partial_launch<64, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, &ctas, stream);
    else
        e = half_pairs(rope_style)
                ? qkq::dequant_partial_launch<128, qkq::ROPE_HALF>(p, mode, b, group, dev, &ctas, stream)
                : qkq::dequant_partial_launch<128, qkq::ROPE_INTERLEAVED>(p, mode, b, group, dev, &ctas, stream);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(qkq::dequant_final_launch(p.partials, ctas, stats, stream));
}

}  // extern "C"

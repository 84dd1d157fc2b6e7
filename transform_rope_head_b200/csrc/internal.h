// Internal declarations shared by the kernels (*.cu) and the C ABI layer (api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

namespace qkq {

// Launch limits of the device the call runs on (queried once per device).
struct DeviceInfo {
    int ordinal = -1;
    int num_sms = 0;
    int smem_per_sm = 0;         // bytes of shared memory per SM
    int smem_per_block_optin = 0;
    int cc_major = 0, cc_minor = 0;
};

// The current device's launch limits, queried once per device and cached (api.cu); returns a
// qkq_err code (QKQ_ERR_UNSUPPORTED on a device other than sm_100).
int current_device(DeviceInfo *out);

// An NVTX range around each entry point that launches work (named after the entry point), for
// timelines taken with a profiler; without one attached, NVTX calls return at once.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// ---- fused transform + quantisation ------------------------------------------------

struct TransformParams {
    const uint16_t *q;
    const uint16_t *k;
    const int32_t *pos;
    int64_t T;
    int Hq, Hkv;
    const float *cos_t, *sin_t;
    int max_pos;
    bool split;            // split (two-level) RoPE tables
    const float *phi;
    float kappa;           // fp32(1/sqrt(n)) of the mixing block n
    uint16_t *q_out;
    uint8_t *k_codes;
    uint16_t *k_scales;
    float *k_f32;          // nullable
    // value rows (all null when the call has no V): Hadamard of support d_h, no RoPE
    const uint16_t *v;
    uint8_t *v_codes;
    uint16_t *v_scales;
    float *v_f32;          // nullable
    float kappa_v;         // fp32(1/sqrt(d_h))
    double *stat_partials; // nullable: [grid][6] measurement statistics of the K rows
    int parts;             // filled by the launcher: 1 = whole tokens, else row-split units
    int *status;           // nullable
    int stages;            // filled by the launcher
    int stage_bytes;       // filled by the launcher
};

constexpr int TQ_PHI_BYTES = 2 * 64 * 4;   // cos, sin of up to 64 pair angles

template <int DH, int STYLE>
cudaError_t transform_quant_launch(const TransformParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, cudaStream_t stream,
                                   int *ctas_used = nullptr);

// The transform with the calibration moments of the same tokens (moments partials per
// CTA: [grid][2][d_h/2][5]); no value rows, no statistics.
template <int DH, int STYLE>
cudaError_t transform_calib_launch(const TransformParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, double *mom_partials, int max_ctas,
                                   int *ctas_used, cudaStream_t stream);

// Tensor-core variant of the Hadamard modes (HADAMARD, PAIRWISE_HADAMARD, BLOCK_HADAMARD);
// one-row-per-position tables only.
template <int DH, int STYLE>
cudaError_t transform_quant_tc_launch(const TransformParams &p, int mode, int b, int group,
                                      const DeviceInfo &dev, cudaStream_t stream);

// ---- calibration: moments ------------------------------------------------------------

struct MomentsParams {
    const uint16_t *q, *k;     // [T][Hq][d_h], [T][Hkv][d_h]
    const int32_t *pos;
    int64_t T;
    int Hq, Hkv;
    const float *cos_t, *sin_t;
    int max_pos;
    bool split;                // split (two-level) RoPE tables
    double *partials;          // [grid][2][P][5]: per-CTA sums (Sa, Sb, Saa, Sab, Sbb)
    int *status;
    int stages;                // filled by the launcher
    int stage_bytes;           // filled by the launcher
};

constexpr int MOM_WARPS = 4;
constexpr int MOM_MAX_CTAS = 1024;  // above the resident CTAs of any persistent grid here

// Upper bound of the CTAs a moments launch uses for T tokens (workspace sizing).
inline int moments_max_ctas(int64_t T)
{
    const int64_t need = (T + MOM_WARPS - 1) / MOM_WARPS;
    return static_cast<int>(need < MOM_MAX_CTAS ? need : MOM_MAX_CTAS);
}

inline size_t moments_partial_bytes(int ctas, int d_h)
{
    return static_cast<size_t>(ctas) * 2 * (d_h / 2) * 5 * sizeof(double);
}

// Launches the per-CTA accumulation with at most max_ctas CTAs; *ctas_used receives the
// grid size (the number of partials the final reduction adds).
template <int DH, int STYLE>
cudaError_t moments_partial_launch(const MomentsParams &p, const DeviceInfo &dev, int max_ctas,
                                   int *ctas_used, cudaStream_t stream);

cudaError_t moments_final_launch(const double *partials, int ctas, int64_t rows_q, int64_t rows_k,
                                 int P, double *moments, cudaStream_t stream);

// ---- calibration: closed-form angle ------------------------------------------------

cudaError_t solve_angles_launch(const double *moments, int P, int estimator, float *phi,
                                double *min_maxvar, int *status, cudaStream_t stream);

// ---- measurement -----------------------------------------------------------------------

struct DequantParams {
    const uint16_t *k;
    const int32_t *pos;
    int64_t T;
    int Hkv;
    const float *cos_t, *sin_t;
    int max_pos;
    bool split;            // split (two-level) RoPE tables
    const float *phi;
    float kappa;
    const uint8_t *k_codes;
    const uint16_t *k_scales;
    double *partials;      // [grid][6]
    int *status;
    int stages;            // filled by the launcher
    int stage_bytes;       // filled by the launcher
};

constexpr int DQ_WARPS = 4;
constexpr int DQ_MAX_CTAS = 1024;

inline int dequant_max_ctas(int64_t T)
{
    const int64_t need = (T + DQ_WARPS - 1) / DQ_WARPS;
    return static_cast<int>(need < DQ_MAX_CTAS ? need : DQ_MAX_CTAS);
}

template <int DH, int STYLE>
cudaError_t dequant_partial_launch(const DequantParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, int *ctas_used, cudaStream_t stream);

cudaError_t dequant_final_launch(const double *partials, int ctas, double *stats,
                                 cudaStream_t stream);

// The same statistics from a given fp32 K~ (no recomputation): rows [T * Hkv][d_h].
struct DequantF32Params {
    const float *k_f32;        // [T][Hkv][d_h]
    const uint8_t *k_codes;    // [T][Hkv][d_h/2]
    const uint16_t *k_scales;  // [T][Hkv][d_h/group] fp16
    int64_t T;
    int Hkv;
    double *partials;          // [grid][6]
    int *status;
};

cudaError_t dequant_f32_partial_launch(const DequantF32Params &p, int d_h, int group,
                                       const DeviceInfo &dev, int max_ctas, int *ctas_used,
                                       cudaStream_t stream);

// ---- KV4 consumer: attention logits from the int4 key cache ---------------------------

struct ScoresParams {
    const uint16_t *q;        // [Tq][Hq][d_h] bf16 (transformed queries)
    int64_t Tq;
    const uint8_t *k_codes;   // [Tk][Hkv][d_h/2]
    const uint16_t *k_scales; // [Tk][Hkv][d_h/group] fp16
    int64_t Tk;
    int Hq, Hkv;
    float *scores;            // [Tq][Hq][Tk]
    int *status;              // nullable (the tensor-core kernel's bounded waits)
};

cudaError_t attention_scores_launch(const ScoresParams &p, int d_h, int group, cudaStream_t stream);
cudaError_t attention_scores_tc_launch(const ScoresParams &p, int d_h, int group,
                                       const DeviceInfo &dev, cudaStream_t stream);
cudaError_t attention_scores_mma_launch(const ScoresParams &p, const DeviceInfo &dev, int d_h,
                                        int group, cudaStream_t stream);

// ---- test hook: the error path of the time-bounded waits ------------------------------

cudaError_t bounded_wait_selftest_launch(unsigned long long limit_ns, int *status,
                                         cudaStream_t stream);

}  // namespace qkq

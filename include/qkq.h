/*
 * qkq.h — C ABI of libqkq: the online post-RoPE Q/K transform with dynamic KV4
 * quantisation on NVIDIA B200 (sm_100a).
 *
 * The method is the one studied in "When Local Variance Optimality Is Not Enough:
 * RoPE-Aligned Q/K Rotations for Dynamic 4-Bit Quantisation" (technical summary,
 * sections "Problem statement", "Methodology", "Optimisation objective",
 * "Estimation strategies", "Core contributions"): after RoPE, Q and K are mixed by
 * one of four orthogonal maps; K is then quantised to symmetric 4-bit codes with a
 * per-group step set from the tokenwise group range; a calibration side path
 * chooses the head-shared pair angle phi*_k in closed form.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensors are caller-owned, contiguous, token-major buffers.  Unless a
 *   parameter says "host", a pointer is DEVICE memory on the current device.
 *   The library allocates nothing and keeps no per-call global state.
 * - Layouts: q [T][Hq][d_h] bf16, k [T][Hkv][d_h] bf16, pos [T] int32,
 *   cos_tab / sin_tab [max_pos][d_h/2] fp32 (or the split layout, see
 *   qkq_rope_table_split), phi [d_h/2] fp32,
 *   k_codes [T][Hkv][d_h/2] uint8, k_scales [T][Hkv][d_h/group] IEEE fp16.
 *   bf16 / fp16 values are passed as their 16-bit patterns (void*).
 * - RoPE pairs: QKQ_ROPE_HALF pairs channel k with k + d_h/2 (k < d_h/2);
 *   QKQ_ROPE_INTERLEAVED pairs 2k with 2k + 1.  Pair k at position m is turned by
 *   m * w_k with w_k = theta^(-2k/d_h) (the table below).
 * - Every device call enqueues work on `stream` (a cudaStream_t; NULL = the
 *   legacy default stream) and returns after the launch check; nothing
 *   synchronises.  Host-detectable problems return a negative qkq_err before any
 *   launch; a failed launch returns QKQ_ERR_CUDA.
 * - Data problems found on the device are OR-ed into *status (device int,
 *   nullable): QKQ_STATUS_* below.  The caller zeroes it.
 * - Supported: d_h in {64, 128}; group in {32, 64, 128} dividing d_h; 16-byte
 *   aligned q, k, q_out, k_f32, cos_tab, sin_tab; 4-byte aligned k_codes;
 *   2-byte aligned k_scales.  sm_100a only.
 * - Thread safety: calls may be made from any thread.  The only host state is a
 *   cache of launch parameters per device and kernel (occupancy, registers), filled
 *   on first use under a lock.  (qkq_accumulate_moments_noalloc's device scratch
 *   is the one shared device state; see there.)
 */
#ifndef QKQ_H
#define QKQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qkq_stream_t; /* identical to cudaStream_t */

enum qkq_err {
    QKQ_OK = 0,
    QKQ_ERR_ARG = -1,         /* null pointer or bad enum value              */
    QKQ_ERR_SHAPE = -2,       /* unsupported or inconsistent sizes            */
    QKQ_ERR_ALIGN = -3,       /* a pointer is not aligned as required          */
    QKQ_ERR_CUDA = -4,        /* the CUDA runtime reported an error            */
    QKQ_ERR_UNSUPPORTED = -5, /* combination not built (e.g. device not sm_100) */
    QKQ_ERR_WORKSPACE = -6    /* workspace missing or smaller than required     */
};

enum qkq_mode {
    QKQ_MODE_HADAMARD = 0,          /* x H_{d_h} / sqrt(d_h): the full-head baseline   */
    QKQ_MODE_PAIRWISE = 1,          /* head-shared rotation of pair k by phi_k         */
    QKQ_MODE_PAIRWISE_HADAMARD = 2, /* pairwise rotation, then the full-head Hadamard  */
    QKQ_MODE_BLOCK_HADAMARD = 3,    /* x (I_{d_h/b} (x) H_b) / sqrt(b), contiguous blocks */
    QKQ_MODE_ROPE_ONLY = 4          /* control: RoPE and no mixing                     */
};

enum qkq_estimator {
    QKQ_EST_POOLED = 0,  /* raw Q and K accumulators pooled, then centred (default) */
    QKQ_EST_K_ONLY = 1,  /* K accumulators only                                     */
    QKQ_EST_BALANCED = 2 /* equal weights on the Q and K uncentred moments          */
};

enum qkq_rope_style {
    QKQ_ROPE_HALF = 0,
    QKQ_ROPE_INTERLEAVED = 1,
    /* Flag OR-ed into a rope_style argument: the cos/sin tables are in the split
     * layout of qkq_rope_table_split (see there) instead of one row per position. */
    QKQ_ROPE_SPLIT_TABLE = 0x100
};

/* Positions per high row of a split RoPE table (the low part of m is m % 64). */
#define QKQ_ROPE_SPLIT_LOW 64

enum qkq_status_bits {
    QKQ_STATUS_NONFINITE = 1,      /* a transformed K value was NaN or Inf                */
    QKQ_STATUS_SCALE_OVERFLOW = 2, /* a group step amax/7 overflowed fp16 (> 65504)       */
    QKQ_STATUS_POS_RANGE = 4,      /* a position was outside [0, max_pos); it was clamped */
    QKQ_STATUS_TIMEOUT = 8,        /* a bounded on-chip wait gave up; outputs incomplete   */
    QKQ_STATUS_EMPTY_STREAM = 16,  /* qkq_solve_angles: a stream the estimator uses had no
                                      observations; those pairs got phi = 0               */
    QKQ_STATUS_BOUNDS = 32         /* bounds-checking debug build only: an index check of a
                                      copy or store failed; that access was skipped        */
};

/* Library version (major * 10000 + minor * 100 + patch). */
int qkq_version(void);

/* Human-readable text for a qkq_err code or a status bit mask (static storage). */
const char *qkq_error_string(int code);
const char *qkq_status_string(int status_bits);

/*
 * qkq_rope_table — HOST function: fill the RoPE cos/sin tables.
 *   cos_host[m * (d_h/2) + k] = fp32(cos(m * w_k)), sin_host likewise, computed in
 *   fp64 with w_k = theta^(-2k/d_h) (or inv_freq_host[k] when not NULL), for
 *   0 <= m < max_pos.  RoPE's frequency pairs: "Problem statement" of the paper.
 *   The tables are a model constant: fill them once and copy them to the device.
 * Arguments: cos_host / sin_host: HOST buffers of max_pos * d_h/2 floats, owned by
 *   the caller.  inv_freq_host: HOST, d_h/2 doubles, nullable.
 * Returns QKQ_OK, QKQ_ERR_ARG (null output), QKQ_ERR_SHAPE (max_pos < 1, d_h odd or
 *   < 2, theta <= 0 without inv_freq).
 */
int qkq_rope_table(float *cos_host, float *sin_host, int max_pos, int d_h, double theta,
                   const double *inv_freq_host);

/*
 * qkq_rope_table_split — HOST function: fill the split (two-level) RoPE tables.
 *   A position m = 64 * h + l (l = m % 64) turns pair k by (64 h) w_k + l w_k, so its
 *   cos/sin follow from two small tables by the angle-addition rule of two plane
 *   rotations ("Problem statement": RoPE turns fixed 2-D frequency pairs by
 *   position-dependent angles).  Rows:
 *     rows [0, 64):             cos/sin(l * w_k),        l = 0 .. 63
 *     rows [64, 64 + n_high):   cos/sin((64 h) * w_k),   h = 0 .. n_high - 1,
 *   n_high = ceil(max_pos / 64); each entry fp32 of the fp64 value, as in qkq_rope_table.
 *   With QKQ_ROPE_SPLIT_TABLE in rope_style the kernels read the two rows of a position
 *   and compose them in fp32, high turned by low:
 *     c = fma(c_h, c_l, -(s_h*s_l)),  s = fma(c_h, s_l, s_h*c_l)
 *   (RoPE with that entry, then, in the pairwise modes, the pair rotation by phi as its
 *   own step).  The two tables hold 64 + n_high rows
 *   (1.1 MB at d_h = 128, max_pos = 131072, against 67 MB with one row per position):
 *   they stay in L2, so the per-token table reads leave HBM.
 * Arguments: cos_host / sin_host: HOST buffers of qkq_rope_table_rows(max_pos, 1) * d_h/2
 *   floats; the rest as qkq_rope_table.  Returns as qkq_rope_table.
 */
int qkq_rope_table_split(float *cos_host, float *sin_host, int max_pos, int d_h, double theta,
                         const double *inv_freq_host);

/* Rows of the RoPE tables for positions [0, max_pos): max_pos, or with split != 0
 * 64 + ceil(max_pos / 64).  0 if max_pos < 1. */
size_t qkq_rope_table_rows(int max_pos, int split);

/*
 * qkq_transform_quantize — the fused hot path (one kernel).
 *   For every token t and head h: y = RoPE(x) with the table row pos[t]; then the
 *   mixing `mode` ("Methodology": full-head Hadamard, pairwise-only, pairwise +
 *   Hadamard; "Core contributions": block Hadamard of support b); Q~ = y is stored
 *   as bf16 (Q is not quantised, "Estimation strategies"); for K~, every group of
 *   `group` contiguous channels gets s = max|x|/7 and codes clip(round(x/s), -7, 7)
 *   ("Core contributions": the dynamic quantiser's step comes from the tokenwise
 *   group range; quantiser formula: "LLM旋转量化笔记" §1.2).
 *   The fp32 order of operations is fixed (bit-exact contract), step by step in the
 *   method's order:
 *     RoPE: rotation of a pair a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c) with the RoPE
 *     table entry (c, s) (with a split table: composed from its two rows first, see
 *     qkq_rope_table_split);
 *     pairwise modes: then the pair rotation, its own step with the same two lines and
 *     (cos phi_k, sin phi_k) in place of (c, s);
 *     butterflies (u, v) -> (u+v, u-v) at strides 1, 2, ..., n/2, then * fp32(1/sqrt(n));
 *     r = fp32(7/amax), code = the exact product x*r rounded once to the nearest integer
 *     (ties to even), scale = fp16_rn(fp32(amax/7));
 *     groups with amax < 2^-125 get codes 0 and scale 0;
 *     phi's cos/sin = fp32 of the fp64 cos/sin of the fp32 angle.
 * Arguments
 *   q_bf16 [T][Hq][d_h], k_bf16 [T][Hkv][d_h]: inputs (device).  Hq % Hkv == 0 is
 *     not required; T >= 0 (T == 0 is a no-op).
 *   pos [T]: positions (device int32); rows outside [0, max_pos) are computed at
 *     the clamped position and QKQ_STATUS_POS_RANGE is set.
 *   rope_style: QKQ_ROPE_HALF or QKQ_ROPE_INTERLEAVED, optionally | QKQ_ROPE_SPLIT_TABLE.
 *   cos_tab, sin_tab [qkq_rope_table_rows(max_pos, split)][d_h/2]: the RoPE tables
 *     (device fp32) in the layout rope_style names.
 *   phi [d_h/2]: pair angles (device fp32); required for the two pairwise modes,
 *     ignored (may be NULL) otherwise.
 *   mode: qkq_mode.  b: block support for QKQ_MODE_BLOCK_HADAMARD, a power of two in
 *     [2, d_h]; ignored otherwise.  group: K quantisation group, {32, 64, 128}, divides d_h.
 *   q_out_bf16 [T][Hq][d_h]: Q~ (device); must not overlap q_bf16 unless identical
 *     (in-place is allowed).
 *   k_codes [T][Hkv][d_h/2]: packed codes, byte j = code[2j] & 0xF | (code[2j+1] & 0xF) << 4.
 *   k_scales_f16 [T][Hkv][d_h/group]: per-group fp16 scale (device).
 *   k_transformed_f32 [T][Hkv][d_h]: nullable; fp32 K~ before quantisation (tests,
 *     measurement).
 *   status: nullable device int, QKQ_STATUS_* OR-ed in.
 * Returns QKQ_OK or a negative qkq_err (nothing launched on error).
 */
int qkq_transform_quantize(const void *q_bf16, const void *k_bf16, const int32_t *pos, int64_t T,
                           int Hq, int Hkv, int d_h, int rope_style, const float *cos_tab,
                           const float *sin_tab, int max_pos, const float *phi, int mode, int b,
                           int group, void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                           float *k_transformed_f32, int *status, qkq_stream_t stream);

/*
 * qkq_moments_workspace_bytes — scratch needed by qkq_accumulate_moments for
 *   these sizes (device memory the caller allocates; 0 when T == 0): the per-CTA
 *   partial sums, at most 1024 CTAs x 2 x d_h/2 x 5 doubles (5.2 MB at d_h = 128).
 */
size_t qkq_moments_workspace_bytes(int64_t T, int Hq, int Hkv, int d_h);

/*
 * qkq_transform_quantize_stats — qkq_transform_quantize with the measurement statistics of
 *   its K rows computed in the same pass (the a11 statistics of qkq_dequant_error, fused into
 *   the producing kernel instead of re-reading and re-transforming K).
 *   Outputs as qkq_transform_quantize (no fp32 K~ copy), plus stats [6] fp64 (device):
 *   sum (K~ - K^)^2, sum K~^2, sum of group max|K~|, sum of group (max - min), max of group
 *   max|K~|, number of groups — the same definitions and fp32/fp64 arithmetic as
 *   qkq_dequant_error, summed in another order (results agree to the stated tolerance of
 *   those sums, not bit for bit).  One more small launch reduces the per-CTA partials.
 * Arguments (beyond qkq_transform_quantize's)
 *   stats [6]: device, written (not accumulated).
 *   workspace / workspace_bytes: device scratch of at least
 *     qkq_dequant_error_workspace_bytes(T, Hkv, d_h, group) bytes, 16-byte aligned.
 * Returns as qkq_transform_quantize; QKQ_ERR_ARG for a null stats, QKQ_ERR_WORKSPACE for a
 *   missing or small workspace.
 */
int qkq_transform_quantize_stats(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                                 int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                                 const float *cos_tab, const float *sin_tab, int max_pos,
                                 const float *phi, int mode, int b, int group, void *q_out_bf16,
                                 uint8_t *k_codes, void *k_scales_f16, double *stats,
                                 void *workspace, size_t workspace_bytes, int *status,
                                 qkq_stream_t stream);

/*
 * qkq_transform_quantize_calibrate — qkq_transform_quantize and qkq_accumulate_moments of the
 *   same tokens in one pass (Q and K read from HBM once).
 *   The moments are of the post-RoPE, pre-mixing values, so they do not depend on phi: a
 *   calibrating pass transforms with the current angles and accumulates the raw sums for the
 *   next qkq_solve_angles ("Estimation strategies": pooled raw accumulators; calibration over
 *   the positions the model sees).  Outputs Q~, codes, scales exactly as
 *   qkq_transform_quantize (bit for bit), and adds to moments exactly what
 *   qkq_accumulate_moments would (same fp64 sums, another summation order).
 * Arguments (beyond qkq_transform_quantize's; no k_transformed_f32)
 *   moments [2][d_h/2][6] fp64: ADDED TO (caller zeroes), as qkq_accumulate_moments.
 *   workspace / workspace_bytes: at least qkq_moments_workspace_bytes(T, Hq, Hkv, d_h).
 *   q_out must not overlap q (the moment warps read Q while Q~ is written).
 * Returns as qkq_transform_quantize; QKQ_ERR_ARG for a null moments or an overlapping
 *   q_out, QKQ_ERR_WORKSPACE for a missing or small workspace.
 */
int qkq_transform_quantize_calibrate(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                                     int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                                     const float *cos_tab, const float *sin_tab, int max_pos,
                                     const float *phi, int mode, int b, int group,
                                     void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                                     double *moments, void *workspace, size_t workspace_bytes,
                                     int *status, qkq_stream_t stream);

/*
 * qkq_transform_quantize_qkv — qkq_transform_quantize with the value rows in the same launch.
 *   Q and K exactly as qkq_transform_quantize (same arguments, outputs and bits).  V gets
 *   no RoPE and no pair rotation: each value row is turned by the full-head normalised
 *   Hadamard, V~ = V H_{d_h} / sqrt(d_h) (the value rotation of "LLM旋转量化笔记" §3.2.2,
 *   which flattens the value cache; its H on the attention output folds into the output
 *   projection), then quantised like K with the same group.  fp32 sequence of a value
 *   row: bf16 -> fp32, butterflies at strides 1 .. d_h/2, * fp32(1/sqrt(d_h)), the K
 *   quantiser of qkq_transform_quantize.
 * Arguments (beyond qkq_transform_quantize's)
 *   v_bf16 [T][Hkv][d_h]: value rows (device, 16-byte aligned).
 *   v_codes [T][Hkv][d_h/2], v_scales_f16 [T][Hkv][d_h/group]: as k_codes / k_scales.
 *   v_transformed_f32 [T][Hkv][d_h]: nullable fp32 V~.
 *   Status bits 1 and 2 cover the value rows too.
 * Returns as qkq_transform_quantize; QKQ_ERR_ARG for a null v, v_codes or v_scales
 *   when T > 0.
 */
int qkq_transform_quantize_qkv(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                               const int32_t *pos, int64_t T, int Hq, int Hkv, int d_h,
                               int rope_style, const float *cos_tab, const float *sin_tab,
                               int max_pos, const float *phi, int mode, int b, int group,
                               void *q_out_bf16, uint8_t *k_codes, void *k_scales_f16,
                               uint8_t *v_codes, void *v_scales_f16, float *k_transformed_f32,
                               float *v_transformed_f32, int *status, qkq_stream_t stream);

/*
 * qkq_transform_quantize_tc — the Hadamard modes with the mixing on the tensor cores.
 *   Same arguments, outputs and status bits as qkq_transform_quantize, for modes
 *   QKQ_MODE_HADAMARD, QKQ_MODE_PAIRWISE_HADAMARD and QKQ_MODE_BLOCK_HADAMARD (others:
 *   QKQ_ERR_UNSUPPORTED) and one-row-per-position tables (a split table:
 *   QKQ_ERR_UNSUPPORTED); q_out must not overlap q (no in-place).  The mixing of each
 *   128-row tile is the product with (I (x) H_b) on tcgen05 tensor cores ("Methodology":
 *   the normalised Hadamard is an orthogonal matrix applied per head; "Core contributions":
 *   support b), with each post-RoPE fp32 row split into two bf16 halves
 *   (x = hi + lo to 16 significant bits) and fp32 accumulation.
 *   Numerics: NOT the bit-exact fp32 sequence of qkq_transform_quantize.  Every K~ and
 *   Q~ value is within 2^-14 * ||row||_2 of the exact fp64 transform of the fp32 RoPE
 *   output (split error 2^-16 per element plus the fp32 accumulation), so codes can
 *   differ from the butterfly's only where |x/s| lies that close to a rounding midpoint.
 *   This variant exists to measure tensor cores against the butterfly on this path.
 */
int qkq_transform_quantize_tc(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                              int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                              const float *cos_tab, const float *sin_tab, int max_pos,
                              const float *phi, int mode, int b, int group, void *q_out_bf16,
                              uint8_t *k_codes, void *k_scales_f16, float *k_transformed_f32,
                              int *status, qkq_stream_t stream);

/*
 * qkq_attention_scores — KV4 consumer: attention logits against the int4 key cache.
 *   S[tq][h][tk] = sum_c q~[tq][h][c] * scale[tk][h/(Hq/Hkv)][c/group] * code[tk][h/(Hq/Hkv)][c]
 *   for transformed queries q~ (the bf16 Q~ of qkq_transform_quantize) and the packed codes
 *   and fp16 scales it wrote.  The online rotation cancels in this product
 *   ("LLM旋转量化笔记" §3.2.1: Q~ K~^T = RoPE(Q) RoPE(K)^T for an orthogonal per-head map), so
 *   S approximates RoPE(Q) RoPE(K)^T up to the quantisation error.  No softmax scale.
 *   fp32 arithmetic: per group the products q * code (exact) summed, then scale * sum added;
 *   within (d_h + d_h/group + 2) * 2^-24 * sum_c |q~_c| |scale * code_c| of the exact value.
 * Arguments
 *   q_bf16 [Tq][Hq][d_h] (device), Tq <= 65535.
 *   k_codes [Tk][Hkv][d_h/2] (device, 16-byte aligned), k_scales_f16 [Tk][Hkv][d_h/group].
 *   Hq / Hkv in {1, 2, 3, 4, 6, 8} (grouped-query heads), d_h in {64, 128}, group as
 *   quantised.
 *   scores [Tq][Hq][Tk] fp32 (device, written).
 * Returns QKQ_OK (Tq == 0 or Tk == 0: nothing), or a negative qkq_err.
 */
int qkq_attention_scores(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                         const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h, int group,
                         float *scores, qkq_stream_t stream);

/*
 * qkq_attention_scores_tc — the same logits with the per-group sums on the tensor cores.
 *   For each key head the sums over a group's channels, sum_c q~[tq][h][c] * code[tk][c], are
 *   one matrix product (cached tokens x query rows, contraction over the channels): the
 *   codes (-7 .. 7) and the bf16 queries are bf16 operands of tcgen05.mma, every product is
 *   exact and the accumulator fp32; the group scales are applied afterwards in fp32 exactly
 *   as by qkq_attention_scores (scale_g times the group's sum, added in group order).  The
 *   tensor cores add a group's products in an order of their own: each score is within
 *   2 (d_h + d_h/group + 2) 2^-24 sum_c |q~_c| |scale * code_c| of the exact value.
 *   Query tokens are taken in blocks of at most 256 / (d_h/group) query rows per launch.
 * Arguments: as qkq_attention_scores (q_bf16 16-byte aligned here), plus
 *   status: nullable device int, QKQ_STATUS_TIMEOUT OR-ed in if the kernel's time-bounded
 *   wait for the tensor cores gave up (the affected scores are then unspecified).
 * Returns QKQ_OK (Tq == 0 or Tk == 0: nothing), or a negative qkq_err.
 */
int qkq_attention_scores_tc(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                            const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h,
                            int group, float *scores, int *status, qkq_stream_t stream);

/*
 * qkq_attention_scores_mma — the same logits on the tensor cores with register operands,
 *   for decode-sized query blocks.
 *   Each warp takes 16 cached tokens of one key head at a time, unpacks their codes (-7 .. 7,
 *   exact in bf16) straight into the A fragments of warp-level bf16 MMAs (m16n8k16, fp32
 *   accumulators) against the query rows of the block (B, from shared memory), one
 *   accumulator per scale group, then applies the group scales in fp32 exactly as
 *   qkq_attention_scores does (scale_g times the group's sum, added in group order).  The key
 *   cache is read once per block of at most 64 query rows (query tokens x Hq/Hkv heads), so
 *   one decode token reads it once.  Numerics: products exact, a group's products added by
 *   the tensor cores in an order of their own; each score is within
 *   2 (d_h + d_h/group + 2) 2^-24 sum_c |q~_c| |scale * code_c| of the exact value.
 * Arguments: as qkq_attention_scores (q_bf16 2-byte aligned), and Tk * Hkv < 2^32
 *   (QKQ_ERR_SHAPE otherwise).  No waits, no status.
 * Returns QKQ_OK (Tq == 0 or Tk == 0: nothing), or a negative qkq_err.
 */
int qkq_attention_scores_mma(const void *q_bf16, int64_t Tq, const uint8_t *k_codes,
                             const void *k_scales_f16, int64_t Tk, int Hq, int Hkv, int d_h,
                             int group, float *scores, qkq_stream_t stream);

/*
 * qkq_accumulate_moments — calibration side path, step 1.
 *   Adds into moments[s][k][0..5] = (n, Sa, Sb, Saa, Sab, Sbb) the raw (uncentred)
 *   accumulators of the post-RoPE, pre-mixing values of pair k (a = first channel,
 *   b = second) for stream s (0 = Q, 1 = K), pooled over all heads and tokens of the
 *   call ("Estimation strategies": raw Q and K moment accumulators pooled across
 *   heads before centring; "Optimisation objective": the position-averaged
 *   surrogate).  Products of fp32 values are exact in fp64; the sums are fp64 in a
 *   fixed order (deterministic for a given device and sizes).  One streaming pass over
 *   Q and K; a second, small kernel adds the per-CTA partial sums.
 * Arguments: q/k/pos/T/Hq/Hkv/d_h/rope_style/cos_tab/sin_tab/max_pos as above.
 *   moments: device double [2][d_h/2][6], ADDED TO (zero it to start a calibration;
 *   call repeatedly to add batches).  workspace: device scratch of at least
 *   qkq_moments_workspace_bytes(T, Hq, Hkv, d_h) bytes, 16-byte aligned, contents
 *   irrelevant, reused freely between calls on the same stream.
 *   status: nullable, QKQ_STATUS_POS_RANGE / QKQ_STATUS_NONFINITE.
 */
int qkq_accumulate_moments(const void *q_bf16, const void *k_bf16, const int32_t *pos, int64_t T,
                           int Hq, int Hkv, int d_h, int rope_style, const float *cos_tab,
                           const float *sin_tab, int max_pos, double *moments, void *workspace,
                           size_t workspace_bytes, int *status, qkq_stream_t stream);

/*
 * qkq_accumulate_moments_noalloc — qkq_accumulate_moments for callers that cannot
 *   allocate device memory at the point where they calibrate: for example an
 *   inference-runtime plugin whose per-batch enqueue step is not allowed to allocate,
 *   or a serving engine that keeps all free HBM in its own pool and forbids ad-hoc
 *   allocations.  The paper has no counterpart: it is a deployment variant of the same
 *   step, with the same arguments and results, except that the per-CTA partial sums
 *   live in a fixed 5 MiB array inside the library (held on every GPU that loads the
 *   library until the process exits) instead of a caller workspace.  Allocates nothing
 *   (no cudaMalloc / cudaFree).
 * Limit: the array holds the partial sums of the largest grid the moments kernel runs
 *   (1024 CTAs x 2 x d_h/2 x 5 doubles at d_h = 128).  This variant launches the same grid
 *   as qkq_accumulate_moments, so its results are bit for bit the same, and since the
 *   partial sums depend on the grid and not on T, every batch size fits.  The call still
 *   checks the planned partial sums against the array and would refuse with
 *   QKQ_ERR_WORKSPACE, before any launch, if they did not fit.
 * The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the process; make
 *   that first call before any stream capture.  The cached address belongs to the device's
 *   primary context: after cudaDeviceReset (or from another driver context) it is stale,
 *   so such a caller must not use this entry point afterwards in the same process.  All
 *   calls share the array, which keeps the last call's partial sums (every call overwrites
 *   them in full): calls whose kernels overlap on the GPU race on it and must be
 *   serialised by the caller.
 */
int qkq_accumulate_moments_noalloc(const void *q_bf16, const void *k_bf16, const int32_t *pos,
                                   int64_t T, int Hq, int Hkv, int d_h, int rope_style,
                                   const float *cos_tab, const float *sin_tab, int max_pos,
                                   double *moments, int *status, qkq_stream_t stream);

/*
 * qkq_solve_angles — calibration side path, step 2 ("Optimisation objective").
 *   From the accumulators, the estimator's 2x2 covariance [[A, C], [C, D]] per pair
 *   (POOLED: sums of Q and K, centred once; K_ONLY: K; BALANCED: mean of the two
 *   streams' normalised uncentred moments, then centred) and the angle that
 *   minimises the larger channel variance:  phi*_k = atan2(A - D, 2C) / 2 reduced
 *   into (-pi/4, pi/4]; isotropic pairs (|A-D| + 2|C| <= 1e-12 (A+D)) get 0.
 *   The minimum of the larger variance is (A + D)/2.  Computed in fp64 on the device.
 *   A pair whose estimator needs a stream with no observations (n = 0: K_ONLY without
 *   keys, BALANCED with either stream empty, POOLED with both) has no covariance: it gets
 *   phi = 0 (the identity rotation), min_maxvar NaN, and QKQ_STATUS_EMPTY_STREAM is set.
 * Arguments: moments device double [2][d_h/2][6]; phi device float [d_h/2] (out);
 *   min_maxvar: nullable device double [d_h/2], the attained larger variance;
 *   status: nullable device int, QKQ_STATUS_EMPTY_STREAM OR-ed in.
 */
int qkq_solve_angles(const double *moments, int d_h, int estimator, float *phi,
                     double *min_maxvar, int *status, qkq_stream_t stream);

/*
 * qkq_dequant_error_workspace_bytes — scratch needed by qkq_dequant_error.
 */
size_t qkq_dequant_error_workspace_bytes(int64_t T, int Hkv, int d_h, int group);

/*
 * qkq_dequant_error — measurement path ("Core contributions" / "Results": K range
 *   and relative quantisation error along the mixing support).
 *   Compares the given transformed keys K~ with their dequantised codes
 *   K^ = fp16 scale * code, group by group, and writes
 *     stats[0] = sum (K~ - K^)^2     stats[1] = sum K~^2
 *     stats[2] = sum over groups of max|K~|      stats[3] = sum over groups of (max - min)
 *     stats[4] = max over groups of max|K~|      stats[5] = number of groups
 *   in fp64 (overwritten, deterministic for a device and sizes).  qkq_dequant_summary turns
 *   them into the K range and the relative error.  The codes may come from any producer:
 *   qkq_transform_quantize (its k_transformed_f32 output), qkq_transform_quantize_tc,
 *   value rows, or another implementation of the quantiser.
 *   Arithmetic: per lane and group the terms (K~ - s c)/s and K~/s are squared and summed
 *   in fp32, weighted by s^2 in fp64 (s the fp16 scale; 1 for a scale of 0 or Inf), so
 *   stats[0] and stats[1] are within 24 * 2^-24 relative of the exact sums; stats[2..5]
 *   are fp64 sums of fp32 values (exact maxima).
 * Arguments
 *   k_transformed_f32 [T][Hkv][d_h]: fp32 K~ (device, 16-byte aligned).
 *   k_codes [T][Hkv][d_h/2] (4-byte aligned), k_scales_f16 [T][Hkv][d_h/group]: the
 *     quantised K (device), packed as qkq_transform_quantize writes them.
 *   T >= 0 (T == 0 writes zeros; the three inputs may then be NULL), Hkv >= 1,
 *     d_h in {64, 128}, group in {32, 64, 128} dividing d_h.
 *   stats: device double [6] (out).
 *   workspace: device scratch of at least qkq_dequant_error_workspace_bytes(T, Hkv, d_h,
 *     group) bytes, 16-byte aligned.
 *   status: nullable device int; QKQ_STATUS_NONFINITE if a sum came out NaN or Inf.
 * Returns QKQ_OK or a negative qkq_err (nothing launched on error).
 */
int qkq_dequant_error(const float *k_transformed_f32, const uint8_t *k_codes,
                      const void *k_scales_f16, int64_t T, int Hkv, int d_h, int group,
                      double *stats, void *workspace, size_t workspace_bytes, int *status,
                      qkq_stream_t stream);

/*
 * qkq_dequant_summary — HOST function: the measurement's summary figures from a stats[6]
 *   record of qkq_dequant_error / qkq_dequant_error_recompute /
 *   qkq_transform_quantize_stats, copied to the host ("Core contributions": the K range
 *   is the tokenwise group range that sets the step; the relative quantisation error):
 *     summary[0] = K range = stats[2] / stats[5]   (mean over groups of max|K~|)
 *     summary[1] = relative error = sqrt(stats[0] / stats[1])   (||K~ - K^||_F / ||K~||_F)
 *     summary[2] = mean group range = stats[3] / stats[5]   (mean of max - min)
 *     summary[3] = largest group max|K~| = stats[4]
 *   No groups: summary[0] = summary[2] = 0.  stats[1] == 0: summary[1] = 0 if stats[0] == 0,
 *   else +Inf.
 * Arguments: stats_host: HOST double [6]; summary_host: HOST double [4] (out).
 * Returns QKQ_OK or QKQ_ERR_ARG (a null pointer).
 */
int qkq_dequant_summary(const double *stats_host, double *summary_host);

/*
 * qkq_dequant_error_recompute — qkq_dequant_error for codes that qkq_transform_quantize
 *   produced, without a materialised K~: recomputes K~ from k_bf16 exactly as
 *   qkq_transform_quantize does (same fp32 sequence, same arguments; bit-identical values)
 *   and writes the same stats[6] with the same arithmetic.  It reads 2 bytes per K value
 *   instead of 4 and needs no fp32 K~ output from the transform.
 * Arguments: k/pos/T/Hkv/d_h/rope_style/tables/phi/mode/b/group as for
 *   qkq_transform_quantize; k_codes (16-byte aligned here: it is staged with bulk
 *   copies) / k_scales_f16: the quantised K to measure (device); stats: device double
 *   [6] (out); workspace: device scratch of at least
 *   qkq_dequant_error_workspace_bytes(...) bytes, 16-byte aligned.
 */
int qkq_dequant_error_recompute(const void *k_bf16, const int32_t *pos, int64_t T, int Hkv,
                                int d_h, int rope_style, const float *cos_tab,
                                const float *sin_tab, int max_pos, const float *phi, int mode,
                                int b, int group, const uint8_t *k_codes,
                                const void *k_scales_f16, double *stats, void *workspace,
                                size_t workspace_bytes, int *status, qkq_stream_t stream);

/*
 * qkq_selftest_bounded_wait — test hook for the failure path of the on-chip waits.
 *   Launches one warp that waits on an mbarrier nothing will complete; the wait gives up
 *   after limit_ns (at most 100 ms) by the global timer, and the kernel ORs
 *   QKQ_STATUS_TIMEOUT into *status and returns — the same path a pipeline stage whose
 *   copies never landed takes in every streaming kernel (there with a 2 s limit).  No fault,
 *   no hang; the context stays usable.  No counterpart in the paper.
 * Returns QKQ_OK, QKQ_ERR_ARG (null status, limit 0 or above 100 ms), QKQ_ERR_ALIGN.
 */
int qkq_selftest_bounded_wait(unsigned long long limit_ns, int *status, qkq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QKQ_H */

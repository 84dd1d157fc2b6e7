// Fused post-RoPE Q/K transform + dynamic KV4 quantisation (sm_100a).
//
// One kernel does, per token and head: bf16 load, RoPE from the fp32 cos/sin table,
// the head-shared pair rotation, the fast Walsh-Hadamard butterflies, the Q~ bf16
// store, and for K the group absmax, round, pack and int4 + fp16 scale store —
// one HBM read and one HBM write per element.  (Method: paper summary "When Local
// Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for Dynamic 4-Bit
// Quantisation", "Methodology" and "Core contributions"; online FWHT: "LLM旋转量化笔记"
// §3.3; quantiser: same notes §1.2.)
//
// Data movement.  Each warp runs its own pipeline of S shared-memory stages; a stage
// holds one token: its Hq query rows, Hkv key rows (contiguous in HBM, so two bulk
// copies) and the token's cos and sin table rows.  Lane 0 issues the bulk copies
// (cp.async.bulk, no multicast) S tokens ahead onto a per-stage mbarrier; all lanes
// wait on it with a time bound.  Tokens are dealt to warps round-robin over a
// persistent grid (a multiple of the SM count).  Positions are prefetched 32 tokens
// at a time, one per lane, so the table row address never waits on a load.
//
// Compute.  A quad of lanes owns a row (rowops.cuh): 8 rows per warp step, with the
// token's RoPE table entries held in registers across its rows; in the pairwise modes each
// row then takes the pair rotation with the angles' cos/sin from shared memory.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "moments.cuh"
#include "pipeline.cuh"
#include "rowops.cuh"

namespace qkq {

namespace {

#ifndef QKQ_TQ_WARPS
#define QKQ_TQ_WARPS 4
#endif
constexpr int TQ_WARPS = QKQ_TQ_WARPS;
constexpr int TQ_MAX_STAGES = 4;
constexpr int TQ_BAR_BYTES = (TQ_WARPS * TQ_MAX_STAGES * 8 + 127) / 128 * 128;  // mbarriers
constexpr int TQ_RED_BYTES = (TQ_WARPS * 6 * 8 + 127) / 128 * 128;  // statistics reduction

// CTAs per SM a kernel instance is built and launched for.  Stages are sized so that many
// CTAs share an SM (at the 8B shape: one stage per warp).  The pairwise modes without the
// statistics fit in 128 registers without spills and run four CTAs (16 warps) per SM
// (pairwise + Hadamard at the 8B shape: 0.455 ms at four and at three, 0.513 ms at two);
// the other modes run three.  The instances with fused statistics (the quantiser and the
// statistics in one pass, quantize_row_stats) are built for three CTAs: at most 168
// registers, no spills at any group size (without the cap they took up to 232 registers and
// only two fitted: Hadamard 0.468 against 0.526 ms, block b = 16 0.414 against 0.470 ms at
// the 8B shape).
// The row-split instances (few tokens: latency, not occupancy) keep their registers too.
// At d_h = 64 the full-head and RoPE-only instances without the statistics (at most 113
// registers anyway) run four CTAs too: 0.215 vs 0.230 ms (Hadamard) and 0.220 vs 0.230 ms
// (RoPE only) on 131 072 tokens of the 1B shape; the block modes there measured slower at
// four (0.240 vs 0.203 ms at b = 16) and keep three.
template <int DH, int NMIX, bool PAIRROT, bool MEASURE, bool PARTS = false>
constexpr int tq_ctas_per_sm()
{
    const bool four = PAIRROT || (DH == 64 && (NMIX == 1 || NMIX == DH));
    return (four && !MEASURE && !PARTS) ? 4 : 3;
}

// The register cap of an instance (__launch_bounds__ minimum CTAs per SM): four-CTA instances
// at 128 registers, statistics instances at 168 (see above), none for the rest.
template <int DH, int NMIX, bool PAIRROT, int G, bool MEASURE, bool PARTS>
constexpr int tq_min_blocks()
{
    return tq_ctas_per_sm<DH, NMIX, PAIRROT, MEASURE, PARTS>() == 4
               ? 4
               : (MEASURE ? 3 : 1);
}

// NGRP groups of 8 query rows (rows r0 + 8*g + rq; the stage holds rows from row_base on):
// load, RoPE, the pair rotation (pairwise modes), FWHT, bf16 store.
template <class L, int NMIX, bool PAIRROT, int NGRP, class PC>
__device__ __forceinline__ void query_groups(const uint8_t *st, int row_base, int r0, int Hq,
                                             int rq, int l, const float2 (&C)[L::NT],
                                             const float2 (&S)[L::NT], const PC &pc,
                                             float kappa, uint8_t *qout_token, int &flags)
{
    constexpr int ROWB = L::NCH * 8;
    float2 V[NGRP][L::NV];
#pragma unroll
    for (int g = 0; g < NGRP; ++g) {
        const int row = r0 + 8 * g + rq;  // staged from row_base on
        load_row_bf16<L>(V[g], st + ((row < Hq ? row : Hq - 1) - row_base) * ROWB, l);
    }
#pragma unroll
    for (int g = 0; g < NGRP; ++g) {
        rotate_pairs<L>(V[g], C, S);
        if (PAIRROT) pc.turn(V[g]);
    }
#pragma unroll
    for (int g = 0; g < NGRP; ++g) fwht<L, NMIX>(V[g], l, kappa);
#pragma unroll
    for (int g = 0; g < NGRP; ++g) {
        const int row = r0 + 8 * g + rq;
        if (row < Hq && QKQ_IN_BOUNDS(row >= 0, flags))
            store_row_bf16<L>(V[g], qout_token + row * ROWB, l);
    }
}

// Quantise one transformed row held by a quad and store its codes (and fp32 copy when
// asked); the quad's lanes l < groups store the fp16 scales.  Rows past the end (valid ==
// false) take part in the quad's shuffles and store nothing.
// r[g] receives every group's 7/amax and shat_mine the stored (fp16) scale of this lane's
// group l % groups, as fp32 (for the measurement statistics).
template <class L, int G>
__device__ __forceinline__ void quantize_store(const float2 (&V)[L::NV], bool valid, int64_t gr,
                                               uint8_t *codes, uint16_t *scales, float *f32,
                                               int l, int lane, int &flags,
                                               float (&r)[Groups<L, G>::NG], float &shat_mine,
                                               int64_t rows = 0)
{
    using GR = Groups<L, G>;
    constexpr int DH = L::NCH * 4;
    // rows: T * Hkv, the output rows (checked in the bounds-checking build only)
    if (valid) valid = QKQ_IN_BOUNDS(gr >= 0 && gr < rows, flags);
    if (f32 != nullptr && valid) store_row_f32<L>(V, f32 + gr * DH, l);
    uint32_t words[L::NJ];
    float s_mine;
    int qf = 0;
    quantize_row<L, G>(V, l, lane, words, s_mine, qf, r);
    const uint16_t hb = __half_as_ushort(__float2half_rn(s_mine));
    shat_mine = __half2float(__ushort_as_half(hb));
    if (valid) {
        flags |= qf;
        uint32_t *crow = reinterpret_cast<uint32_t *>(codes + gr * (DH / 2));
#pragma unroll
        for (int j = 0; j < L::NJ; ++j) crow[j * 4 + l] = words[j];
        if (l < GR::NG) {
            if ((hb & 0x7fffu) == 0x7c00u && !(qf & ST_NONFINITE)) flags |= ST_SCALE_OVERFLOW;
            scales[gr * GR::NG + l] = hb;
        }
    }
}

// quantize_store with the measurement statistics of the row added to st in the same pass
// (quantize_row_stats); no fp32 copy.
template <class L, int G>
__device__ __forceinline__ void quantize_store_stats(const float2 (&V)[L::NV], bool valid,
                                                     int64_t gr, uint8_t *codes,
                                                     uint16_t *scales, int l, int lane,
                                                     int &flags, RowStats &st, int64_t rows)
{
    using GR = Groups<L, G>;
    constexpr int DH = L::NCH * 4;
    if (valid) valid = QKQ_IN_BOUNDS(gr >= 0 && gr < rows, flags);
    uint32_t words[L::NJ];
    uint16_t hb;
    int qf = 0;
    quantize_row_stats<L, G>(V, l, lane, valid, words, hb, qf, st);
    if (valid) {
        flags |= qf;
        uint32_t *crow = reinterpret_cast<uint32_t *>(codes + gr * (DH / 2));
#pragma unroll
        for (int j = 0; j < L::NJ; ++j) crow[j * 4 + l] = words[j];
        if (l < GR::NG) {
            if ((hb & 0x7fffu) == 0x7c00u && !(qf & ST_NONFINITE)) flags |= ST_SCALE_OVERFLOW;
            scales[gr * GR::NG + l] = hb;
        }
    }
}

// One staged unit (a whole token, or a row-split part of one): RoPE from its table rows at
// ctab, then the pair rotation in the pairwise modes, the mixing, and
//   query row groups q_begin .. q_end - 1 (rows staged at q_rows from row q_begin on): Q~ bf16;
//   k_rows (nullable): every K row, the quantiser (and its statistics when MEASURE);
//   v_rows (nullable): every value row, full-head Hadamard and the quantiser.
// Every lane of the warp takes part.
template <class L, int NMIX, bool PAIRROT, int G, bool MEASURE, class PC>
__device__ __forceinline__ void transform_unit(const TransformParams &p, const uint8_t *q_rows,
                                               int q_begin, int q_end, const uint8_t *k_rows,
                                               const uint8_t *v_rows, const float *ctab,
                                               int64_t t, const PC &pc, int l, int rq,
                                               int lane, int &flags, RowStats &stats)
{
    using GR = Groups<L, G>;
    constexpr int DH = L::NCH * 4;
    constexpr int P = DH / 2;
    constexpr int ROWB = DH * 2;
    const float kappa = p.kappa;
    float2 C[L::NT], Sn[L::NT];
    load_rope<L>(C, Sn, ctab, P, p.split, l);

    // query rows: transform, store bf16, one group of 8 rows at a time (rows past Hq are
    // computed on a clamped row, keeping every lane in the shuffles, and not stored; two
    // interleaved groups measured slower: 531 vs 478 us per launch)
    uint8_t *qout_token = reinterpret_cast<uint8_t *>(p.q_out) + t * p.Hq * ROWB;
    for (int r0 = q_begin; r0 < q_end; r0 += 8)
        query_groups<L, NMIX, PAIRROT, 1>(q_rows, q_begin, r0, p.Hq, rq, l, C, Sn, pc,
                                          kappa, qout_token, flags);
    // key rows: transform, quantise, store codes and scales
    if (k_rows != nullptr) {
        for (int r0 = 0; r0 < p.Hkv; r0 += 8) {
            const int row = r0 + rq;
            const int rowc = row < p.Hkv ? row : p.Hkv - 1;
            float2 V[L::NV];
            load_row_bf16<L>(V, k_rows + rowc * ROWB, l);
            rotate_pairs<L>(V, C, Sn);
            if (PAIRROT) pc.turn(V);
            fwht<L, NMIX>(V, l, kappa);
            if (MEASURE) {  // the quantiser and the statistics in one pass
                quantize_store_stats<L, G>(V, row < p.Hkv, t * p.Hkv + row, p.k_codes,
                                           p.k_scales, l, lane, flags, stats, p.T * p.Hkv);
            } else {
                float r[GR::NG], shat_mine;
                quantize_store<L, G>(V, row < p.Hkv, t * p.Hkv + row, p.k_codes, p.k_scales,
                                     p.k_f32, l, lane, flags, r, shat_mine, p.T * p.Hkv);
            }
        }
    }
    // value rows (when given): the full-head normalised Hadamard and no RoPE, then the
    // same quantiser ("LLM旋转量化笔记" §3.2.2: V~ = V H_head flattens the value cache;
    // the H_head on the attention output folds into the output projection)
    if (v_rows != nullptr) {
        for (int r0 = 0; r0 < p.Hkv; r0 += 8) {
            const int row = r0 + rq;
            const int rowc = row < p.Hkv ? row : p.Hkv - 1;
            float2 V[L::NV];
            load_row_bf16<L>(V, v_rows + rowc * ROWB, l);
            fwht<L, DH>(V, l, p.kappa_v);
            float r[GR::NG], shat_mine;
            quantize_store<L, G>(V, row < p.Hkv, t * p.Hkv + row, p.v_codes, p.v_scales,
                                 p.v_f32, l, lane, flags, r, shat_mine, p.T * p.Hkv);
        }
    }
}

// A whole staged token (Q rows, then K rows, then table rows, then the extra block).
template <class L, int NMIX, bool PAIRROT, int G, bool MEASURE, class PC>
__device__ __forceinline__ void transform_token(const TransformParams &p, const uint8_t *st,
                                                uint32_t qbytes, uint32_t kbytes,
                                                uint32_t extra_off, int64_t t,
                                                const PC &pc, int l, int rq, int lane,
                                                int &flags, RowStats &stats)
{
    transform_unit<L, NMIX, PAIRROT, G, MEASURE>(
        p, st, 0, p.Hq, st + qbytes, p.v != nullptr ? st + extra_off : nullptr,
        reinterpret_cast<const float *>(st + qbytes + kbytes), t, pc, l, rq, lane, flags,
        stats);
}

// Head-shared pair rotation table in shared memory: cos and sin of each angle, each the fp32
// rounding of the fp64 function of the fp32 angle.  Thread i < P evaluates cos of angle i
// and thread P + i its sin, so that no thread waits for two fp64 functions; the angle is
// loaded (pair_angle_load) before the pipeline set-up to overlap the two latencies.  Every
// lane then reads its pairs' entries into registers (PairCoeffs).
template <int P>
__device__ __forceinline__ float pair_angle_load(const float *phi)
{
    return threadIdx.x < 2 * P ? __ldg(phi + (threadIdx.x % P)) : 0.0f;
}

template <int P>
__device__ __forceinline__ void pair_table_fill(float ph, float *phi_tab)
{
    const int i = threadIdx.x;
    if (i < P) {
        phi_tab[i] = static_cast<float>(cos(static_cast<double>(ph)));
    } else if (i < 2 * P) {
        phi_tab[i] = static_cast<float>(sin(static_cast<double>(ph)));
    }
}

// PARTS: the warps take row-split units (p.parts per token) instead of whole tokens; its own
// instances, so that the whole-token ones compile exactly as without it.
template <int DH, int NMIX, bool PAIRROT, int G, int STYLE, bool MEASURE, bool PARTS>
__global__ void __launch_bounds__(TQ_WARPS * 32, (tq_min_blocks<DH, NMIX, PAIRROT, G, MEASURE, PARTS>()))
    k_transform_quant(const TransformParams p)
{
    using L = Layout<DH, STYLE>;
    constexpr int P = DH / 2;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);                    // [WARPS][MAX_STAGES]
    float *phi_tab = reinterpret_cast<float *>(smem + TQ_BAR_BYTES);       // [2][P]
    double *red = reinterpret_cast<double *>(smem + TQ_BAR_BYTES + TQ_PHI_BYTES);  // [WARPS][6]
    uint8_t *stage_mem = smem + TQ_BAR_BYTES + TQ_PHI_BYTES + TQ_RED_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane & 3, rq = lane >> 2;
    int flags = 0;
    RowStats stats;  // measurement statistics of the K rows, when asked for
    static_assert(TQ_WARPS * 32 >= DH, "one thread per pair-table entry");
    // launched early behind the previous kernel of the stream (it may have written q, k,
    // pos or phi): wait for it before any read; the next launch may start early in turn
    wait_prior_grid();
    const float ph = PAIRROT ? pair_angle_load<P>(p.phi) : 0.0f;
    TokenPipe pipe;
    pipe.start(stage_mem + static_cast<size_t>(warp) * p.stages * p.stage_bytes,
               bars + warp * TQ_MAX_STAGES, p.stages, p.stage_bytes,
               static_cast<int64_t>(blockIdx.x) * TQ_WARPS + warp,
               static_cast<int64_t>(gridDim.x) * TQ_WARPS, p.T, p.Hq, p.Hkv, DH, p.q, p.k, p.cos_t,
               p.sin_t, p.pos, p.max_pos, p.split, flags, true, p.v,
               p.v != nullptr ? static_cast<uint32_t>(p.Hkv) * DH * 2 : 0u, PARTS ? p.parts : 1,
               true);  // last token first: the moment pass before it read the batch in order
    const uint32_t qbytes = pipe.qbytes, kbytes = pipe.kbytes;

    // the pair rotation's coefficients, in registers for the whole launch (pairwise modes)
    PairCoeffs<L> pc;
    if (PAIRROT) {
        pair_table_fill<P>(ph, phi_tab);
        __syncthreads();
        pc.load(phi_tab, P, lane & 3);
    }

    for (int64_t n = 0; n < pipe.ntok; ++n) {
        const uint8_t *st = pipe.wait(n, flags);
        if (st == nullptr) break;  // bounded wait gave up (all lanes together)
        if (!PARTS) {
            transform_token<L, NMIX, PAIRROT, G, MEASURE>(p, st, qbytes, kbytes, pipe.extra_offset(),
                                                           pipe.token(n), pc, l, rq, lane,
                                                           flags, stats);
        } else {  // row-split unit: one group of 8 query rows, or every key (and value) row
            const int part = pipe.part(n);
            const float *ctab = reinterpret_cast<const float *>(st + pipe.unit_table_offset(part));
            if (part < pipe.nqp)
                transform_unit<L, NMIX, PAIRROT, G, MEASURE>(p, st, 8 * part, 8 * part + 8, nullptr,
                                                             nullptr, ctab, pipe.token(n), pc,
                                                             l, rq, lane, flags, stats);
            else
                transform_unit<L, NMIX, PAIRROT, G, MEASURE>(
                    p, st, 0, 0, st, p.v != nullptr ? st + pipe.unit_extra_offset(part) : nullptr,
                    ctab, pipe.token(n), pc, l, rq, lane, flags, stats);
        }
        pipe.release(n, flags);
    }
    allow_next_grid();
    if (MEASURE)
        reduce_row_stats(stats, red, TQ_WARPS, p.stat_partials + static_cast<int64_t>(blockIdx.x) * 6,
                         flags);
    if (flags && p.status) atomicOr(p.status, flags);
}

// ---- the calibrating transform: the transform and the calibration moments of the same
// tokens in one pass -------------------------------------------------------------------
//
// The moments are of post-RoPE, pre-mixing values, so they do not depend on the angles the
// transform uses: a calibrating pass transforms with the current angles and accumulates
// the moments for the next solve, reading Q and K from HBM once.  Warp roles in a CTA of
// 8 warps: warps 0-3 run the transform exactly as k_transform_quant (each owns its token
// pipeline: stages, copies, "full" barriers); warp 4 + w reads warp w's staged tokens and
// accumulates the moments with the moments kernel's code, then arrives on the stage's
// "empty" barrier; warp w refills a stage only after that arrival.  Every wait is bounded.
constexpr int TCAL_WARPS = 2 * TQ_WARPS;
constexpr int TCAL_BAR_BYTES = (2 * TQ_WARPS * TQ_MAX_STAGES * 8 + 127) / 128 * 128;  // full, empty
constexpr int TCAL_CTAS = 2;  // CTAs per SM: 128 registers per thread, 16 warps
constexpr int TCAL_RED_BYTES = moments_red_bytes(TQ_WARPS);  // the moment warps' reduction

template <int DH, int NMIX, bool PAIRROT, int G, int STYLE>
__global__ void __launch_bounds__(TCAL_WARPS * 32, TCAL_CTAS)
    k_transform_calib(const TransformParams p, double *mom_partials)
{
    using L = Layout<DH, STYLE>;
    using ML = MomentLanes<DH>;
    constexpr int P = DH / 2;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);            // [TQ_WARPS][MAX_STAGES]
    uint64_t *empty = full + TQ_WARPS * TQ_MAX_STAGES;             // [TQ_WARPS][MAX_STAGES]
    float *phi_tab = reinterpret_cast<float *>(smem + TCAL_BAR_BYTES);  // [2][P]
    double *red = reinterpret_cast<double *>(smem + TCAL_BAR_BYTES + TQ_PHI_BYTES);  // moments
    uint8_t *stage_mem = smem + TCAL_BAR_BYTES + TQ_PHI_BYTES + TCAL_RED_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool moment_role = warp >= TQ_WARPS;
    const int w = warp & (TQ_WARPS - 1);  // the pipeline this warp works on
    int flags = 0;

    const float ph = PAIRROT ? pair_angle_load<P>(p.phi) : 0.0f;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * TQ_WARPS + w;
    const int64_t nw = static_cast<int64_t>(gridDim.x) * TQ_WARPS;
    uint8_t *my_stages = stage_mem + static_cast<size_t>(w) * p.stages * p.stage_bytes;
    TokenPipe pipe;
    if (!moment_role) {
        // barriers, position prefetch and the first copies
        pipe.start(my_stages, full + w * TQ_MAX_STAGES, p.stages, p.stage_bytes, gw, nw, p.T,
                   p.Hq, p.Hkv, DH, p.q, p.k, p.cos_t, p.sin_t, p.pos, p.max_pos, p.split, flags);
    } else if (lane == 0) {
        for (int s = 0; s < p.stages; ++s) mbar_init(smem_addr(empty + w * TQ_MAX_STAGES + s), 1);
        fence_mbar_init();
    }
    if (PAIRROT) pair_table_fill<P>(ph, phi_tab);
    __syncthreads();  // barriers initialised (and phi staged) before either role waits
    // the transform warps' pair-rotation coefficients, re-read from shared memory for every
    // row (the role split leaves 128 registers per thread, too few to hold them)
    PairCoeffsShared<L> pc;
    if (PAIRROT && !moment_role) pc.load(phi_tab, P, lane & 3);

    const uint32_t qbytes = static_cast<uint32_t>(p.Hq) * DH * 2;
    const uint32_t kbytes = static_cast<uint32_t>(p.Hkv) * DH * 2;
    if (!moment_role) {
        const int l = lane & 3, rq = lane >> 2;
        RowStats unused;
        for (int64_t n = 0; n < pipe.ntok; ++n) {
            const uint8_t *st = pipe.wait(n, flags);
            if (st == nullptr) break;
            transform_token<L, NMIX, PAIRROT, G, false>(p, st, qbytes, kbytes, pipe.extra_offset(),
                                                        pipe.token(n), pc, l, rq, lane,
                                                        flags, unused);
            // the stage is refilled once the moment warp has read it too
            if (n + p.stages < pipe.ntok) {
                const uint32_t eb = smem_addr(empty + w * TQ_MAX_STAGES + static_cast<int>(n % p.stages));
                const uint32_t par = static_cast<uint32_t>((n / p.stages) & 1);
                if (!__all_sync(FULL_MASK, mbar_wait_bounded(eb, par))) {
                    flags |= ST_TIMEOUT;
                    pipe.drain(n + 1, n + p.stages);  // tokens issued but not yet waited for
                    break;
                }
            }
            pipe.release(n, flags);
        }
    } else {
        const int lr = lane % ML::LPR, sub = lane / ML::LPR;
        MomentAcc acc;  // only the moment warps hold the sums
        moments_clear(acc);
        const int64_t ntok = p.T > gw ? (p.T - gw + nw - 1) / nw : 0;
        for (int64_t n = 0; n < ntok; ++n) {
            const int s = static_cast<int>(n % p.stages);
            const uint32_t fb = smem_addr(full + w * TQ_MAX_STAGES + s);
            if (!__all_sync(FULL_MASK, mbar_wait_bounded(fb, static_cast<uint32_t>((n / p.stages) & 1)))) {
                flags |= ST_TIMEOUT;
                break;
            }
            const uint8_t *st = my_stages + static_cast<size_t>(s) * p.stage_bytes;
            moments_token<DH, STYLE>(st, st + qbytes,
                                     reinterpret_cast<const float *>(st + qbytes + kbytes),
                                     p.split, p.Hq, p.Hkv, lr, sub, acc);
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(empty + w * TQ_MAX_STAGES + s));
        }
        // the CTA partial, among the moment warps only (their own reduction buffer)
        moments_stash<DH>(acc, w, lr, sub, red);
        asm volatile("bar.sync 1, %0;" ::"n"(TQ_WARPS * 32) : "memory");
        moments_reduce<DH>(red, TQ_WARPS, threadIdx.x - TQ_WARPS * 32, TQ_WARPS * 32,
                           mom_partials + static_cast<int64_t>(blockIdx.x) * 2 * P * 5, flags);
    }
    if (flags && p.status) atomicOr(p.status, flags);
}

using CalibKernel = void (*)(TransformParams, double *);

using TransformKernel = void (*)(TransformParams);

// A kernel instance and the CTAs per SM it is built and launched for.
struct TqPick {
    TransformKernel kern = nullptr;
    int ctas = 0;
};

template <int DH, int NMIX, bool PAIRROT, int G, int STYLE, bool M, bool U>
TqPick tq_pick()
{
    return {k_transform_quant<DH, NMIX, PAIRROT, G, STYLE, M, U>,
            tq_ctas_per_sm<DH, NMIX, PAIRROT, M, U>()};
}

// The kernel instance for (mode, b, group, statistics, row-split units), or none.
template <int DH, int G, int STYLE, bool M, bool U>
TqPick pick_mix(int mode, int b)
{
    switch (mode) {
    case MODE_HADAMARD: return tq_pick<DH, DH, false, G, STYLE, M, U>();
    case MODE_PAIRWISE: return tq_pick<DH, 1, true, G, STYLE, M, U>();
    case MODE_PAIRWISE_HADAMARD: return tq_pick<DH, DH, true, G, STYLE, M, U>();
    case MODE_ROPE_ONLY: return tq_pick<DH, 1, false, G, STYLE, M, U>();
    case MODE_BLOCK_HADAMARD:
        switch (b) {
        case 2: return tq_pick<DH, 2, false, G, STYLE, M, U>();
        case 4: return tq_pick<DH, 4, false, G, STYLE, M, U>();
        case 8: return tq_pick<DH, 8, false, G, STYLE, M, U>();
        case 16: return tq_pick<DH, 16, false, G, STYLE, M, U>();
        case 32: return tq_pick<DH, 32, false, G, STYLE, M, U>();
        case 64: return tq_pick<DH, 64, false, G, STYLE, M, U>();
        case 128:
            if (DH == 128) return tq_pick<DH, (DH == 128 ? 128 : 64), false, G, STYLE, M, U>();
            break;
        }
        break;
    }
    return {};
}

template <int DH, int STYLE, bool M, bool U>
TqPick pick_kernel(int mode, int b, int group)
{
    switch (group) {
    case 32: return pick_mix<DH, 32, STYLE, M, U>(mode, b);
    case 64: return pick_mix<DH, 64, STYLE, M, U>(mode, b);
    case 128:
        if (DH == 128) return pick_mix<DH, (DH == 128 ? 128 : 64), STYLE, M, U>(mode, b);
        break;
    }
    return {};
}

template <int DH, int G, int STYLE>
CalibKernel pick_calib_mix(int mode, int b)
{
    switch (mode) {
    case MODE_HADAMARD: return k_transform_calib<DH, DH, false, G, STYLE>;
    case MODE_PAIRWISE: return k_transform_calib<DH, 1, true, G, STYLE>;
    case MODE_PAIRWISE_HADAMARD: return k_transform_calib<DH, DH, true, G, STYLE>;
    case MODE_ROPE_ONLY: return k_transform_calib<DH, 1, false, G, STYLE>;
    case MODE_BLOCK_HADAMARD:
        switch (b) {
        case 2: return k_transform_calib<DH, 2, false, G, STYLE>;
        case 4: return k_transform_calib<DH, 4, false, G, STYLE>;
        case 8: return k_transform_calib<DH, 8, false, G, STYLE>;
        case 16: return k_transform_calib<DH, 16, false, G, STYLE>;
        case 32: return k_transform_calib<DH, 32, false, G, STYLE>;
        case 64: return k_transform_calib<DH, 64, false, G, STYLE>;
        case 128:
            if (DH == 128) return k_transform_calib<DH, (DH == 128 ? 128 : 64), false, G, STYLE>;
            break;
        }
        break;
    }
    return nullptr;
}

template <int DH, int STYLE>
CalibKernel pick_calib(int mode, int b, int group)
{
    switch (group) {
    case 32: return pick_calib_mix<DH, 32, STYLE>(mode, b);
    case 64: return pick_calib_mix<DH, 64, STYLE>(mode, b);
    case 128:
        if (DH == 128) return pick_calib_mix<DH, (DH == 128 ? 128 : 64), STYLE>(mode, b);
        break;
    }
    return nullptr;
}

}  // namespace

// Host-side launch of the fused transform (arguments validated by the caller).
template <int DH, int STYLE>
cudaError_t transform_quant_launch(const TransformParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, cudaStream_t stream, int *ctas_used)
{
    if (ctas_used != nullptr) *ctas_used = 0;
    const bool measure = p.stat_partials != nullptr;
    TqPick pick = measure ? pick_kernel<DH, STYLE, true, false>(mode, b, group)
                          : pick_kernel<DH, STYLE, false, false>(mode, b, group);
    if (pick.kern == nullptr) return cudaErrorInvalidValue;
    const int vbytes = p.v != nullptr ? p.Hkv * DH * 2 : 0;
    int SB = token_stage_bytes(p.Hq, p.Hkv, DH, p.split, vbytes);
    TransformParams q = p;
    q.parts = 1;
    PipeLaunch pl;
    // with statistics, at most DQ_MAX_CTAS partials (the measurement's workspace size)
    const int max_ctas = p.stat_partials != nullptr ? DQ_MAX_CTAS : (1 << 30);
    const size_t fixed = TQ_BAR_BYTES + TQ_PHI_BYTES + TQ_RED_BYTES;
    cudaError_t e = plan_pipeline(pick.kern, TQ_WARPS, SB, fixed, 0, TQ_MAX_STAGES, pick.ctas,
                                  int64_t(1) << 40, max_ctas, dev, &pl);
    if (e != cudaSuccess) return e;
    // Few tokens for the resident warps (decode batches): split each token into units of 8
    // query rows plus one unit of its key (and value) rows, so that more warps share it
    const int64_t warps_resident = static_cast<int64_t>(pl.grid) * TQ_WARPS;
    int64_t units = p.T;
    // (the statistics instances keep whole tokens; T * parts stays far below 2^31 here)
    if (!measure && 2 * p.T <= warps_resident && p.Hq > 8) {
        pick = pick_kernel<DH, STYLE, false, true>(mode, b, group);
        q.parts = (p.Hq + 7) / 8 + 1;
        units = p.T * q.parts;
        const int qpart = (p.Hq < 8 ? p.Hq : 8) * DH * 2, kpart = p.Hkv * DH * 2;
        SB = token_stage_bytes(0, 0, DH, p.split, (qpart > kpart + vbytes ? qpart : kpart + vbytes));
    }
    e = plan_pipeline(pick.kern, TQ_WARPS, SB, fixed, 0, TQ_MAX_STAGES, pick.ctas, units, max_ctas,
                      dev, &pl);
    if (e != cudaSuccess) return e;
    if (pl.grid == 0) return cudaSuccess;
    q.stages = pl.stages;
    q.stage_bytes = SB;
    // may be launched while the stream's previous kernel runs (the kernel waits for it)
    const cudaError_t le = launch_after_prior(pick.kern, dim3(static_cast<unsigned>(pl.grid)),
                                              dim3(TQ_WARPS * 32), pl.smem, stream, q);
    if (le != cudaSuccess) return le;
    if (ctas_used != nullptr) *ctas_used = pl.grid;
    return cudaGetLastError();
}

// Host-side launch of the calibrating transform: moment partials into mom_partials (one
// [2][d_h/2][5] block per CTA, at most max_ctas CTAs); *ctas_used receives the grid.
template <int DH, int STYLE>
cudaError_t transform_calib_launch(const TransformParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, double *mom_partials, int max_ctas,
                                   int *ctas_used, cudaStream_t stream)
{
    *ctas_used = 0;
    if (p.v != nullptr || p.stat_partials != nullptr) return cudaErrorInvalidValue;
    const CalibKernel kern = pick_calib<DH, STYLE>(mode, b, group);
    if (kern == nullptr) return cudaErrorInvalidValue;
    const int SB = token_stage_bytes(p.Hq, p.Hkv, DH, p.split);
    PipeLaunch pl;
    // stage area: TQ_WARPS pipelines (the moment warps read the same stages)
    cudaError_t e = plan_pipeline(kern, TQ_WARPS, SB, TCAL_BAR_BYTES + TQ_PHI_BYTES + TCAL_RED_BYTES,
                                  0, TQ_MAX_STAGES, TCAL_CTAS, p.T, max_ctas, dev, &pl);
    if (e != cudaSuccess) return e;
    if (pl.grid == 0) return cudaSuccess;
    TransformParams q = p;
    q.stages = pl.stages;
    q.stage_bytes = SB;
    kern<<<pl.grid, TCAL_WARPS * 32, pl.smem, stream>>>(q, mom_partials);
    *ctas_used = pl.grid;
    return cudaGetLastError();
}

// One translation unit per (d_h, RoPE layout) when built with -DQKQ_DH/-DQKQ_STYLE
// (the build compiles them in parallel); all four otherwise.
#if defined(QKQ_DH) && defined(QKQ_STYLE)
template cudaError_t transform_quant_launch<QKQ_DH, QKQ_STYLE>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t, int *);
template cudaError_t transform_calib_launch<QKQ_DH, QKQ_STYLE>(const TransformParams &, int, int, int, const DeviceInfo &, double *, int, int *, cudaStream_t);
#else
template cudaError_t transform_quant_launch<64, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t, int *);
template cudaError_t transform_calib_launch<64, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, double *, int, int *, cudaStream_t);
template cudaError_t transform_quant_launch<64, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t, int *);
template cudaError_t transform_calib_launch<64, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, double *, int, int *, cudaStream_t);
template cudaError_t transform_quant_launch<128, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t, int *);
template cudaError_t transform_calib_launch<128, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, double *, int, int *, cudaStream_t);
template cudaError_t transform_quant_launch<128, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t, int *);
template cudaError_t transform_calib_launch<128, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, double *, int, int *, cudaStream_t);
#endif

}  // namespace qkq

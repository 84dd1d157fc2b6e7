// Measurement path: K range and relative quantisation error of the quantised keys
// ("When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for
// Dynamic 4-Bit Quantisation", "Core contributions" and "Results": K range,
// relative quantisation error and perplexity gap all fall as the mixing support b
// grows from 2 to d_h).
//
// The kernel recomputes K~ from the bf16 keys with the fused transform's row code
// (rowops.cuh, so the values are bit-identical to those that were quantised) and
// compares them with the dequantised codes K^ = fp16 scale * code.  Per (token, head,
// group) it also gathers max|K~| (the step-setting statistic) and max - min.  The
// squared error and reference are fp32 sums per lane and group of scale-normalised terms
// (row_stats in rowops.cuh, shared with the transform launch that computes the same
// statistics in its own pass), the totals fp64; reduced per CTA in a fixed order into the
// caller's workspace, then across CTAs in order by a second kernel.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"
#include "rowops.cuh"

namespace qkq {

namespace {

constexpr int DQ_MAX_STAGES = 4;
constexpr int DQ_WANT_CTAS = 2;
constexpr int DQ_BAR_BYTES = DQ_WARPS * DQ_MAX_STAGES * 8;
constexpr int DQ_FIXED_SMEM = (DQ_BAR_BYTES + 2 * 64 * 4 + DQ_WARPS * 6 * 8 + 127) / 128 * 128;  // bars, phi, red

template <int DH, int NMIX, bool PAIRROT, int G, int STYLE>
__global__ void __launch_bounds__(DQ_WARPS * 32) k_dequant_partial(const DequantParams p)
{
    using L = Layout<DH, STYLE>;
    using GR = Groups<L, G>;
    constexpr int P = DH / 2;
    constexpr int ROWB = DH * 2;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    float *phi_tab = reinterpret_cast<float *>(smem + DQ_BAR_BYTES);
    double *red = reinterpret_cast<double *>(smem + DQ_BAR_BYTES + 2 * 64 * 4);
    uint8_t *stage_mem = smem + DQ_FIXED_SMEM;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane & 3, rq = lane >> 2;
    int flags = 0;
    const uint32_t cbytes = static_cast<uint32_t>(p.Hkv) * (DH / 2);  // packed codes per token
    TokenPipe pipe;  // key rows, table rows and the token's packed codes
    pipe.start(stage_mem + static_cast<size_t>(warp) * p.stages * p.stage_bytes,
               bars + warp * DQ_MAX_STAGES, p.stages, p.stage_bytes,
               static_cast<int64_t>(blockIdx.x) * DQ_WARPS + warp,
               static_cast<int64_t>(gridDim.x) * DQ_WARPS, p.T, 0, p.Hkv, DH, nullptr, p.k,
               p.cos_t, p.sin_t, p.pos, p.max_pos, p.split, flags, false, p.k_codes, cbytes);

    PairCoeffs<L> pc;  // cos and sin of the pair angles, in registers (pairwise modes)
    if (PAIRROT) {
        for (int i = threadIdx.x; i < P; i += blockDim.x) {
            const double ph = static_cast<double>(p.phi[i]);
            phi_tab[i] = static_cast<float>(cos(ph));
            phi_tab[P + i] = static_cast<float>(sin(ph));
        }
        __syncthreads();
        pc.load(phi_tab, P, l);
    }

    RowStats stats;
    // scales of the first row group of a token, read one token ahead (their global loads
    // then overlap the previous token's work instead of stalling this one)
    const int row0c = rq < p.Hkv ? rq : p.Hkv - 1;
    auto load_scales = [&](int64_t n, uint16_t (&out)[GR::NG]) {
        if (n < pipe.ntok) {
            const int64_t gr = pipe.token(n) * p.Hkv + row0c;
#pragma unroll
            for (int g = 0; g < GR::NG; ++g) out[g] = __ldg(p.k_scales + gr * GR::NG + g);
        }
    };
    uint16_t sc_cur[GR::NG], sc_nxt[GR::NG];
    load_scales(0, sc_cur);
    for (int64_t n = 0; n < pipe.ntok; ++n) {
        load_scales(n + 1, sc_nxt);
        const uint8_t *st = pipe.wait(n, flags);
        if (st == nullptr) break;
        const int64_t t = pipe.token(n);
        const float *ctab = reinterpret_cast<const float *>(st + pipe.table_offset());
        float2 C[L::NT], Sn[L::NT];
        load_rope<L>(C, Sn, ctab, P, p.split, l);
        for (int r0 = 0; r0 < p.Hkv; r0 += 8) {
            const int row = r0 + rq;
            const bool active = row < p.Hkv;
            const int rowc = active ? row : p.Hkv - 1;  // keep every lane in the shuffles
            const int64_t gr = t * p.Hkv + rowc;
            // codes of the row (staged with the token) and its scales
            const uint32_t *crow = reinterpret_cast<const uint32_t *>(
                st + pipe.extra_offset() + rowc * (DH / 2));
            uint32_t cw[L::NJ];
#pragma unroll
            for (int j = 0; j < L::NJ; ++j) cw[j] = crow[j * 4 + l];
            float scl[GR::NG];
#pragma unroll
            for (int g = 0; g < GR::NG; ++g)
                scl[g] = __half2float(__ushort_as_half(
                    r0 == 0 ? sc_cur[g] : __ldg(p.k_scales + gr * GR::NG + g)));
            float2 V[L::NV];
            load_row_bf16<L>(V, st + rowc * ROWB, l);
            rotate_pairs<L>(V, C, Sn);
            if (PAIRROT) rotate_pairs<L>(V, pc.c, pc.s);  // RoPE, then the pair angle
            fwht<L, NMIX>(V, l, p.kappa);

            // codes of V[p] (p = 4j + k) as floats: biased nibbles c + 8 from the packed word,
            // placed into 2^23 + c + 8 by a byte permutation, then 2^23 + 8 subtracted (exact)
            auto code_of = [&](int pidx) {
                const int j = pidx >> 2, k = pidx & 3;
                const uint32_t wb = cw[j] ^ 0x88888888u;
                const uint32_t ev = wb & 0x0F0F0F0Fu, od = (wb >> 4) & 0x0F0F0F0Fu;
                // element pairs of V[4j + k]: (2k, 2k+1) for PB = 0; (0,2), (1,3), (4,6), (5,7)
                // for PB = 1
                const uint32_t xa = L::PB == 0 ? ev : ((k & 1) ? od : ev);
                const uint32_t xb = L::PB == 0 ? od : ((k & 1) ? od : ev);
                const int ba = L::PB == 0 ? k : (k >> 1) * 2;
                const int bb = L::PB == 0 ? k : (k >> 1) * 2 + 1;
                return __fadd2_rn(
                    make_float2(__uint_as_float(__byte_perm(xa, 0x4B000000u, 0x7540u | ba)),
                                __uint_as_float(__byte_perm(xb, 0x4B000000u, 0x7540u | bb))),
                    make_float2(-8388616.0f, -8388616.0f));
            };
            row_stats<L, G>(V, code_of, scl, l, active, stats);
        }
        pipe.release(n, flags);
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) sc_cur[g] = sc_nxt[g];
    }
    // NaN / Inf in K~ propagate into the sums (max/min would skip a NaN)
    reduce_row_stats(stats, red, DQ_WARPS, p.partials + static_cast<int64_t>(blockIdx.x) * 6, flags);
    if (flags && p.status) atomicOr(p.status, flags);
}

using DequantKernel = void (*)(DequantParams);

template <int DH, int G, int STYLE>
DequantKernel pick_mix(int mode, int b)
{
    switch (mode) {
    case MODE_HADAMARD: return k_dequant_partial<DH, DH, false, G, STYLE>;
    case MODE_PAIRWISE: return k_dequant_partial<DH, 1, true, G, STYLE>;
    case MODE_PAIRWISE_HADAMARD: return k_dequant_partial<DH, DH, true, G, STYLE>;
    case MODE_ROPE_ONLY: return k_dequant_partial<DH, 1, false, G, STYLE>;
    case MODE_BLOCK_HADAMARD:
        switch (b) {
        case 2: return k_dequant_partial<DH, 2, false, G, STYLE>;
        case 4: return k_dequant_partial<DH, 4, false, G, STYLE>;
        case 8: return k_dequant_partial<DH, 8, false, G, STYLE>;
        case 16: return k_dequant_partial<DH, 16, false, G, STYLE>;
        case 32: return k_dequant_partial<DH, 32, false, G, STYLE>;
        case 64: return k_dequant_partial<DH, 64, false, G, STYLE>;
        case 128:
            if (DH == 128) return k_dequant_partial<DH, (DH == 128 ? 128 : 64), false, G, STYLE>;
            break;
        }
        break;
    }
    return nullptr;
}

template <int DH, int STYLE>
DequantKernel pick_kernel(int mode, int b, int group)
{
    switch (group) {
    case 32: return pick_mix<DH, 32, STYLE>(mode, b);
    case 64: return pick_mix<DH, 64, STYLE>(mode, b);
    case 128:
        if (DH == 128) return pick_mix<DH, (DH == 128 ? 128 : 64), STYLE>(mode, b);
        break;
    }
    return nullptr;
}

}  // namespace

template <int DH, int STYLE>
cudaError_t dequant_partial_launch(const DequantParams &p, int mode, int b, int group,
                                   const DeviceInfo &dev, int *ctas_used, cudaStream_t stream)
{
    *ctas_used = 0;
    if (p.T <= 0) return cudaSuccess;
    const DequantKernel kern = pick_kernel<DH, STYLE>(mode, b, group);
    if (kern == nullptr) return cudaErrorInvalidValue;
    const int SB = token_stage_bytes(0, p.Hkv, DH, p.split, p.Hkv * (DH / 2));
    PipeLaunch pl;
    cudaError_t e = plan_pipeline(kern, DQ_WARPS, SB, DQ_FIXED_SMEM, 0, DQ_MAX_STAGES,
                                  DQ_WANT_CTAS, p.T, DQ_MAX_CTAS, dev, &pl);
    if (e != cudaSuccess) return e;
    DequantParams q = p;
    q.stages = pl.stages;
    q.stage_bytes = SB;
    kern<<<pl.grid, DQ_WARPS * 32, pl.smem, stream>>>(q);
    *ctas_used = pl.grid;
    return cudaGetLastError();
}

// One translation unit per (d_h, RoPE layout) when built with -DQKQ_DH/-DQKQ_STYLE
// (the build compiles them in parallel); all four otherwise.
#if defined(QKQ_DH) && defined(QKQ_STYLE)
template cudaError_t dequant_partial_launch<QKQ_DH, QKQ_STYLE>(const DequantParams &, int, int, int, const DeviceInfo &, int *, cudaStream_t);
#else
template cudaError_t dequant_partial_launch<64, ROPE_HALF>(const DequantParams &, int, int, int, const DeviceInfo &, int *, cudaStream_t);
template cudaError_t dequant_partial_launch<64, ROPE_INTERLEAVED>(const DequantParams &, int, int, int, const DeviceInfo &, int *, cudaStream_t);
template cudaError_t dequant_partial_launch<128, ROPE_HALF>(const DequantParams &, int, int, int, const DeviceInfo &, int *, cudaStream_t);
template cudaError_t dequant_partial_launch<128, ROPE_INTERLEAVED>(const DequantParams &, int, int, int, const DeviceInfo &, int *, cudaStream_t);
#endif


// The cross-CTA reduction is not templated: built in one translation unit only.
#if !defined(QKQ_DH) || (QKQ_DH == 64 && QKQ_STYLE == 0)
namespace {
__global__ void k_dequant_final(const double *partials, int ctas, double *stats)
{
    const int f = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (f >= 6) return;
    double acc = 0.0;
    for (int c = lane; c < ctas; c += 32) {
        const double x = partials[static_cast<int64_t>(c) * 6 + f];
        acc = f == 4 ? fmax(acc, x) : acc + x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double other = __shfl_xor_sync(FULL_MASK, acc, o);
        acc = f == 4 ? fmax(acc, other) : acc + other;
    }
    if (lane == 0) stats[f] = acc;
}

}  // namespace

cudaError_t dequant_final_launch(const double *partials, int blocks, double *stats,
                                 cudaStream_t stream)
{
    k_dequant_final<<<1, 6 * 32, 0, stream>>>(partials, blocks, stats);
    return cudaGetLastError();
}
#endif

}  // namespace qkq

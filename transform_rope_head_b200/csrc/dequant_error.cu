// Measurement path: K range and relative quantisation error of the quantised keys
// ("When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for
// Dynamic 4-Bit Quantisation", "Core contributions" and "Results": K range,
// relative quantisation error and perplexity gap all fall as the mixing support b
// grows from 2 to d_h).
//
// The kernel recomputes K~ from the bf16 keys with the fused transform's row code
// (rowops.cuh, so the values are bit-identical to those that were quantised) and
// compares them with the dequantised codes K^ = fp16 scale * code.  Per (token, head,
// group) it also gathers max|K~| (the step-setting statistic) and max - min.  Sums
// are fp64, reduced per CTA in a fixed order into the caller's workspace, then across
// CTAs in order by a second kernel.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "rowops.cuh"

namespace qkq {

namespace {

constexpr int DQ_WARPS = DQ_THREADS / 32;

template <int DH, int NMIX, bool PAIRROT, int G, int STYLE>
__global__ void __launch_bounds__(DQ_THREADS) k_dequant_partial(const DequantParams p)
{
    using L = Layout<DH, STYLE>;
    using GR = Groups<L, G>;
    constexpr int P = DH / 2;
    __shared__ float phi_tab[2 * P];
    __shared__ double red[DQ_WARPS][6];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane & 3, rq = lane >> 2;
    const int64_t rows = p.T * p.Hkv;
    const int64_t chunk = (rows + gridDim.x - 1) / gridDim.x;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t row1 = row0 + chunk < rows ? row0 + chunk : rows;
    int flags = 0;

    float2 CP[L::NT], SP[L::NT], NSP[L::NT];
    if (PAIRROT) {
        for (int i = threadIdx.x; i < P; i += blockDim.x) {
            const double ph = static_cast<double>(p.phi[i]);
            phi_tab[i] = static_cast<float>(cos(ph));
            phi_tab[P + i] = static_cast<float>(sin(ph));
        }
        __syncthreads();
        load_pair_table<L>(CP, phi_tab, l);
        load_pair_table<L>(SP, phi_tab + P, l);
        negate_table<L>(NSP, SP);
    }

    double err2 = 0.0, ref2 = 0.0, s_amax = 0.0, s_range = 0.0, mx_amax = 0.0, n_groups = 0.0;
    for (int64_t base = row0 + warp * 8; base < row1; base += DQ_WARPS * 8) {
        const int64_t row = base + rq;
        const bool active = row < row1;
        const int64_t rowc = active ? row : row1 - 1;
        const int64_t t = rowc / p.Hkv;
        const int64_t m = clamp_pos(__ldg(p.pos + t), p.max_pos, flags);
        float2 C[L::NT], Sn[L::NT], NS[L::NT];
        load_pair_table<L>(C, p.cos_t + m * P, l);
        load_pair_table<L>(Sn, p.sin_t + m * P, l);
        negate_table<L>(NS, Sn);
        float2 V[L::NV];
        load_row_bf16<L>(V, reinterpret_cast<const uint8_t *>(p.k + rowc * DH), l);
        rotate_pairs<L>(V, C, Sn, NS);
        if (PAIRROT) rotate_pairs<L>(V, CP, SP, NSP);
        fwht<L, NMIX>(V, l, p.kappa);

        // group statistics over the quad
        float amax[GR::NG], gmax[GR::NG], gmin[GR::NG];
        group_amax<L, G>(V, amax);
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) {
            gmax[g] = -INFINITY;
            gmin[g] = INFINITY;
        }
#pragma unroll
        for (int p2 = 0; p2 < L::NV; ++p2) {
            const int g = GR::of_chunk(L::elem(p2, 0) >> 3);
            gmax[g] = fmaxf(gmax[g], fmaxf(V[p2].x, V[p2].y));
            gmin[g] = fminf(gmin[g], fminf(V[p2].x, V[p2].y));
        }
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) {
            gmax[g] = fmaxf(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 1));
            gmax[g] = fmaxf(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 2));
            gmin[g] = fminf(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 1));
            gmin[g] = fminf(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 2));
        }
        if (!active) continue;
        // dequantise and compare
        const uint32_t *crow = reinterpret_cast<const uint32_t *>(p.k_codes + rowc * (DH / 2));
        float scl[GR::NG];
#pragma unroll
        for (int g = 0; g < GR::NG; ++g)
            scl[g] = __half2float(__ushort_as_half(p.k_scales[rowc * GR::NG + g]));
#pragma unroll
        for (int j = 0; j < L::NJ; ++j) {
            const uint32_t w = crow[j * 4 + l];
            const float sg = scl[GR::of_chunk(j)];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int code = static_cast<int>(((w >> (4 * e)) & 0xfu) ^ 8u) - 8;
                const float x = get_el<L>(V, j * 8 + e);
                const float dq = sg * static_cast<float>(code);  // exact: 11-bit * 4-bit
                const double d = static_cast<double>(x) - static_cast<double>(dq);
                err2 = fma(d, d, err2);
                ref2 = fma(static_cast<double>(x), static_cast<double>(x), ref2);
            }
        }
        if (l == 0) {
#pragma unroll
            for (int g = 0; g < GR::NG; ++g) {
                if (!(amax[g] <= 3.402823466e38f)) flags |= ST_NONFINITE;
                s_amax += amax[g];
                s_range += static_cast<double>(gmax[g]) - static_cast<double>(gmin[g]);
                mx_amax = fmax(mx_amax, static_cast<double>(amax[g]));
                n_groups += 1.0;
            }
        }
    }
    // warp reduction (fixed xor tree), then warps in order
    double v[6] = {err2, ref2, s_amax, s_range, mx_amax, n_groups};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int f = 0; f < 6; ++f) {
            const double other = __shfl_xor_sync(FULL_MASK, v[f], o);
            v[f] = f == 4 ? fmax(v[f], other) : v[f] + other;
        }
    if (lane == 0)
#pragma unroll
        for (int f = 0; f < 6; ++f) red[warp][f] = v[f];
    __syncthreads();
    if (threadIdx.x < 6) {
        const int f = threadIdx.x;
        double acc = red[0][f];
        for (int w = 1; w < DQ_WARPS; ++w) acc = f == 4 ? fmax(acc, red[w][f]) : acc + red[w][f];
        p.partials[static_cast<int64_t>(blockIdx.x) * 6 + f] = acc;
    }
    if (flags && p.status) atomicOr(p.status, flags);
}

template <int DH, int NMIX, bool PAIRROT, int G, int STYLE>
cudaError_t launch_dq(const DequantParams &p, int blocks, cudaStream_t s)
{
    k_dequant_partial<DH, NMIX, PAIRROT, G, STYLE><<<blocks, DQ_THREADS, 0, s>>>(p);
    return cudaGetLastError();
}

template <int DH, int G, int STYLE>
cudaError_t dq_dispatch_mix(const DequantParams &p, int mode, int b, int blocks, cudaStream_t s)
{
    switch (mode) {
    case MODE_HADAMARD: return launch_dq<DH, DH, false, G, STYLE>(p, blocks, s);
    case MODE_PAIRWISE: return launch_dq<DH, 1, true, G, STYLE>(p, blocks, s);
    case MODE_PAIRWISE_HADAMARD: return launch_dq<DH, DH, true, G, STYLE>(p, blocks, s);
    case MODE_ROPE_ONLY: return launch_dq<DH, 1, false, G, STYLE>(p, blocks, s);
    case MODE_BLOCK_HADAMARD:
        switch (b) {
        case 2: return launch_dq<DH, 2, false, G, STYLE>(p, blocks, s);
        case 4: return launch_dq<DH, 4, false, G, STYLE>(p, blocks, s);
        case 8: return launch_dq<DH, 8, false, G, STYLE>(p, blocks, s);
        case 16: return launch_dq<DH, 16, false, G, STYLE>(p, blocks, s);
        case 32: return launch_dq<DH, 32, false, G, STYLE>(p, blocks, s);
        case 64: return launch_dq<DH, 64, false, G, STYLE>(p, blocks, s);
        case 128:
            if (DH == 128) return launch_dq<DH, (DH == 128 ? 128 : 64), false, G, STYLE>(p, blocks, s);
            break;
        }
        break;
    }
    return cudaErrorInvalidValue;
}

}  // namespace

template <int DH, int STYLE>
cudaError_t dequant_partial_launch(const DequantParams &p, int mode, int b, int group, int blocks,
                                   cudaStream_t stream)
{
    if (blocks <= 0) return cudaSuccess;
    switch (group) {
    case 32: return dq_dispatch_mix<DH, 32, STYLE>(p, mode, b, blocks, stream);
    case 64: return dq_dispatch_mix<DH, 64, STYLE>(p, mode, b, blocks, stream);
    case 128:
        if (DH == 128) return dq_dispatch_mix<DH, (DH == 128 ? 128 : 64), STYLE>(p, mode, b, blocks, stream);
        break;
    }
    return cudaErrorInvalidValue;
}

// One translation unit per (d_h, RoPE layout) when built with -DQKQ_DH/-DQKQ_STYLE
// (the build compiles them in parallel); all four otherwise.
#if defined(QKQ_DH) && defined(QKQ_STYLE)
template cudaError_t dequant_partial_launch<QKQ_DH, QKQ_STYLE>(const DequantParams &, int, int, int, int, cudaStream_t);
#else
template cudaError_t dequant_partial_launch<64, ROPE_HALF>(const DequantParams &, int, int, int, int, cudaStream_t);
template cudaError_t dequant_partial_launch<64, ROPE_INTERLEAVED>(const DequantParams &, int, int, int, int, cudaStream_t);
template cudaError_t dequant_partial_launch<128, ROPE_HALF>(const DequantParams &, int, int, int, int, cudaStream_t);
template cudaError_t dequant_partial_launch<128, ROPE_INTERLEAVED>(const DequantParams &, int, int, int, int, cudaStream_t);
#endif


// The cross-CTA reduction is not templated: built in one translation unit only.
#if !defined(QKQ_DH) || (QKQ_DH == 64 && QKQ_STYLE == 0)
namespace {
__global__ void k_dequant_final(const double *partials, int blocks, double *stats)
{
    const int f = threadIdx.x;
    if (f >= 6) return;
    double acc = 0.0;
    for (int b = 0; b < blocks; ++b) {
        const double x = partials[static_cast<int64_t>(b) * 6 + f];
        acc = f == 4 ? fmax(acc, x) : acc + x;
    }
    stats[f] = acc;
}

}  // namespace

cudaError_t dequant_final_launch(const double *partials, int blocks, double *stats,
                                 cudaStream_t stream)
{
    k_dequant_final<<<1, 32, 0, stream>>>(partials, blocks, stats);
    return cudaGetLastError();
}
#endif

}  // namespace qkq

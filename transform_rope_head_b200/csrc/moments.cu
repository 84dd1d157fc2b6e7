// Calibration side path, step 1: raw per-pair moment accumulators of the post-RoPE
// (pre-mixing) Q and K values, pooled over heads and tokens ("When Local Variance
// Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for Dynamic 4-Bit
// Quantisation", "Estimation strategies": the default estimator pools the raw Q and
// K moment accumulators across heads before centring; "Optimisation objective": a
// position-averaged surrogate).
//
// A blocked, deterministic reduction: each CTA owns a contiguous range of rows of one
// stream; 16 lanes share a row (each holds d_h/32 frequency pairs, both channels of
// each pair in registers), apply RoPE with the same fp32 operations as the fused
// transform, widen to fp64 and accumulate Sa, Sb, Saa, Sab, Sbb (products of fp32
// values are exact in fp64).  CTA partials go to the caller's workspace; a second
// kernel adds them in a fixed order into the caller's accumulator.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace qkq {

namespace {

template <int DH, int STYLE>
__global__ void __launch_bounds__(MOM_THREADS) k_moments_partial(const MomentsParams p)
{
    constexpr int P = DH / 2;
    constexpr int PPT = P / 16;              // pairs per lane
    constexpr int NWARP = MOM_THREADS / 32;
    __shared__ double red[NWARP][16][PPT * 5];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l16 = lane & 15, rr = lane >> 4;
    const int64_t rows = p.T * p.H;
    const int64_t chunk = (rows + gridDim.x - 1) / gridDim.x;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t row1 = row0 + chunk < rows ? row0 + chunk : rows;
    const int k0 = l16 * PPT;                // first pair of this lane

    double acc[PPT][5];
#pragma unroll
    for (int u = 0; u < PPT; ++u)
#pragma unroll
        for (int f = 0; f < 5; ++f) acc[u][f] = 0.0;
    int flags = 0;

    for (int64_t row = row0 + warp * 2 + rr; row < row1; row += NWARP * 2) {
        const int64_t t = row / p.H;
        const int64_t m = clamp_pos(__ldg(p.pos + t), p.max_pos, flags);
        const uint16_t *x = p.x + row * DH;
        float a[PPT], b[PPT], c[PPT], s[PPT];
        if constexpr (STYLE == ROPE_HALF) {
            // channels k0..k0+PPT-1 and k0+P..k0+P+PPT-1
            if constexpr (PPT == 4) {
                const uint2 wa = *reinterpret_cast<const uint2 *>(x + k0);
                const uint2 wb = *reinterpret_cast<const uint2 *>(x + k0 + P);
                a[0] = __uint_as_float(wa.x << 16); a[1] = __uint_as_float(wa.x & 0xffff0000u);
                a[2] = __uint_as_float(wa.y << 16); a[3] = __uint_as_float(wa.y & 0xffff0000u);
                b[0] = __uint_as_float(wb.x << 16); b[1] = __uint_as_float(wb.x & 0xffff0000u);
                b[2] = __uint_as_float(wb.y << 16); b[3] = __uint_as_float(wb.y & 0xffff0000u);
            } else {
                const uint32_t wa = *reinterpret_cast<const uint32_t *>(x + k0);
                const uint32_t wb = *reinterpret_cast<const uint32_t *>(x + k0 + P);
                a[0] = __uint_as_float(wa << 16); a[1] = __uint_as_float(wa & 0xffff0000u);
                b[0] = __uint_as_float(wb << 16); b[1] = __uint_as_float(wb & 0xffff0000u);
            }
        } else {
            // channels 2k0 .. 2k0 + 2*PPT - 1, pairs adjacent
            if constexpr (PPT == 4) {
                const uint4 w = *reinterpret_cast<const uint4 *>(x + 2 * k0);
                const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int u = 0; u < PPT; ++u) {
                    a[u] = __uint_as_float(wd[u] << 16);
                    b[u] = __uint_as_float(wd[u] & 0xffff0000u);
                }
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(x + 2 * k0);
                const uint32_t wd[2] = {w.x, w.y};
#pragma unroll
                for (int u = 0; u < PPT; ++u) {
                    a[u] = __uint_as_float(wd[u] << 16);
                    b[u] = __uint_as_float(wd[u] & 0xffff0000u);
                }
            }
        }
        const float *crow = p.cos_t + m * P + k0;
        const float *srow = p.sin_t + m * P + k0;
#pragma unroll
        for (int u = 0; u < PPT; ++u) {
            c[u] = __ldg(crow + u);
            s[u] = __ldg(srow + u);
        }
#pragma unroll
        for (int u = 0; u < PPT; ++u) {
            // RoPE, the same fp32 operations as the fused transform
            const float ra = __fmaf_rn(a[u], c[u], -__fmul_rn(b[u], s[u]));
            const float rb = __fmaf_rn(a[u], s[u], __fmul_rn(b[u], c[u]));
            const double da = ra, db = rb;
            acc[u][0] += da;
            acc[u][1] += db;
            acc[u][2] = fma(da, da, acc[u][2]);
            acc[u][3] = fma(da, db, acc[u][3]);
            acc[u][4] = fma(db, db, acc[u][4]);
        }
    }
    // the two row halves of the warp
#pragma unroll
    for (int u = 0; u < PPT; ++u)
#pragma unroll
        for (int f = 0; f < 5; ++f) acc[u][f] += __shfl_xor_sync(FULL_MASK, acc[u][f], 16);
    if (rr == 0)
#pragma unroll
        for (int u = 0; u < PPT; ++u)
#pragma unroll
            for (int f = 0; f < 5; ++f) red[warp][l16][u * 5 + f] = acc[u][f];
    __syncthreads();
    // one thread per (pair, field): add the warps in order
    for (int i = threadIdx.x; i < P * 5; i += MOM_THREADS) {
        const int k = i / 5, f = i % 5;
        const int ln = k / PPT, u = k % PPT;
        double sum = 0.0;
        for (int w = 0; w < NWARP; ++w) sum += red[w][ln][u * 5 + f];
        if (!isfinite(sum)) flags |= ST_NONFINITE;
        p.partials[(static_cast<int64_t>(blockIdx.x) * P + k) * 5 + f] = sum;
    }
    if (flags && p.status) atomicOr(p.status, flags);
}

// moments[s][k][0] += rows of stream s; moments[s][k][1 + f] += sum over blocks (in order).
__global__ void k_moments_final(const double *pq, int bq, int64_t rq, const double *pk, int bk,
                                int64_t rk, int P, double *moments)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * P * 6) return;
    const int s = i / (P * 6), k = (i / 6) % P, f = i % 6;
    const double *part = s == 0 ? pq : pk;
    const int nb = s == 0 ? bq : bk;
    double sum;
    if (f == 0) {
        sum = static_cast<double>(s == 0 ? rq : rk);
    } else {
        sum = 0.0;
        for (int b = 0; b < nb; ++b) sum += part[(static_cast<int64_t>(b) * P + k) * 5 + (f - 1)];
    }
    moments[(s * P + k) * 6 + f] += sum;
}

}  // namespace

template <int DH, int STYLE>
cudaError_t moments_partial_launch(const MomentsParams &p, int blocks, cudaStream_t stream)
{
    if (blocks <= 0) return cudaSuccess;
    k_moments_partial<DH, STYLE><<<blocks, MOM_THREADS, 0, stream>>>(p);
    return cudaGetLastError();
}

template cudaError_t moments_partial_launch<64, ROPE_HALF>(const MomentsParams &, int, cudaStream_t);
template cudaError_t moments_partial_launch<64, ROPE_INTERLEAVED>(const MomentsParams &, int, cudaStream_t);
template cudaError_t moments_partial_launch<128, ROPE_HALF>(const MomentsParams &, int, cudaStream_t);
template cudaError_t moments_partial_launch<128, ROPE_INTERLEAVED>(const MomentsParams &, int, cudaStream_t);

cudaError_t moments_final_launch(const double *partials_q, int blocks_q, int64_t rows_q,
                                 const double *partials_k, int blocks_k, int64_t rows_k, int P,
                                 double *moments, cudaStream_t stream)
{
    const int n = 2 * P * 6;
    k_moments_final<<<(n + 127) / 128, 128, 0, stream>>>(partials_q, blocks_q, rows_q, partials_k,
                                                         blocks_k, rows_k, P, moments);
    return cudaGetLastError();
}

}  // namespace qkq

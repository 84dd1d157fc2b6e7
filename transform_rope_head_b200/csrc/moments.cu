// Calibration side path, step 1: raw per-pair moment accumulators of the post-RoPE
// (pre-mixing) Q and K values, pooled over heads and tokens ("When Local Variance
// Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for Dynamic 4-Bit
// Quantisation", "Estimation strategies": the default estimator pools the raw Q and
// K moment accumulators across heads before centring; "Optimisation objective": a
// position-averaged surrogate).
//
// Streaming, on the same per-warp token pipeline as the fused transform (one HBM read
// of Q and K).  Lanes map to frequency pairs: a lane owns two adjacent pairs (both
// channels of each), 32 lanes cover one row at d_h = 128 (16 lanes at d_h = 64, the
// half-warps taking alternate rows).  RoPE is applied with the transform's fp32
// operations, the values are widened to fp64 and accumulated (products of fp32 values
// are exact in fp64) per stream in registers for all of the warp's tokens.  Each CTA
// writes one partial; a second kernel adds the partials in a fixed order, so the sums
// are deterministic for a given device and size.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"

namespace qkq {

namespace {

#ifndef QKQ_MOM_MIN_CTAS
#define QKQ_MOM_MIN_CTAS 4
#endif
constexpr int MOM_MAX_STAGES = 4;
constexpr int MOM_BAR_BYTES = (MOM_WARPS * MOM_MAX_STAGES * 8 + 127) / 128 * 128;
// Four CTAs per SM: the fp64 accumulation wants warps more than stages in flight.
constexpr int MOM_WANT_CTAS = QKQ_MOM_MIN_CTAS;

// [warps][lanes][2 streams x 2 pairs x 5 sums], in the stage area once the loop is done
constexpr int MOM_RED_BYTES = MOM_WARPS * 32 * 20 * 8;

__device__ __forceinline__ void accumulate(double (&acc)[2][5], float2 a, float2 b)
{
    const double a0 = a.x, a1 = a.y, b0 = b.x, b1 = b.y;
    acc[0][0] += a0;
    acc[0][1] += b0;
    acc[0][2] = fma(a0, a0, acc[0][2]);
    acc[0][3] = fma(a0, b0, acc[0][3]);
    acc[0][4] = fma(b0, b0, acc[0][4]);
    acc[1][0] += a1;
    acc[1][1] += b1;
    acc[1][2] = fma(a1, a1, acc[1][2]);
    acc[1][3] = fma(a1, b1, acc[1][3]);
    acc[1][4] = fma(b1, b1, acc[1][4]);
}

// First / second channels of the lane's pairs (k0, k0 + 1) in one bf16 row.
template <int DH, int STYLE>
__device__ __forceinline__ void load_pairs(const uint8_t *row, int lr, float2 &a, float2 &b)
{
    if constexpr (STYLE == ROPE_HALF) {
        const uint32_t wa = *reinterpret_cast<const uint32_t *>(row + 4 * lr);
        const uint32_t wb = *reinterpret_cast<const uint32_t *>(row + 4 * lr + DH);
        a = make_float2(__uint_as_float(wa << 16), __uint_as_float(wa & 0xffff0000u));
        b = make_float2(__uint_as_float(wb << 16), __uint_as_float(wb & 0xffff0000u));
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(row + 8 * lr);
        a = make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.y << 16));
        b = make_float2(__uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y & 0xffff0000u));
    }
}

template <int DH, int STYLE>
__global__ void __launch_bounds__(MOM_WARPS * 32, QKQ_MOM_MIN_CTAS) k_moments_partial(const MomentsParams p)
{
    constexpr int P = DH / 2;
    constexpr int ROWB = DH * 2;
    constexpr int LPR = P / 2;            // lanes per row: 32 (d_h 128) or 16 (d_h 64)
    constexpr int RPS = 32 / LPR;         // rows per warp step
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint8_t *stage_mem = smem + MOM_BAR_BYTES;
    double *red = reinterpret_cast<double *>(stage_mem);  // reused after every warp's loop

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lr = lane % LPR, sub = lane / LPR;
    const int k0 = 2 * lr;
    int flags = 0;
    TokenPipe pipe;
    pipe.start(stage_mem + static_cast<size_t>(warp) * p.stages * p.stage_bytes,
               bars + warp * MOM_MAX_STAGES, p.stages, p.stage_bytes,
               static_cast<int64_t>(blockIdx.x) * MOM_WARPS + warp,
               static_cast<int64_t>(gridDim.x) * MOM_WARPS, p.T, p.Hq, p.Hkv, DH, p.q, p.k,
               p.cos_t, p.sin_t, p.pos, p.max_pos, p.split, flags);

    double acc[2][2][5];  // [stream][pair][Sa, Sb, Saa, Sab, Sbb]
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int f = 0; f < 5; ++f) acc[s][u][f] = 0.0;

    for (int64_t n = 0; n < pipe.ntok; ++n) {
        const uint8_t *st = pipe.wait(n, flags);
        if (st == nullptr) break;
        const float *ct = reinterpret_cast<const float *>(st + pipe.table_offset());
        float2 c = *reinterpret_cast<const float2 *>(ct + k0);
        float2 s = *reinterpret_cast<const float2 *>(ct + P + k0);
        if (p.split) {  // high row turned by low row: c = fma(ch, cl, -(sh*sl)), s = fma(ch, sl, sh*cl)
            const float2 ch = *reinterpret_cast<const float2 *>(ct + 2 * P + k0);
            const float2 sh = *reinterpret_cast<const float2 *>(ct + 3 * P + k0);
            const float2 cl = c, sl = s;
            c = __ffma2_rn(ch, cl, __fmul2_rn(sh, make_float2(-sl.x, -sl.y)));
            s = __ffma2_rn(ch, sl, __fmul2_rn(sh, cl));
        }
        const float2 ns = make_float2(-s.x, -s.y);
#pragma unroll 4
        for (int r = sub; r < p.Hq; r += RPS) {
            float2 a, b;
            load_pairs<DH, STYLE>(st + r * ROWB, lr, a, b);
            // RoPE: a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c), the transform's fp32 steps
            accumulate(acc[0], __ffma2_rn(a, c, __fmul2_rn(b, ns)), __ffma2_rn(a, s, __fmul2_rn(b, c)));
        }
        const uint8_t *kst = st + pipe.qbytes;
#pragma unroll 4
        for (int r = sub; r < p.Hkv; r += RPS) {
            float2 a, b;
            load_pairs<DH, STYLE>(kst + r * ROWB, lr, a, b);
            accumulate(acc[1], __ffma2_rn(a, c, __fmul2_rn(b, ns)), __ffma2_rn(a, s, __fmul2_rn(b, c)));
        }
        pipe.release(n, flags);
    }

    // half-warps of d_h = 64 hold the same pairs
    if (RPS == 2) {
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int f = 0; f < 5; ++f) acc[s][u][f] += __shfl_xor_sync(FULL_MASK, acc[s][u][f], 16);
    }
    __syncthreads();  // every warp is done with its stages (no copy in flight)
    if (sub == 0) {
        double *mine = red + (warp * 32 + lr) * 20;
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int f = 0; f < 5; ++f) mine[(s * 2 + u) * 5 + f] = acc[s][u][f];
    }
    __syncthreads();
    // one thread per (stream, pair, sum): add the warps in order
    for (int i = threadIdx.x; i < 2 * P * 5; i += MOM_WARPS * 32) {
        const int s = i / (P * 5), k = (i / 5) % P, f = i % 5;
        const int ln = k / 2, u = k % 2;
        double sum = 0.0;
        for (int w = 0; w < MOM_WARPS; ++w) sum += red[(w * 32 + ln) * 20 + (s * 2 + u) * 5 + f];
        if (!isfinite(sum)) flags |= ST_NONFINITE;
        p.partials[static_cast<int64_t>(blockIdx.x) * 2 * P * 5 + i] = sum;
    }
    if (flags && p.status) atomicOr(p.status, flags);
}

// moments[s][k][0] += rows of stream s; moments[s][k][1 + f] += the CTA partials, added by
// one warp per output in a fixed order (lane-strided, then a fixed shuffle tree).
__global__ void k_moments_final(const double *__restrict__ partials, int ctas, int64_t rows_q,
                                int64_t rows_k, int P, double *__restrict__ moments)
{
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int nout = 2 * P * 5;
    if (w >= nout) return;  // whole warps leave together
    double sum = 0.0;
    for (int c = lane; c < ctas; c += 32) sum += partials[static_cast<int64_t>(c) * nout + w];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, o);
    if (lane == 0) {
        const int s = w / (P * 5), k = (w / 5) % P, f = w % 5;
        moments[(s * P + k) * 6 + 1 + f] += sum;
        if (f == 0) moments[(s * P + k) * 6] += static_cast<double>(s == 0 ? rows_q : rows_k);
    }
}

}  // namespace

template <int DH, int STYLE>
cudaError_t moments_partial_launch(const MomentsParams &p, const DeviceInfo &dev, int max_ctas,
                                   int *ctas_used, cudaStream_t stream)
{
    *ctas_used = 0;
    if (p.T <= 0) return cudaSuccess;
    const int SB = token_stage_bytes(p.Hq, p.Hkv, DH, p.split);
    auto kern = k_moments_partial<DH, STYLE>;
    PipeLaunch pl;
    cudaError_t e = plan_pipeline(kern, MOM_WARPS, SB, MOM_BAR_BYTES, MOM_RED_BYTES, MOM_MAX_STAGES,
                                  MOM_WANT_CTAS, p.T, max_ctas, dev, &pl);
    if (e != cudaSuccess) return e;
    MomentsParams q = p;
    q.stages = pl.stages;
    q.stage_bytes = SB;
    kern<<<pl.grid, MOM_WARPS * 32, pl.smem, stream>>>(q);
    *ctas_used = pl.grid;
    return cudaGetLastError();
}

template cudaError_t moments_partial_launch<64, ROPE_HALF>(const MomentsParams &, const DeviceInfo &, int, int *, cudaStream_t);
template cudaError_t moments_partial_launch<64, ROPE_INTERLEAVED>(const MomentsParams &, const DeviceInfo &, int, int *, cudaStream_t);
template cudaError_t moments_partial_launch<128, ROPE_HALF>(const MomentsParams &, const DeviceInfo &, int, int *, cudaStream_t);
template cudaError_t moments_partial_launch<128, ROPE_INTERLEAVED>(const MomentsParams &, const DeviceInfo &, int, int *, cudaStream_t);

cudaError_t moments_final_launch(const double *partials, int ctas, int64_t rows_q, int64_t rows_k,
                                 int P, double *moments, cudaStream_t stream)
{
    const int threads = 2 * P * 5 * 32;
    k_moments_final<<<(threads + 255) / 256, 256, 0, stream>>>(partials, ctas, rows_q, rows_k, P,
                                                               moments);
    return cudaGetLastError();
}

}  // namespace qkq

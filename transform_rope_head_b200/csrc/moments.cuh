// Device code of the calibration moments, shared by the moments kernel and the calibrating
// transform (which accumulates the same sums from the tokens it has staged anyway).
//
// Per stream (Q, K) and frequency pair k: Sa, Sb, Saa, Sab, Sbb of the post-RoPE (pre-mixing)
// values, pooled over heads and tokens ("When Local Variance Optimality Is Not Enough:
// RoPE-Aligned Q/K Rotations for Dynamic 4-Bit Quantisation", "Estimation strategies":
// raw accumulators pooled before centring).  Lanes map to pairs: a lane owns two adjacent
// pairs (both channels of each); 32 lanes cover one row at d_h = 128 (16 at d_h = 64, the
// half-warps taking alternate rows).  RoPE uses the transform's fp32 steps; the values are
// widened to fp64 (products of fp32 values are exact in fp64) and summed per lane.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace qkq {

// [stream][pair of the lane][Sa, Sb, Saa, Sab, Sbb]
using MomentAcc = double[2][2][5];

__device__ __forceinline__ void moments_clear(MomentAcc &acc)
{
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int f = 0; f < 5; ++f) acc[s][u][f] = 0.0;
}

__device__ __forceinline__ void moments_add(double (&acc)[2][5], float2 a, float2 b)
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
__device__ __forceinline__ void moments_load_pairs(const uint8_t *row, int lr, float2 &a, float2 &b)
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

// Lane roles for a warp: lr = pair slot (pairs 2 lr, 2 lr + 1), sub = row offset of the
// half-warp (d_h = 64), RPS = rows per warp step.
template <int DH>
struct MomentLanes {
    static constexpr int P = DH / 2;
    static constexpr int LPR = P / 2;     // lanes per row: 32 (d_h 128) or 16 (d_h 64)
    static constexpr int RPS = 32 / LPR;  // rows per warp step
};

// Add one staged token: Hq query rows at q_rows, Hkv key rows at k_rows (bf16, d_h each), and
// its table rows at tab (cos, sin; or low cos, low sin, high cos, high sin for a split table).
// UNROLL rows at a time (more conversions and fp64 updates in flight per warp: the moments
// kernel takes 8, 0.258 vs 0.266 ms at the 8B shape; the rows of each accumulator are added
// in the same order either way).
template <int DH, int STYLE, int UNROLL = 4>
__device__ __forceinline__ void moments_token(const uint8_t *q_rows, const uint8_t *k_rows,
                                              const float *tab, bool split, int Hq, int Hkv,
                                              int lr, int sub, MomentAcc &acc)
{
    using ML = MomentLanes<DH>;
    constexpr int P = ML::P;
    constexpr int ROWB = DH * 2;
    const int k0 = 2 * lr;
    float2 c = *reinterpret_cast<const float2 *>(tab + k0);
    float2 s = *reinterpret_cast<const float2 *>(tab + P + k0);
    if (split) {  // high row turned by low row: c = fma(ch, cl, -(sh*sl)), s = fma(ch, sl, sh*cl)
        const float2 ch = *reinterpret_cast<const float2 *>(tab + 2 * P + k0);
        const float2 sh = *reinterpret_cast<const float2 *>(tab + 3 * P + k0);
        const float2 cl = c, sl = s;
        c = __ffma2_rn(ch, cl, __fmul2_rn(sh, make_float2(-sl.x, -sl.y)));
        s = __ffma2_rn(ch, sl, __fmul2_rn(sh, cl));
    }
    const float2 ns = make_float2(-s.x, -s.y);
#pragma unroll UNROLL
    for (int r = sub; r < Hq; r += ML::RPS) {
        float2 a, b;
        moments_load_pairs<DH, STYLE>(q_rows + r * ROWB, lr, a, b);
        // RoPE: a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c), the transform's fp32 steps
        moments_add(acc[0], __ffma2_rn(a, c, __fmul2_rn(b, ns)), __ffma2_rn(a, s, __fmul2_rn(b, c)));
    }
#pragma unroll UNROLL
    for (int r = sub; r < Hkv; r += ML::RPS) {
        float2 a, b;
        moments_load_pairs<DH, STYLE>(k_rows + r * ROWB, lr, a, b);
        moments_add(acc[1], __ffma2_rn(a, c, __fmul2_rn(b, ns)), __ffma2_rn(a, s, __fmul2_rn(b, c)));
    }
}

// Bytes of the per-CTA reduction buffer for `warps` moment warps.
__host__ __device__ constexpr int moments_red_bytes(int warps) { return warps * 32 * 20 * 8; }

// Stash this warp's sums for the CTA reduction: red[mwarp][lane slot][20].
template <int DH>
__device__ __forceinline__ void moments_stash(MomentAcc &acc, int mwarp, int lr, int sub, double *red)
{
    using ML = MomentLanes<DH>;
    if (ML::RPS == 2) {  // half-warps of d_h = 64 hold the same pairs
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int f = 0; f < 5; ++f) acc[s][u][f] += __shfl_xor_sync(FULL_MASK, acc[s][u][f], 16);
    }
    if (sub == 0) {
        double *mine = red + (mwarp * 32 + lr) * 20;
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int f = 0; f < 5; ++f) mine[(s * 2 + u) * 5 + f] = acc[s][u][f];
    }
}

// After every moment warp stashed (a barrier in between): the CTA partial[2][P][5], one
// thread per (stream, pair, sum) adding the warps in order; NaN / Inf set ST_NONFINITE.
// mtid / mthreads: this thread's index among the moment threads and their number.
template <int DH>
__device__ __forceinline__ void moments_reduce(const double *red, int mwarps, int mtid,
                                               int mthreads, double *partial, int &flags)
{
    constexpr int P = DH / 2;
    for (int i = mtid; i < 2 * P * 5; i += mthreads) {
        const int s = i / (P * 5), k = (i / 5) % P, f = i % 5;
        const int ln = k / 2, u = k % 2;
        double sum = 0.0;
        for (int w = 0; w < mwarps; ++w) sum += red[(w * 32 + ln) * 20 + (s * 2 + u) * 5 + f];
        if (!isfinite(sum)) flags |= ST_NONFINITE;
        partial[i] = sum;
    }
}

}  // namespace qkq

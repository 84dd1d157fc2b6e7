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
#include "moments.cuh"
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
constexpr int MOM_RED_BYTES = moments_red_bytes(MOM_WARPS);

template <int DH, int STYLE>
__global__ void __launch_bounds__(MOM_WARPS * 32, QKQ_MOM_MIN_CTAS) k_moments_partial(const MomentsParams p)
{
    using ML = MomentLanes<DH>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint8_t *stage_mem = smem + MOM_BAR_BYTES;
    double *red = reinterpret_cast<double *>(stage_mem);  // reused after every warp's loop

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lr = lane % ML::LPR, sub = lane / ML::LPR;
    int flags = 0;
    TokenPipe pipe;
    pipe.start(stage_mem + static_cast<size_t>(warp) * p.stages * p.stage_bytes,
               bars + warp * MOM_MAX_STAGES, p.stages, p.stage_bytes,
               static_cast<int64_t>(blockIdx.x) * MOM_WARPS + warp,
               static_cast<int64_t>(gridDim.x) * MOM_WARPS, p.T, p.Hq, p.Hkv, DH, p.q, p.k,
               p.cos_t, p.sin_t, p.pos, p.max_pos, p.split, flags);

    MomentAcc acc;
    moments_clear(acc);
    for (int64_t n = 0; n < pipe.ntok; ++n) {
        const uint8_t *st = pipe.wait(n, flags);
        if (st == nullptr) break;
        moments_token<DH, STYLE, 8>(st, st + pipe.qbytes,
                                 reinterpret_cast<const float *>(st + pipe.table_offset()),
                                 p.split, p.Hq, p.Hkv, lr, sub, acc);
        pipe.release(n, flags);
    }
    __syncthreads();  // every warp is done with its stages (no copy in flight)
    moments_stash<DH>(acc, warp, lr, sub, red);
    __syncthreads();
    moments_reduce<DH>(red, MOM_WARPS, threadIdx.x, MOM_WARPS * 32,
                       p.partials + static_cast<int64_t>(blockIdx.x) * 2 * ML::P * 5, flags);
    if (flags && p.status) atomicOr(p.status, flags);
}

// moments[s][k][0] += rows of stream s; moments[s][k][1 + f] += the CTA partials, added by
// one warp per output in a fixed order (lane-strided, then a fixed shuffle tree).
__global__ void k_moments_final(const double *__restrict__ partials, int ctas, int64_t rows_q,
                                int64_t rows_k, int P, double *__restrict__ moments)
{
    wait_prior_grid();  // the partials are the previous kernel's output
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
    return launch_after_prior(k_moments_final, dim3((threads + 255) / 256), dim3(256), 0, stream,
                              partials, ctas, rows_q, rows_k, P, moments);
}

}  // namespace qkq

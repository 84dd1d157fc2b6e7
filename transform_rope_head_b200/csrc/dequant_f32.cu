// Measurement path on a given fp32 K~: K range and relative quantisation error of quantised
// keys against the transformed values they were quantised from ("When Local Variance
// Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for Dynamic 4-Bit Quantisation",
// "Core contributions" and "Results": K range and relative quantisation error along the
// mixing support b).
//
// Unlike the recomputing measurement (dequant_error.cu), this kernel takes K~ itself, so it
// measures codes from any producer: the butterfly transform's k_transformed_f32 output, the
// tensor-core variant's, value rows, or another library's.  Rows are [T * Hkv][d_h] fp32
// with their packed codes [T * Hkv][d_h/2] and fp16 scales [T * Hkv][d_h/group].
//
// A quad of lanes owns a row (the channel layout of rowops.cuh: lane slot l holds the
// 8-channel chunks j * 32 + l * 8, each two 16-byte loads of K~ and one 32-bit word of
// codes), eight rows per warp step; a persistent grid strides over the rows.  The
// statistics are row_stats (rowops.cuh), the same arithmetic as the recomputing kernel and
// the transform's fused statistics: fp32 sums per lane and group of scale-normalised terms,
// fp64 totals; per CTA in a fixed order, then across CTAs by k_dequant_final.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "rowops.cuh"

namespace qkq {

namespace {

constexpr int DF_WARPS = 8;
constexpr int DF_CTAS_PER_SM = 4;

template <int DH, int G>
__global__ void __launch_bounds__(DF_WARPS * 32, DF_CTAS_PER_SM)
    k_dequant_f32_partial(const DequantF32Params p)
{
    using L = Layout<DH, ROPE_HALF>;  // float2 = two neighbouring channels
    using GR = Groups<L, G>;
    __shared__ double red[DF_WARPS * 6];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane & 3, rq = lane >> 2;
    int flags = 0;
    RowStats stats;
    const int64_t rows = p.T * p.Hkv;
    const int64_t step = static_cast<int64_t>(gridDim.x) * DF_WARPS * 8;
    for (int64_t r0 = (static_cast<int64_t>(blockIdx.x) * DF_WARPS + warp) * 8; r0 < rows;
         r0 += step) {
        const int64_t row = r0 + rq;
        const bool valid = row < rows;
        const int64_t rc = valid ? row : rows - 1;  // keep every lane in the quad shuffles
        const float *xr = p.k_f32 + rc * DH;
        float2 V[L::NV];
        uint32_t cw[L::NJ];
#pragma unroll
        for (int j = 0; j < L::NJ; ++j) {
            const float4 a = __ldcs(reinterpret_cast<const float4 *>(xr + j * 32 + l * 8));
            const float4 b = __ldcs(reinterpret_cast<const float4 *>(xr + j * 32 + l * 8 + 4));
            V[j * 4 + 0] = make_float2(a.x, a.y);
            V[j * 4 + 1] = make_float2(a.z, a.w);
            V[j * 4 + 2] = make_float2(b.x, b.y);
            V[j * 4 + 3] = make_float2(b.z, b.w);
            cw[j] = __ldcs(reinterpret_cast<const uint32_t *>(p.k_codes + rc * (DH / 2)) + j * 4 + l);
        }
        float shat[GR::NG];
#pragma unroll
        for (int g = 0; g < GR::NG; ++g)
            shat[g] = __half2float(__ushort_as_half(__ldg(p.k_scales + rc * GR::NG + g)));
        // codes of V[4j + k] = channels (2k, 2k + 1) of chunk j as floats: the biased nibbles
        // c + 8 placed into 2^23 + c + 8 by a byte permutation, then 2^23 + 8 subtracted
        auto code_of = [&](int pidx) {
            const int j = pidx >> 2, k = pidx & 3;
            const uint32_t wb = cw[j] ^ 0x88888888u;
            const uint32_t ev = wb & 0x0F0F0F0Fu, od = (wb >> 4) & 0x0F0F0F0Fu;
            return __fadd2_rn(make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u | k)),
                                          __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u | k))),
                              make_float2(-8388616.0f, -8388616.0f));
        };
        row_stats<L, G>(V, code_of, shat, l, valid, stats);
    }
    reduce_row_stats(stats, red, DF_WARPS, p.partials + static_cast<int64_t>(blockIdx.x) * 6, flags);
    if (flags && p.status) atomicOr(p.status, flags);
}

template <int DH>
void (*pick_f32(int group))(DequantF32Params)
{
    switch (group) {
    case 32: return k_dequant_f32_partial<DH, 32>;
    case 64: return k_dequant_f32_partial<DH, 64>;
    case 128:
        if (DH == 128) return k_dequant_f32_partial<DH, (DH == 128 ? 128 : 64)>;
        break;
    }
    return nullptr;
}

}  // namespace

cudaError_t dequant_f32_partial_launch(const DequantF32Params &p, int d_h, int group,
                                       const DeviceInfo &dev, int max_ctas, int *ctas_used,
                                       cudaStream_t stream)
{
    *ctas_used = 0;
    if (p.T <= 0) return cudaSuccess;
    auto kern = d_h == 64 ? pick_f32<64>(group) : pick_f32<128>(group);
    if (kern == nullptr) return cudaErrorInvalidValue;
    // persistent grid: the resident CTAs, at most one warp step of rows per warp, at most
    // max_ctas (the workspace's partials)
    const int64_t rows = p.T * p.Hkv;
    int64_t grid = static_cast<int64_t>(dev.num_sms) * DF_CTAS_PER_SM;
    const int64_t need = (rows + DF_WARPS * 8 - 1) / (DF_WARPS * 8);
    if (need < grid) grid = need;
    if (max_ctas < grid) grid = max_ctas;
    if (grid < 1) grid = 1;
    kern<<<static_cast<int>(grid), DF_WARPS * 32, 0, stream>>>(p);
    *ctas_used = static_cast<int>(grid);
    return cudaGetLastError();
}

}  // namespace qkq

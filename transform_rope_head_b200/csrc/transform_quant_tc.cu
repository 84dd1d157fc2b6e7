// Tensor-core variant of the fused transform: the Hadamard mixing as a GEMM on the
// 5th-generation tensor cores (tcgen05), to measure against the butterfly.
//
// The mixing of every Hadamard mode is one matrix product per row, y = x (I (x) H_b) / sqrt(b)
// ("Methodology" of "When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K
// Rotations for Dynamic 4-Bit Quantisation": the full-head normalised Hadamard; "Core
// contributions": block Hadamard of support b; b = d_h is the full head).  Here 128 rows
// (query or key rows of consecutive tokens) form the M = 128 side of
//   D[128 x d_h] = A[128 x d_h] * B[d_h x d_h]^T,   B[n][k] = (I (x) H_b)[k][n]  (entries +-1, 0)
// with A the post-RoPE rows.  The tensor cores take bf16 operands, so each fp32 row is
// split into x = hi + lo (hi = bf16(x), lo = bf16(x - hi), 16 significant bits in all)
// and the product is accumulated in fp32 over both halves: 2 x d_h/16 MMAs of
// 128 x d_h x 16 per tile.  The accumulator lives in tensor memory (d_h columns); one
// thread per row reads it back (tcgen05.ld, 32 lanes x 32 columns) and finishes the row
// exactly like the butterfly kernel: * fp32(1/sqrt(b)), then Q -> bf16, or the K group
// quantiser.
//
// Numerics differ from the butterfly's fp32 sequence (the split drops bits below 2^-16
// of each element, and the tensor cores add in their own order), so this variant is
// checked against the fp64 definition within a derived bound, not bit for bit.
//
// One CTA of 4 warps: thread t owns row t of a tile and TMEM lane t (warp w reads lanes
// 32w .. 32w + 31).  A persistent loop walks the query tiles, then the key tiles.  Per
// tile: rows are read from HBM by their owning threads (16-byte loads), RoPE (then the pair
// angle in the pairwise mode) is applied in fp32, hi/lo are written into
// shared memory in the 128-byte-swizzled K-major layout the MMA reads, one elected thread
// issues the MMAs and commits them to an mbarrier, and all threads wait (time-bounded) and
// run the epilogue.  B is built once per CTA.  No TMA, no multicast.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace qkq {

namespace {

constexpr int TCQ_THREADS = 128;
constexpr int TCQ_M = 128;

// Split 8 fp32 values into bf16 hi and lo (x = hi + lo + O(2^-16 |x|)), packed 8 x bf16.
__device__ __forceinline__ void split8(const float (&y)[8], uint4 &hi, uint4 &lo)
{
    float h[8], d[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = __bfloat162float(__float2bfloat16_rn(y[i]));
        d[i] = y[i] - h[i];  // exact
    }
    hi = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]),
                    pack_bf16x2(h[6], h[7]));
    lo = make_uint4(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]), pack_bf16x2(d[4], d[5]),
                    pack_bf16x2(d[6], d[7]));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&x)[8])
{
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(a[i] << 16);
        x[2 * i + 1] = __uint_as_float(a[i] & 0xffff0000u);
    }
}

// The row's bf16 values, as DH / 8 16-byte words (loaded one tile ahead).
template <int DH>
struct RowRegs {
    uint4 w[DH / 8];
};

template <int DH>
__device__ __forceinline__ void load_row(RowRegs<DH> &x, const uint16_t *row)
{
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) x.w[i] = __ldg(reinterpret_cast<const uint4 *>(row) + i);
}

// RoPE (and then the pair angle) on one row, written as hi / lo into the A operands.
// Rotation a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c) with the table entry; in the pairwise
// mode the result is turned by phi with the same two lines, as the butterfly kernel does.
template <int DH, int STYLE, bool PAIRROT>
__device__ __forceinline__ void rope_row_to_operands(const RowRegs<DH> &row, const float *ct,
                                                     const float *st, const float *phi_tab,
                                                     uint8_t *a_hi, uint8_t *a_lo, int r)
{
    constexpr int P = DH / 2;
    // the table entries of pairs k0 .. k0 + N - 1 (16-byte loads)
    auto coeffs = [&](int k0, auto &c, auto &s) {
        constexpr int N = sizeof(c) / sizeof(float);
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 cv = __ldg(reinterpret_cast<const float4 *>(ct + k0 + i));
            const float4 sv = __ldg(reinterpret_cast<const float4 *>(st + k0 + i));
            c[i] = cv.x; c[i + 1] = cv.y; c[i + 2] = cv.z; c[i + 3] = cv.w;
            s[i] = sv.x; s[i + 1] = sv.y; s[i + 2] = sv.z; s[i + 3] = sv.w;
        }
    };
    // the pair rotation of pair k after RoPE (pairwise mode)
    auto turn_phi = [&](int k, float &a, float &b) {
        if (PAIRROT) {
            const float cp = phi_tab[k], sp = phi_tab[P + k];
            const float a2 = __fmaf_rn(a, cp, -__fmul_rn(b, sp));
            const float b2 = __fmaf_rn(a, sp, __fmul_rn(b, cp));
            a = a2;
            b = b2;
        }
    };
    if (STYLE == ROPE_HALF) {
        // pairs (k, k + P): 8 pairs per step, both halves written
#pragma unroll
        for (int k0 = 0; k0 < P; k0 += 8) {
            float xa[8], xb[8], ya[8], yb[8], cc[8], ss[8];
            bf16x8_to_f32(row.w[k0 / 8], xa);
            bf16x8_to_f32(row.w[(P + k0) / 8], xb);
            coeffs(k0, cc, ss);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float c = cc[i], s = ss[i];
                ya[i] = __fmaf_rn(xa[i], c, -__fmul_rn(xb[i], s));
                yb[i] = __fmaf_rn(xa[i], s, __fmul_rn(xb[i], c));
                turn_phi(k0 + i, ya[i], yb[i]);
            }
            uint4 h, l;
            split8(ya, h, l);
            *reinterpret_cast<uint4 *>(a_hi + sw128_offset<TCQ_M>(r, k0)) = h;
            *reinterpret_cast<uint4 *>(a_lo + sw128_offset<TCQ_M>(r, k0)) = l;
            split8(yb, h, l);
            *reinterpret_cast<uint4 *>(a_hi + sw128_offset<TCQ_M>(r, P + k0)) = h;
            *reinterpret_cast<uint4 *>(a_lo + sw128_offset<TCQ_M>(r, P + k0)) = l;
        }
    } else {
        // pairs (2k, 2k + 1): 8 consecutive channels = 4 pairs per step
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 8) {
            float x[8], y[8], cc[4], ss[4];
            bf16x8_to_f32(row.w[c0 / 8], x);
            coeffs(c0 / 2, cc, ss);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float c = cc[i], s = ss[i];
                y[2 * i] = __fmaf_rn(x[2 * i], c, -__fmul_rn(x[2 * i + 1], s));
                y[2 * i + 1] = __fmaf_rn(x[2 * i], s, __fmul_rn(x[2 * i + 1], c));
                turn_phi(c0 / 2 + i, y[2 * i], y[2 * i + 1]);
            }
            uint4 h, l;
            split8(y, h, l);
            *reinterpret_cast<uint4 *>(a_hi + sw128_offset<TCQ_M>(r, c0)) = h;
            *reinterpret_cast<uint4 *>(a_lo + sw128_offset<TCQ_M>(r, c0)) = l;
        }
    }
}

// Shared memory: [A hi | A lo | B | bars, tmem slot, phi] with A and B 1024-aligned.
template <int DH>
struct TcSmem {
    static constexpr int A_BYTES = TCQ_M * DH * 2;
    static constexpr int B_BYTES = DH * DH * 2;
    static constexpr int OFF_AHI = 0;
    static constexpr int OFF_ALO = A_BYTES;
    static constexpr int OFF_B = 2 * A_BYTES;
    static constexpr int OFF_MISC = 2 * A_BYTES + B_BYTES;        // mbarrier (8) + tmem slot (4)
    static constexpr int OFF_PHI = OFF_MISC + 16;                 // cos, sin of phi: 2 x DH/2 floats
    static constexpr int BYTES = OFF_PHI + DH * 4;
    static constexpr int ALLOC = BYTES + 1024;                    // room to align the base
};

template <int DH, int STYLE, bool PAIRROT, int G>
__global__ void __launch_bounds__(TCQ_THREADS) k_transform_quant_tc(const TransformParams p, int b)
{
    using S = TcSmem<DH>;
    constexpr int P = DH / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *a_hi = smem + S::OFF_AHI;
    uint8_t *a_lo = smem + S::OFF_ALO;
    uint8_t *bmat = smem + S::OFF_B;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + S::OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::OFF_MISC + 8);
    float *phi_tab = reinterpret_cast<float *>(smem + S::OFF_PHI);
    const int tid = threadIdx.x, warp = tid >> 5;
    int flags = 0;

    // B[n][k] = (I (x) H_b)[k][n]: +-1 on the diagonal blocks (Sylvester order), else 0
    for (int i = tid; i < DH * DH; i += TCQ_THREADS) {
        const int n = i / DH, k = i % DH;
        uint16_t v = 0;
        if (n / b == k / b) v = (__popc((n % b) & (k % b)) & 1) ? 0xBF80u : 0x3F80u;
        *reinterpret_cast<uint16_t *>(bmat + sw128_offset<DH>(n, k)) = v;
    }
    if (PAIRROT)
        for (int i = tid; i < P; i += TCQ_THREADS) {
            const double ph = static_cast<double>(p.phi[i]);
            phi_tab[i] = static_cast<float>(cos(ph));
            phi_tab[P + i] = static_cast<float>(sin(ph));
        }
    if (tid == 0) {
        mbar_init(smem_addr(bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), DH);
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // B written by the generic proxy, read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t a_hi_s = smem_addr(a_hi), a_lo_s = smem_addr(a_lo), b_s = smem_addr(bmat);
    constexpr uint32_t IDESC = idesc_bf16(DH);

    const int64_t q_rows = p.T * p.Hq, k_rows = p.T * p.Hkv;
    const int64_t q_tiles = (q_rows + TCQ_M - 1) / TCQ_M, k_tiles = (k_rows + TCQ_M - 1) / TCQ_M;
    const int64_t n_tiles = q_tiles + k_tiles;
    // this thread's row of tile `tile`: (stream, clamped row index, valid)
    auto row_of = [&](int64_t tile, bool &is_q, int64_t &Rc, bool &valid) {
        is_q = tile < q_tiles;
        const int64_t R = (is_q ? tile : tile - q_tiles) * TCQ_M + tid;
        const int64_t nrows = is_q ? q_rows : k_rows;
        valid = R < nrows;
        Rc = valid ? R : nrows - 1;  // ragged tail: compute a real row, store nothing
    };
    uint32_t phase = 0;
    bool failed = false;
    RowRegs<DH> x;  // the rows of the tile being processed, loaded one tile ahead
    if (static_cast<int64_t>(blockIdx.x) < n_tiles) {
        bool q0, v0;
        int64_t r0;
        row_of(blockIdx.x, q0, r0, v0);
        load_row<DH>(x, (q0 ? p.q : p.k) + r0 * DH);
    }
    for (int64_t tile = blockIdx.x; tile < n_tiles && !failed; tile += gridDim.x) {
        bool is_q, valid;
        int64_t Rc;
        row_of(tile, is_q, Rc, valid);
        const int H = is_q ? p.Hq : p.Hkv;
        const int64_t t = Rc / H;
        const int64_t m = clamp_pos(__ldg(p.pos + t), p.max_pos, flags);
        rope_row_to_operands<DH, STYLE, PAIRROT>(x, p.cos_t + m * P, p.sin_t + m * P, phi_tab,
                                                 a_hi, a_lo, tid);
        fence_proxy_async_smem();  // operands written by this thread, read by the tensor cores
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int ks = 0; ks < DH / 16; ++ks) {
                    // K-step ks: K-block ks / 4, 32 bytes further per step inside it
                    const uint32_t koff = (ks >> 2) * (TCQ_M * 128) + (ks & 3) * 32;
                    const uint32_t kbo = (ks >> 2) * (DH * 128) + (ks & 3) * 32;
                    mma_bf16(tmem, sw128_desc((h ? a_lo_s : a_hi_s) + koff), sw128_desc(b_s + kbo),
                             IDESC, (h | ks) ? 1u : 0u);
                }
            mma_commit(smem_addr(bar));
        }
        // the next tile's rows are read while the tensor cores run and the epilogue stores
        if (tile + gridDim.x < n_tiles) {
            bool qn, vn;
            int64_t rn;
            row_of(tile + gridDim.x, qn, rn, vn);
            load_row<DH>(x, (qn ? p.q : p.k) + rn * DH);
        }
        const bool ok = mbar_wait_bounded(smem_addr(bar), phase);
        phase ^= 1u;
        if (__syncthreads_or(!ok)) {
            // the MMAs did not complete in time: give them one more bounded wait before the
            // tensor memory is released, and stop
            flags |= ST_TIMEOUT;
            failed = true;
            break;
        }
        tc_fence_after();

        // epilogue: thread tid reads TMEM lane tid
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float kappa = p.kappa;
        if (is_q) {
            uint16_t *dst = p.q_out + Rc * DH;
#pragma unroll
            for (int c0 = 0; c0 < DH; c0 += 32) {
                float v[32];
                tmem_ld32(lane_addr + c0, v);
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__fmul_rn(v[i], kappa), __fmul_rn(v[i + 1], kappa));
                        w.y = pack_bf16x2(__fmul_rn(v[i + 2], kappa), __fmul_rn(v[i + 3], kappa));
                        w.z = pack_bf16x2(__fmul_rn(v[i + 4], kappa), __fmul_rn(v[i + 5], kappa));
                        w.w = pack_bf16x2(__fmul_rn(v[i + 6], kappa), __fmul_rn(v[i + 7], kappa));
                        *reinterpret_cast<uint4 *>(dst + c0 + i) = w;
                    }
                }
            }
        } else {
#pragma unroll
            for (int g0 = 0; g0 < DH; g0 += G) {
                // pass 1: group max|y|
                float am = 0.0f;
#pragma unroll
                for (int c0 = g0; c0 < g0 + G; c0 += 32) {
                    float v[32];
                    tmem_ld32(lane_addr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) am = max_abs_nan(am, __fmul_rn(v[i], kappa));
                }
                am = fabsf(am);
                if (!(am <= 3.402823466e38f)) flags |= ST_NONFINITE;
                const bool zero = !(am >= 0x1p-125f);
                const float r = zero ? 0.0f : __fdiv_rn(7.0f, am);
                const float s = zero ? 0.0f : __fdiv_rn(am, 7.0f);
                // pass 2: codes (the exact product y*r rounded once, ties to even), packed
#pragma unroll
                for (int c0 = g0; c0 < g0 + G; c0 += 32) {
                    float v[32];
                    tmem_ld32(lane_addr + c0, v);
                    uint32_t words[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t w = 0;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float y = __fmul_rn(v[j * 8 + e], kappa);
                            const uint32_t q = __float_as_uint(__fmaf_rn(y, r, 12582912.0f));
                            w |= (q & 0xFu) << (4 * e);
                        }
                        words[j] = w;
                    }
                    if (valid) {
                        uint32_t *cw = reinterpret_cast<uint32_t *>(p.k_codes + Rc * P + c0 / 2);
#pragma unroll
                        for (int j = 0; j < 4; ++j) cw[j] = words[j];
                        if (p.k_f32 != nullptr)
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4 *>(p.k_f32 + Rc * DH + c0 + i) =
                                    make_float4(__fmul_rn(v[i], kappa), __fmul_rn(v[i + 1], kappa),
                                                __fmul_rn(v[i + 2], kappa), __fmul_rn(v[i + 3], kappa));
                    }
                }
                if (valid) {
                    const uint16_t hb = __half_as_ushort(__float2half_rn(s));
                    if ((hb & 0x7fffu) == 0x7c00u && am <= 3.402823466e38f) flags |= ST_SCALE_OVERFLOW;
                    p.k_scales[Rc * (DH / G) + g0 / G] = hb;
                }
            }
        }
        tc_fence_before();
        __syncthreads();  // every lane read back before the next tile's MMAs overwrite it
    }
    if (failed) mbar_wait_bounded(smem_addr(bar), phase ^ 1u);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, DH);
    if (flags && p.status) atomicOr(p.status, flags);
}

using TcKernel = void (*)(TransformParams, int);

// Resident CTAs per SM from the SM's shared memory (each CTA also keeps 1 KB for the
// runtime), its registers and its tensor memory (tmem_cols of 512 columns per CTA).  The
// occupancy calculator reports one CTA for these kernels, while the hardware holds two
// (ncu: launch__occupancy_limit_shared_mem 2), so the limit is computed here.
inline cudaError_t tc_resident_ctas(const void *kern, size_t smem, int tmem_cols,
                                    const DeviceInfo &dev, int *per_sm)
{
    int ignored = 0;  // sets the kernel's shared-memory attributes (and caches)
    cudaError_t e = resident_ctas(kern, TCQ_THREADS, smem, dev, &ignored);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    const int regs_per_warp = ((fa.numRegs + 7) / 8) * 8 * 32;
    const int by_regs = 65536 / (regs_per_warp * (TCQ_THREADS / 32));
    const int by_smem = static_cast<int>(static_cast<size_t>(dev.smem_per_sm) / (smem + 1024));
    const int by_tmem = 512 / tmem_cols;
    int n = by_regs < by_smem ? by_regs : by_smem;
    if (n > by_tmem) n = by_tmem;
    *per_sm = n;
    return cudaSuccess;
}

template <int DH, int STYLE, int G>
TcKernel pick_tc(int mode)
{
    return mode == MODE_PAIRWISE_HADAMARD ? k_transform_quant_tc<DH, STYLE, true, G>
                                          : k_transform_quant_tc<DH, STYLE, false, G>;
}

}  // namespace

template <int DH, int STYLE>
cudaError_t transform_quant_tc_launch(const TransformParams &p, int mode, int b, int group,
                                      const DeviceInfo &dev, cudaStream_t stream)
{
    if (mode != MODE_HADAMARD && mode != MODE_PAIRWISE_HADAMARD && mode != MODE_BLOCK_HADAMARD)
        return cudaErrorInvalidValue;
    const int n = mode == MODE_BLOCK_HADAMARD ? b : DH;
    TcKernel kern = nullptr;
    switch (group) {
    case 32: kern = pick_tc<DH, STYLE, 32>(mode); break;
    case 64: kern = pick_tc<DH, STYLE, 64>(mode); break;
    case 128:
        if (DH == 128) kern = pick_tc<DH, STYLE, (DH == 128 ? 128 : 64)>(mode);
        break;
    }
    if (kern == nullptr) return cudaErrorInvalidValue;
    const int64_t tiles = (p.T * p.Hq + TCQ_M - 1) / TCQ_M + (p.T * p.Hkv + TCQ_M - 1) / TCQ_M;
    if (tiles == 0) return cudaSuccess;
    const size_t smem = TcSmem<DH>::ALLOC;
    int per_sm = 0;
    cudaError_t e = tc_resident_ctas(reinterpret_cast<const void *>(kern), smem, DH, dev, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = static_cast<int64_t>(dev.num_sms) * per_sm;
    if (grid > tiles) grid = tiles;
    kern<<<static_cast<int>(grid), TCQ_THREADS, smem, stream>>>(p, n);
    return cudaGetLastError();
}

#if defined(QKQ_DH) && defined(QKQ_STYLE)
template cudaError_t transform_quant_tc_launch<QKQ_DH, QKQ_STYLE>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t);
#else
template cudaError_t transform_quant_tc_launch<64, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t);
template cudaError_t transform_quant_tc_launch<64, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t);
template cudaError_t transform_quant_tc_launch<128, ROPE_HALF>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t);
template cudaError_t transform_quant_tc_launch<128, ROPE_INTERLEAVED>(const TransformParams &, int, int, int, const DeviceInfo &, cudaStream_t);
#endif

}  // namespace qkq

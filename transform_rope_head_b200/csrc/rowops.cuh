// Per-row register code of the transform: four lanes ("a quad") own one row of
// d_h channels.  Used by the fused transform kernel and by the measurement kernel,
// so both compute the transformed K bit for bit alike.
//
// Channel layout.  Lane slot l = lane & 3 of a quad holds NCH = d_h/4 channels:
//   element i (0 <= i < NCH)  <->  channel c(i) = (i >> 3) * 32 + l * 8 + (i & 7)
// so each 8-channel chunk j = i >> 3 is one 16-byte vector in memory, the quad
// reads/writes 64 contiguous bytes per chunk, channel bits 0-2 and 5-6 are
// register bits and channel bits 3-4 are the quad's lane bits.
//
// Elements live in float2 registers for the packed sm_100 fp32x2 instructions.
// The float2 pairs elements i and i ^ (1 << PB): PB = 0 for rotate-half RoPE (its
// pairs (k, k + d_h/2) then sit in two float2s at the same component), PB = 1 for
// interleaved RoPE (pairs (2k, 2k+1) become float2s (a, a'), (b, b')).
//
// fp32 order of operations (the contract the CPU oracle's fp32 sequence follows):
//   rotation of pair (a, b) by table (c, s):  a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c);
//   a split table's entry is first composed from its high and low rows (load_rope);
//   the pairwise modes then turn every pair of the RoPE output by phi with the same two
//   lines (PairCoeffs): RoPE first, then the pair rotation, each rounded on its own;
//   butterflies (u, v) -> (u+v, u-v) at strides 1, 2, 4, ..., n/2, then * fp32(1/sqrt(n));
//   quantiser per group: r = fp32(7/amax), code = the exact product x*r rounded once to
//   the nearest integer (ties to even; one fused multiply-add), s = fp32(amax/7).
// The packed instructions round each component exactly like their scalar forms.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace qkq {

template <int DH, int STYLE>
struct Layout {
    static_assert(DH == 64 || DH == 128, "d_h must be 64 or 128");
    static constexpr int NCH = DH / 4;                 // elements per lane per row
    static constexpr int NV = NCH / 2;                 // float2 registers per row
    static constexpr int NJ = NCH / 8;                 // 8-channel chunks per lane
    static constexpr int NT = NV / 2;                  // float2 table entries (pairs / 2)
    static constexpr int PB = (STYLE == ROPE_HALF) ? 0 : 1;

    __host__ __device__ static constexpr int vidx(int i)
    {
        return PB == 0 ? (i >> 1) : ((i & 1) | ((i >> 2) << 1));
    }
    __host__ __device__ static constexpr int comp(int i) { return (i >> PB) & 1; }
    __host__ __device__ static constexpr int elem(int p, int c)
    {
        return PB == 0 ? (p * 2 + c) : ((p & 1) | (c << 1) | ((p >> 1) << 2));
    }
    // float2 index of the first / second channel of the q-th pair-of-pairs
    __host__ __device__ static constexpr int pa(int q) { return PB == 0 ? q : 2 * q; }
    __host__ __device__ static constexpr int pb(int q) { return PB == 0 ? q + NV / 2 : 2 * q + 1; }
};

template <class L>
__device__ __forceinline__ float get_el(const float2 (&V)[L::NV], int i)
{
    return L::comp(i) ? V[L::vidx(i)].y : V[L::vidx(i)].x;
}

template <class L>
__device__ __forceinline__ void set_el(float2 (&V)[L::NV], int i, float f)
{
    if (L::comp(i))
        V[L::vidx(i)].y = f;
    else
        V[L::vidx(i)].x = f;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Load one row of bf16 (row points at the row start; shared or global memory).
template <class L>
__device__ __forceinline__ void load_row_bf16(float2 (&V)[L::NV], const uint8_t *row, int l)
{
#pragma unroll
    for (int j = 0; j < L::NJ; ++j) {
        const uint4 w = *reinterpret_cast<const uint4 *>(row + j * 64 + l * 16);
        const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            set_el<L>(V, j * 8 + e, (e & 1) ? bf16hi(wd[e >> 1]) : bf16lo(wd[e >> 1]));
    }
}

// The lane's cos/sin entries of the pairs it holds, from a table row of d_h/2
// floats (pair k at index k), as float2 (pair of the q-th float2 pair-of-pairs).
template <class L>
__device__ __forceinline__ void load_pair_table(float2 (&T)[L::NT], const float *row, int l)
{
    if (L::PB == 0) {
        // pairs k = j*32 + l*8 + e for the first-channel chunks j < NJ/2
#pragma unroll
        for (int j = 0; j < L::NJ / 2; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(row + j * 32 + l * 8);
            const float4 b = *reinterpret_cast<const float4 *>(row + j * 32 + l * 8 + 4);
            T[j * 4 + 0] = make_float2(a.x, a.y);
            T[j * 4 + 1] = make_float2(a.z, a.w);
            T[j * 4 + 2] = make_float2(b.x, b.y);
            T[j * 4 + 3] = make_float2(b.z, b.w);
        }
    } else {
        // pairs k = j*16 + l*4 + {0..3} for every chunk j
#pragma unroll
        for (int j = 0; j < L::NJ; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(row + j * 16 + l * 4);
            T[j * 2 + 0] = make_float2(a.x, a.y);
            T[j * 2 + 1] = make_float2(a.z, a.w);
        }
    }
}

// (a, b) -> (fma(a, c, -(b*s)), fma(a, s, b*c)) on every pair the lane holds (the negated
// product is an operand of the packed fused multiply-add, no table of -s is needed).
template <class L>
__device__ __forceinline__ void rotate_pairs(float2 (&V)[L::NV], const float2 (&C)[L::NT],
                                             const float2 (&S)[L::NT])
{
#pragma unroll
    for (int q = 0; q < L::NT; ++q) {
        const float2 a = V[L::pa(q)], b = V[L::pb(q)];
        const float2 t = __fmul2_rn(b, S[q]);
        V[L::pa(q)] = __ffma2_rn(a, C[q], make_float2(-t.x, -t.y));
        V[L::pb(q)] = __ffma2_rn(a, S[q], __fmul2_rn(b, C[q]));
    }
}

// Turn the table entries (c, s) by (cl, sl) with the fp32 steps of a pair rotation:
//   c' = fma(c, cl, -(s*sl)),  s' = fma(c, sl, s*cl)
// (the angle-addition rule of two plane rotations).  Used for the split RoPE table only:
// a position's entry is its high row turned by its low row.
template <class L>
__device__ __forceinline__ void turn_table(float2 (&C)[L::NT], float2 (&S)[L::NT],
                                           const float2 (&CL)[L::NT], const float2 (&SL)[L::NT])
{
#pragma unroll
    for (int q = 0; q < L::NT; ++q) {
        const float2 c = C[q], s = S[q];
        const float2 t = __fmul2_rn(s, SL[q]);
        C[q] = __ffma2_rn(c, CL[q], make_float2(-t.x, -t.y));
        S[q] = __ffma2_rn(c, SL[q], __fmul2_rn(s, CL[q]));
    }
}

// The head-shared pair rotation: every row of the pairwise modes takes it after RoPE, its own
// rounded step with the RoPE lines (paper summary, "Methodology" item 2: the pairwise
// rotation acts on the post-RoPE pairs).  The coefficients (cos phi, sin phi) come from the
// CTA's pair table in shared memory (cos [P], sin [P]); PairCoeffs reads the lane's entries
// once and holds them in registers, PairCoeffsShared re-reads them for every row (for
// kernels whose registers are already taken).
template <class L>
struct PairCoeffs {
    float2 c[L::NT], s[L::NT];
    __device__ __forceinline__ void load(const float *tab, int P, int l)
    {
        load_pair_table<L>(c, tab, l);
        load_pair_table<L>(s, tab + P, l);
    }
    __device__ __forceinline__ void turn(float2 (&V)[L::NV]) const { rotate_pairs<L>(V, c, s); }
};

// Four floats from shared memory, read at every call (volatile: the compiler must not keep
// them in registers across rows, which is the point of PairCoeffsShared).
__device__ __forceinline__ float4 lds_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

template <class L>
struct PairCoeffsShared {
    uint32_t tab = 0;  // shared-window address of the pair table
    int P = 0, l = 0;
    __device__ __forceinline__ void load(const float *t, int np, int lane_slot)
    {
        tab = smem_addr(t);
        P = np;
        l = lane_slot;
    }
    // load_pair_table's entries of the lane from a shared-memory table row
    __device__ __forceinline__ void entries(float2 (&T)[L::NT], uint32_t row) const
    {
        if (L::PB == 0) {
#pragma unroll
            for (int j = 0; j < L::NJ / 2; ++j) {
                const float4 a = lds_f4(row + 4u * (j * 32 + l * 8));
                const float4 b = lds_f4(row + 4u * (j * 32 + l * 8 + 4));
                T[j * 4 + 0] = make_float2(a.x, a.y);
                T[j * 4 + 1] = make_float2(a.z, a.w);
                T[j * 4 + 2] = make_float2(b.x, b.y);
                T[j * 4 + 3] = make_float2(b.z, b.w);
            }
        } else {
#pragma unroll
            for (int j = 0; j < L::NJ; ++j) {
                const float4 a = lds_f4(row + 4u * (j * 16 + l * 4));
                T[j * 2 + 0] = make_float2(a.x, a.y);
                T[j * 2 + 1] = make_float2(a.z, a.w);
            }
        }
    }
    __device__ __forceinline__ void turn(float2 (&V)[L::NV]) const
    {
        float2 c[L::NT], s[L::NT];
        entries(c, tab);
        entries(s, tab + 4u * P);
        rotate_pairs<L>(V, c, s);
    }
};

// The lane's RoPE coefficients (c, s) of the token from its table rows in a stage: cos and
// sin rows, or with a split table the low rows (m % 64) then the high rows (64 + m / 64),
// high turned by low: c = fma(c_h, c_l, -(s_h*s_l)), s = fma(c_h, s_l, s_h*c_l) (the
// angle-addition rule of two plane rotations).
template <class L>
__device__ __forceinline__ void load_rope(float2 (&C)[L::NT], float2 (&S)[L::NT],
                                          const float *tab, int P, bool split, int l)
{
    if (split) {
        float2 CL[L::NT], SL[L::NT];
        load_pair_table<L>(CL, tab, l);
        load_pair_table<L>(SL, tab + P, l);
        load_pair_table<L>(C, tab + 2 * P, l);
        load_pair_table<L>(S, tab + 3 * P, l);
        turn_table<L>(C, S, CL, SL);
    } else {
        load_pair_table<L>(C, tab, l);
        load_pair_table<L>(S, tab + P, l);
    }
}

// Butterfly stage on register bit rb of the element index.
template <class L, int RB>
__device__ __forceinline__ void stage_reg(float2 (&V)[L::NV])
{
    if (RB == L::PB) {
        // (x, y) -> (x*1 + y, y*(-1) + x): each component one rounding of x + y and x - y
        const float2 pm = make_float2(1.0f, -1.0f);
#pragma unroll
        for (int p = 0; p < L::NV; ++p) V[p] = __ffma2_rn(V[p], pm, make_float2(V[p].y, V[p].x));
    } else {
        constexpr int VB = (RB > L::PB) ? RB - 1 : RB;
        const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
        for (int p = 0; p < L::NV; ++p) {
            if (p & (1 << VB)) continue;
            const float2 u = V[p], w = V[p | (1 << VB)];
            V[p] = __fadd2_rn(u, w);
            V[p | (1 << VB)] = __ffma2_rn(w, neg1, u);  // u - w, one rounding
        }
    }
}

// Butterfly stage across the quad: lane bit `m` (1 or 2) of the slot l.
template <class L>
__device__ __forceinline__ void stage_lane(float2 (&V)[L::NV], int l, int m)
{
    const float sg = (l & m) ? -1.0f : 1.0f;
    const float2 s2 = make_float2(sg, sg);
#ifdef QKQ_SHFL_TWO_PHASE
    float2 P2[L::NV];
#pragma unroll
    for (int p = 0; p < L::NV; ++p)
        P2[p] = make_float2(__shfl_xor_sync(FULL_MASK, V[p].x, m), __shfl_xor_sync(FULL_MASK, V[p].y, m));
#pragma unroll
    for (int p = 0; p < L::NV; ++p) V[p] = __ffma2_rn(V[p], s2, P2[p]);
#else
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const float px = __shfl_xor_sync(FULL_MASK, V[p].x, m);
        const float py = __shfl_xor_sync(FULL_MASK, V[p].y, m);
        // lower lane: own + partner; upper lane: partner - own
        V[p] = __ffma2_rn(V[p], s2, make_float2(px, py));
    }
#endif
}

// Normalised fast Walsh-Hadamard transform over contiguous blocks of NMIX channels
// (NMIX = 1: nothing).  Channel bit t: t < 3 register bit t; t = 3, 4 quad lane bits;
// t = 5, 6 register bits 3, 4.  Stages run t = 0, 1, 2, ... (strides 1, 2, 4, ...).
template <class L, int NMIX>
__device__ __forceinline__ void fwht(float2 (&V)[L::NV], int l, float kappa)
{
    if (NMIX >= 2) stage_reg<L, 0>(V);
    if (NMIX >= 4) stage_reg<L, 1>(V);
    if (NMIX >= 8) stage_reg<L, 2>(V);
    if (NMIX >= 16) stage_lane<L>(V, l, 1);
    if (NMIX >= 32) stage_lane<L>(V, l, 2);
    if (NMIX >= 64) stage_reg<L, 3>(V);
    if (NMIX >= 128) stage_reg<L, 4>(V);
    if (NMIX >= 2) {
        const float2 k2 = make_float2(kappa, kappa);
#pragma unroll
        for (int p = 0; p < L::NV; ++p) V[p] = __fmul2_rn(V[p], k2);
    }
}

// Store the row as bf16 (round to nearest even) to global memory, marked evict-first in
// L2 (streaming: Q~ is not read again by this path, the key and query rows that the next
// launch reads are worth keeping there instead).
template <class L>
__device__ __forceinline__ void store_row_bf16(const float2 (&V)[L::NV], uint8_t *row, int l)
{
#pragma unroll
    for (int j = 0; j < L::NJ; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const __nv_bfloat162 b =
                __floats2bfloat162_rn(get_el<L>(V, j * 8 + 2 * h), get_el<L>(V, j * 8 + 2 * h + 1));
            w[h] = *reinterpret_cast<const uint32_t *>(&b);
        }
        __stcs(reinterpret_cast<uint4 *>(row + j * 64 + l * 16), make_uint4(w[0], w[1], w[2], w[3]));
    }
}

template <class L>
__device__ __forceinline__ void store_row_f32(const float2 (&V)[L::NV], float *row, int l)
{
#pragma unroll
    for (int j = 0; j < L::NJ; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float4 *>(row + j * 32 + l * 8 + h * 4) =
                make_float4(get_el<L>(V, j * 8 + 4 * h + 0), get_el<L>(V, j * 8 + 4 * h + 1),
                            get_el<L>(V, j * 8 + 4 * h + 2), get_el<L>(V, j * 8 + 4 * h + 3));
}

// Group geometry of the quantiser: groups of G contiguous channels, G in {32, 64, 128}.
template <class L, int G>
struct Groups {
    static_assert(G == 32 || G == 64 || G == 128, "group must be 32, 64 or 128");
    static constexpr int DHv = L::NCH * 4;
    static_assert(DHv % G == 0, "group must divide d_h");
    static constexpr int NG = DHv / G;      // groups per row (1, 2 or 4)
    static constexpr int CPG = G / 32;      // lane chunks per group
    __host__ __device__ static constexpr int of_chunk(int j) { return j / CPG; }
};

// Per-group max|x| over the quad, NaN-propagating; amax[g] >= 0 (or NaN).
template <class L, int G>
__device__ __forceinline__ void group_amax(const float2 (&V)[L::NV], float (&amax)[Groups<L, G>::NG])
{
    using GR = Groups<L, G>;
    float acc[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) acc[g] = 0.0f;
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        acc[g] = max_abs_nan(acc[g], V[p].x);
        acc[g] = max_abs_nan(acc[g], V[p].y);
    }
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        acc[g] = max_abs_nan(acc[g], __shfl_xor_sync(FULL_MASK, acc[g], 1));
        acc[g] = max_abs_nan(acc[g], __shfl_xor_sync(FULL_MASK, acc[g], 2));
        amax[g] = fabsf(acc[g]);
    }
}

// Quantise a transformed K row: codes packed into one 32-bit word per chunk
// (byte j = code[2j] & 0xF | code[2j+1] << 4), and this lane's group step.
// Lane slot l computes the divisions of group (l % NG) and shares r with the quad;
// lanes l < NG own the stored scale of group l (returned in s_mine / has_scale).
template <class L, int G>
__device__ __forceinline__ void quantize_row(const float2 (&V)[L::NV], int l, int lane,
                                             uint32_t (&words)[L::NJ], float &s_mine, int &flags,
                                             float (&r)[Groups<L, G>::NG])
{
    using GR = Groups<L, G>;
    float amax[GR::NG];
    group_amax<L, G>(V, amax);
    const int gm = l & (GR::NG - 1);
    float am = amax[0];
#pragma unroll
    for (int g = 1; g < GR::NG; ++g)
        if (gm == g) am = amax[g];
    const bool finite = am <= 3.402823466e38f;  // false for NaN and Inf
    if (!finite) flags |= ST_NONFINITE;
    const bool zero = !(am >= 0x1p-125f);
    const float r_m = zero ? 0.0f : __fdiv_rn(7.0f, am);
    s_mine = zero ? 0.0f : __fdiv_rn(am, 7.0f);
    if (GR::NG == 1) {
        r[0] = r_m;
    } else {
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) r[g] = __shfl_sync(FULL_MASK, r_m, (lane & ~3) | g);
    }
    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    uint32_t m[L::NV][2];
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        // fma(x, r, 1.5 * 2^23): one rounding of the exact product to an integer, ties to even
        const float2 t = __ffma2_rn(V[p], make_float2(r[g], r[g]), magic);
        m[p][0] = __float_as_uint(t.x);   // low 4 bits = code mod 16
        m[p][1] = __float_as_uint(t.y);
    }
#pragma unroll
    for (int j = 0; j < L::NJ; ++j) {
        uint32_t b[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = j * 8 + e;
            b[e] = m[L::vidx(i)][L::comp(i)];
        }
        // gather byte 0 of the even / odd elements, then interleave nibbles
        const uint32_t e01 = __byte_perm(b[0], b[2], 0x0040);
        const uint32_t e23 = __byte_perm(b[4], b[6], 0x0040);
        const uint32_t ev = __byte_perm(e01, e23, 0x5410);
        const uint32_t o01 = __byte_perm(b[1], b[3], 0x0040);
        const uint32_t o23 = __byte_perm(b[5], b[7], 0x0040);
        const uint32_t od = __byte_perm(o01, o23, 0x5410);
        words[j] = (ev & 0x0f0f0f0fu) | ((od << 4) & 0xf0f0f0f0u);
    }
}

// Three-input maximum / minimum of fp32 values with NaN propagation (sm_100).
__device__ __forceinline__ float max3_nan(float a, float b, float c)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float min3_nan(float a, float b, float c)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float max_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float min_nan(float a, float b)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// ---- measurement statistics of quantised rows ----------------------------------------

// Per-lane accumulators of the measurement statistics (summed over lanes and CTAs later):
// sum (x~ - K^)^2, sum x~^2, and per group (counted by quad lane 0) max|x~|, max - min,
// the largest max|x~| and the number of groups.
struct RowStats {
    double err2 = 0.0, ref2 = 0.0, s_amax = 0.0, s_range = 0.0, mx_amax = 0.0, n_groups = 0.0;
};

// Adds one quantised row held by a quad to st.  code_of(p) gives the codes of V[p] as
// floats; shat[g] is group g's stored (fp16) scale as fp32.  Squared error and reference
// are fp32 sums per lane and group of terms normalised by the group's scale, then weighted
// by its square in fp64:
//   d = fma(-s, c, x)  (s * c is exact: an fp16 value times a 4-bit code; the difference is
//                       rounded once),  t = d * (1/s),  v = x * (1/s),  E += t*t,  R += v*v,
//   err2 += s^2 * E,  ref2 += s^2 * R.
// All terms are >= 0, so each sum's relative error stays below 2^-24 times (terms per lane
// + 8).  A scale of 0 (a zero group) or a non-finite one normalises by 1.  Every lane of the
// quad must call it (the group max/min use quad shuffles); rows past the end pass
// valid = false and add nothing.
template <class L, int G, class CodeOf>
__device__ __forceinline__ void row_stats(const float2 (&V)[L::NV], CodeOf code_of,
                                          const float (&shat)[Groups<L, G>::NG], int l,
                                          bool valid, RowStats &st)
{
    using GR = Groups<L, G>;
    float gmax[GR::NG], gmin[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        gmax[g] = -INFINITY;
        gmin[g] = INFINITY;
    }
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        gmax[g] = fmaxf(gmax[g], fmaxf(V[p].x, V[p].y));
        gmin[g] = fminf(gmin[g], fminf(V[p].x, V[p].y));
    }
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        gmax[g] = fmaxf(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 1));
        gmax[g] = fmaxf(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 2));
        gmin[g] = fminf(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 1));
        gmin[g] = fminf(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 2));
    }
    if (!valid) return;
    float2 nsc2[GR::NG], rn2[GR::NG], E2[GR::NG], R2[GR::NG];
    float wg[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        const bool ok = shat[g] > 0.0f && shat[g] < INFINITY;
        const float norm = ok ? shat[g] : 1.0f;
        const float rn = ok ? __frcp_rn(norm) : 1.0f;
        nsc2[g] = make_float2(-shat[g], -shat[g]);
        rn2[g] = make_float2(rn, rn);
        wg[g] = norm * norm;  // exact: an fp16 value squared
        E2[g] = make_float2(0.0f, 0.0f);
        R2[g] = make_float2(0.0f, 0.0f);
    }
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        const float2 x = V[p];
        const float2 t = __fmul2_rn(__ffma2_rn(nsc2[g], code_of(p), x), rn2[g]);
        const float2 v = __fmul2_rn(x, rn2[g]);
        E2[g] = __ffma2_rn(t, t, E2[g]);
        R2[g] = __ffma2_rn(v, v, R2[g]);
    }
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        st.err2 += static_cast<double>((E2[g].x + E2[g].y) * wg[g]);
        st.ref2 += static_cast<double>((R2[g].x + R2[g].y) * wg[g]);
    }
    if (l == 0) {
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) {
            const float amax = fmaxf(gmax[g], -gmin[g]);
            st.s_amax += amax;
            st.s_range += static_cast<double>(gmax[g]) - static_cast<double>(gmin[g]);
            st.mx_amax = fmax(st.mx_amax, static_cast<double>(amax));
            st.n_groups += 1.0;
        }
    }
}

// quantize_row and row_stats of the same row in one pass (the transform with fused
// statistics): the group maximum and minimum (three-input, NaN-propagating) give both the
// quantiser's amax = max(max, -min) — the same value as the |x| maximum, NaN included — and
// the group range; the quantiser's fma(x, r, 1.5 * 2^23) gives both the packed code bits and
// the code c for the statistics' terms.  The statistics' arithmetic is row_stats' (terms
// (x - s c)/s and x/s of the stored fp16 scale s, fp32 per lane and group, then s^2 in fp64),
// term for term in the same order, so the sums are those of row_stats bit for bit.
// Outputs as quantize_row, plus the lane's fp16 scale bits; adds the row to st when valid.
template <class L, int G>
__device__ __forceinline__ void quantize_row_stats(const float2 (&V)[L::NV], int l, int lane,
                                                   bool valid, uint32_t (&words)[L::NJ],
                                                   uint16_t &hb_mine, int &flags, RowStats &st)
{
    using GR = Groups<L, G>;
    float gmax[GR::NG], gmin[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        gmax[g] = -INFINITY;
        gmin[g] = INFINITY;
    }
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        gmax[g] = max3_nan(gmax[g], V[p].x, V[p].y);
        gmin[g] = min3_nan(gmin[g], V[p].x, V[p].y);
    }
    float amax[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        gmax[g] = max_nan(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 1));
        gmax[g] = max_nan(gmax[g], __shfl_xor_sync(FULL_MASK, gmax[g], 2));
        gmin[g] = min_nan(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 1));
        gmin[g] = min_nan(gmin[g], __shfl_xor_sync(FULL_MASK, gmin[g], 2));
        amax[g] = max_nan(gmax[g], -gmin[g]);
    }
    // the quantiser's step of this lane's group (lane slot l computes group l % NG)
    const int gm = l & (GR::NG - 1);
    float am = amax[0];
#pragma unroll
    for (int g = 1; g < GR::NG; ++g)
        if (gm == g) am = amax[g];
    const bool finite = am <= 3.402823466e38f;  // false for NaN and Inf
    if (!finite) flags |= ST_NONFINITE;
    const bool zero = !(am >= 0x1p-125f);
    const float r_m = zero ? 0.0f : __fdiv_rn(7.0f, am);
    const float s_m = zero ? 0.0f : __fdiv_rn(am, 7.0f);
    hb_mine = __half_as_ushort(__float2half_rn(s_m));
    const float shat_m = __half2float(__ushort_as_half(hb_mine));
    float r[GR::NG], shat[GR::NG];
    if (GR::NG == 1) {
        r[0] = r_m;
        shat[0] = shat_m;
    } else {
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) {
            r[g] = __shfl_sync(FULL_MASK, r_m, (lane & ~3) | g);
            shat[g] = __shfl_sync(FULL_MASK, shat_m, (lane & ~3) | g);
        }
    }
    float2 nsc2[GR::NG], rn2[GR::NG], E2[GR::NG], R2[GR::NG];
    float wg[GR::NG];
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        const bool ok = shat[g] > 0.0f && shat[g] < INFINITY;
        const float norm = ok ? shat[g] : 1.0f;
        const float rn = ok ? __frcp_rn(norm) : 1.0f;
        nsc2[g] = make_float2(-shat[g], -shat[g]);
        rn2[g] = make_float2(rn, rn);
        wg[g] = norm * norm;  // exact: an fp16 value squared
        E2[g] = make_float2(0.0f, 0.0f);
        R2[g] = make_float2(0.0f, 0.0f);
    }
    const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    const float2 nmagic = make_float2(-12582912.0f, -12582912.0f);
    uint32_t m[L::NV][2];
#pragma unroll
    for (int p = 0; p < L::NV; ++p) {
        const int g = GR::of_chunk(L::elem(p, 0) >> 3);
        const float2 x = V[p];
        // one rounding of the exact product x * r to an integer, ties to even
        const float2 t = __ffma2_rn(x, make_float2(r[g], r[g]), magic);
        m[p][0] = __float_as_uint(t.x);  // low 4 bits = code mod 16
        m[p][1] = __float_as_uint(t.y);
        const float2 c = __fadd2_rn(t, nmagic);  // the code, exactly
        const float2 d = __fmul2_rn(__ffma2_rn(nsc2[g], c, x), rn2[g]);
        const float2 v = __fmul2_rn(x, rn2[g]);
        E2[g] = __ffma2_rn(d, d, E2[g]);
        R2[g] = __ffma2_rn(v, v, R2[g]);
    }
#pragma unroll
    for (int j = 0; j < L::NJ; ++j) {
        uint32_t b[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = j * 8 + e;
            b[e] = m[L::vidx(i)][L::comp(i)];
        }
        const uint32_t e01 = __byte_perm(b[0], b[2], 0x0040);
        const uint32_t e23 = __byte_perm(b[4], b[6], 0x0040);
        const uint32_t ev = __byte_perm(e01, e23, 0x5410);
        const uint32_t o01 = __byte_perm(b[1], b[3], 0x0040);
        const uint32_t o23 = __byte_perm(b[5], b[7], 0x0040);
        const uint32_t od = __byte_perm(o01, o23, 0x5410);
        words[j] = (ev & 0x0f0f0f0fu) | ((od << 4) & 0xf0f0f0f0u);
    }
    if (!valid) return;
#pragma unroll
    for (int g = 0; g < GR::NG; ++g) {
        st.err2 += static_cast<double>((E2[g].x + E2[g].y) * wg[g]);
        st.ref2 += static_cast<double>((R2[g].x + R2[g].y) * wg[g]);
    }
    if (l == 0) {
#pragma unroll
        for (int g = 0; g < GR::NG; ++g) {
            st.s_amax += amax[g];
            st.s_range += static_cast<double>(gmax[g]) - static_cast<double>(gmin[g]);
            st.mx_amax = fmax(st.mx_amax, static_cast<double>(amax[g]));
            st.n_groups += 1.0;
        }
    }
}

// Reduce the lanes' statistics of a CTA in a fixed order (xor tree over the warp, then the
// warps in order through red[warps][6]) and write the CTA's partial [6]; NaN / Inf in the
// sums set ST_NONFINITE.  Called by every thread of the CTA.
__device__ __forceinline__ void reduce_row_stats(RowStats st, double *red, int nwarps,
                                                 double *partial, int &flags)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!isfinite(st.err2) || !isfinite(st.ref2) || !isfinite(st.s_amax)) flags |= ST_NONFINITE;
    double v[6] = {st.err2, st.ref2, st.s_amax, st.s_range, st.mx_amax, st.n_groups};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int f = 0; f < 6; ++f) {
            const double other = __shfl_xor_sync(FULL_MASK, v[f], o);
            v[f] = f == 4 ? fmax(v[f], other) : v[f] + other;
        }
    if (lane == 0)
#pragma unroll
        for (int f = 0; f < 6; ++f) red[warp * 6 + f] = v[f];
    __syncthreads();
    if (threadIdx.x < 6) {
        const int f = threadIdx.x;
        double acc = red[f];
        for (int w = 1; w < nwarps; ++w) acc = f == 4 ? fmax(acc, red[w * 6 + f]) : acc + red[w * 6 + f];
        partial[f] = acc;
    }
}

}  // namespace qkq

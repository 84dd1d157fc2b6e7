// KV4 consumer on the tensor cores with register operands: attention logits of transformed
// queries against the int4 key cache, for decode-sized query blocks.
//
// The logits are S[tq][h][tk] = sum_g scale[tk][h_kv][g] * sum_{c in g} Q~[tq][h][c] * code[tk][h_kv][c]
// (the online rotation cancels in Q~ K~^T: "LLM旋转量化笔记" §3.2.1).  For one key head and a
// block of at most 64 query rows m = (query token, query head of the key head) the inner sums
// are a contraction over the channels of a group with a small N, so each warp runs it as
// warp-level bf16 MMAs (m16n8k16, fp32 accumulate) whose A fragments are the cached tokens'
// codes unpacked straight into registers: the key cache never sits in shared memory as bf16
// operands (at most its packed codes pass through a copy ring, below).  The codes (-7 .. 7) and the
// bf16 queries are exact bf16 operands and every product is exact; the tensor cores add a
// group's products in fp32 in an order of their own, so a score is within
// 2 (d_h + d_h/group + 2) 2^-24 sum_c |q_c| |scale code_c| of the exact value, the bound of the
// other tensor-core entry.
//
// Channel placement.  The dot product does not care which channel sits at which K index of
// an MMA, as long as A and B agree.  A word of codes holds channels 8w .. 8w + 7 (nibble e =
// channel 8w + e); one mask-and-xor per pair turns nibbles (e, e + 4) into the bf16 pair
// (128 + code + 8) in each half, and one packed bf16 subtraction of 136 leaves the codes.
// A lane of quad position t supplies K indices 2t, 2t + 1 and 2t + 8, 2t + 9 of every K-step;
// it takes, within each scale group, the group's words t * G/32 .. t * G/32 + G/32 - 1, so every
// K-step lies inside one group and each group has its own accumulator; the query fragments
// in shared memory are laid out with the same placement.  The epilogue adds the groups in
// order, S = fma(scale_g, D_g, S), as the CUDA-core kernel does, and stores each logit once
// (a quad of lanes covers 8 consecutive cached tokens of one query row: full 32-byte
// sectors).
//
// Work: one CTA of 8 warps per (run of 16-token tiles, key head, query block); a warp takes
// its tiles in turn.  With one n-tile (one or two decode tokens at 4 query heads a key head)
// or group 32 it loads the next tile's codes and scales into registers while it scores the
// current one, and a group's K-steps alternate between two accumulators (two independent MMA
// chains, added before the scale).  With more n-tiles at group 64 or 128 each warp keeps a
// ring of tiles' packed codes in shared memory, copied ahead by cp.async; each lane reads back
// only the bytes it copied, so the only wait is on its own copy groups (cp.async.wait_group:
// no spin, no barrier).  From four n-tiles at group = d_h a warp scores two tiles per turn, so
// that each query-fragment load from shared memory (the L1 data path was 90 % busy at 16 query
// tokens) feeds the MMAs of both.  Measured over a 131072-token 8B cache
// (group 128): more resident warps (four CTAs per SM) beat a deeper register prefetch at
// fewer warps for one token, the ring wins for 4 and 16 tokens, and the integer ALU pipe, not
// the tensor pipe, is the busiest (the unpacking), hence the 32-bit indices below.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace qkq {

namespace {

constexpr int ASM_WARPS = 8;
constexpr int ASM_ROWS = 64;  // query rows per CTA at most: 8 MMA n-tiles of 8

// The 8 codes of a word as four bf16 pairs x[e] = (code of channel 8w + e, of 8w + e + 4),
// exact: ((w >> 4e) & 0x000F000F) ^ 0x43084308 is the bf16 pair of 128 + (nibble ^ 8) =
// 136 + code (128 has an ulp of 1 in bf16), and 136 is subtracted in bf16.
__device__ __forceinline__ void unpack_codes(uint32_t w, uint32_t (&x)[4])
{
    const __nv_bfloat162 bias = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t y = ((w >> (4 * e)) & 0x000F000Fu) ^ 0x43084308u;
        const __nv_bfloat162 v = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&y), bias);
        x[e] = *reinterpret_cast<const uint32_t *>(&v);
    }
}

// D += A B for one m16n8k16 tile, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B (a group's first K-step: no accumulator to read).
__device__ __forceinline__ void mma_16816_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// One 16-token tile's codes and scales for this lane: rows gq and gq + 8 of the tile.
template <int DH, int G>
struct TileRegs {
    static constexpr int NG = DH / G;
    static constexpr int LW = G / 32;  // words of a group per lane
    uint32_t w[2][NG * LW];
    float s[2][NG];
};

// Row indices tk * Hkv + hk are 32-bit (the entry point requires Tk * Hkv < 2^32) and the
// addresses are formed with one wide multiply-add each, on the FMA pipe: the integer ALU pipe
// is the one the code unpacking keeps busy.
template <int DH, int G>
__device__ __forceinline__ void load_tile(TileRegs<DH, G> &R, const ScoresParams &p, uint32_t hk,
                                          uint32_t tile, int gq, int t)
{
    constexpr int NG = DH / G, LW = G / 32, WPG = G / 8;
    const uint32_t tmax = static_cast<uint32_t>(p.Tk) - 1u;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        uint32_t tk = tile * 16u + static_cast<uint32_t>(gq + 8 * r);
        tk = tk < tmax ? tk : tmax;  // ragged tail: a real row, its logits not stored
        const uint32_t row = tk * static_cast<uint32_t>(p.Hkv) + hk;
        const uint32_t *cw = reinterpret_cast<const uint32_t *>(p.k_codes) + static_cast<size_t>(row) * (DH / 8);
        const uint16_t *sw = p.k_scales + static_cast<size_t>(row) * NG;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint32_t *src = cw + g * WPG + t * LW;
            if (LW == 4) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src));
                R.w[r][g * 4] = v.x;
                R.w[r][g * 4 + 1] = v.y;
                R.w[r][g * 4 + 2] = v.z;
                R.w[r][g * 4 + 3] = v.w;
            } else if (LW == 2) {
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
                R.w[r][g * 2] = v.x;
                R.w[r][g * 2 + 1] = v.y;
            } else {
                R.w[r][g] = __ldg(src);
            }
            R.s[r][g] = __half2float(__ushort_as_half(__ldg(sw + g)));
        }
    }
}

// Asynchronous global -> shared copies (cp.async) of this lane's codes of a tile: the lane
// reads back only what it copied itself, so a wait on its own copy groups is all the
// ordering needed (no barrier, no spin).
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void *src)
{
    if (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(BYTES) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stage layout (one tile of a warp): [row r of the lane's pair][word i][lane], words of
// DH / 32 per lane and row, lane-contiguous (conflict-free 4-byte reads).
template <int DH>
__host__ __device__ constexpr int stage_words() { return 2 * (DH / 32) * 32; }

// Copy this lane's codes of `tile` into a stage and load its scales into registers.
template <int DH, int G>
__device__ __forceinline__ void issue_tile(uint32_t stage, float (&sc)[2][DH / G],
                                           const ScoresParams &p, uint32_t hk, uint32_t tile,
                                           int gq, int t, int lane)
{
    constexpr int NG = DH / G, LW = G / 32, WPG = G / 8, NW = DH / 32;
    const uint32_t tmax = static_cast<uint32_t>(p.Tk) - 1u;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        uint32_t tk = tile * 16u + static_cast<uint32_t>(gq + 8 * r);
        tk = tk < tmax ? tk : tmax;  // ragged tail: a real row, its logits not stored
        const uint32_t row = tk * static_cast<uint32_t>(p.Hkv) + hk;
        const uint32_t *cw = reinterpret_cast<const uint32_t *>(p.k_codes) + static_cast<size_t>(row) * (DH / 8);
        const uint16_t *sw = p.k_scales + static_cast<size_t>(row) * NG;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            // words g * LW .. g * LW + LW - 1 of the lane's row r: LW words at word index
            // (r * NW + g * LW) * 32 + lane * LW ... kept lane-contiguous per copy
            cp_async<4 * LW>(stage + 4u * ((r * NW + g * LW) * 32 + lane * LW), cw + g * WPG + t * LW);
            sc[r][g] = __half2float(__ushort_as_half(__ldg(sw + g)));
        }
    }
}

template <int DH, int G>
__device__ __forceinline__ void read_tile(TileRegs<DH, G> &R, const uint32_t *stage,
                                          const float (&sc)[2][DH / G], int lane)
{
    constexpr int NG = DH / G, LW = G / 32, NW = DH / 32;
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint32_t *src = stage + (r * NW + g * LW) * 32 + lane * LW;
            if (LW == 4) {
                const uint4 v = *reinterpret_cast<const uint4 *>(src);
                R.w[r][g * 4] = v.x;
                R.w[r][g * 4 + 1] = v.y;
                R.w[r][g * 4 + 2] = v.z;
                R.w[r][g * 4 + 3] = v.w;
            } else if (LW == 2) {
                const uint2 v = *reinterpret_cast<const uint2 *>(src);
                R.w[r][g * 2] = v.x;
                R.w[r][g * 2 + 1] = v.y;
            } else {
                R.w[r][g] = *src;
            }
            R.s[r][g] = sc[r][g];
        }
}

// The query fragments of n-tile pair / single n-tile `pass` at K-step s: lane-contiguous,
// 2 NC words a lane (one 8- or 16-byte shared load).
template <int NC>
__device__ __forceinline__ void load_b(const uint32_t *bfrag, int pass, int s, int KS, int lane,
                                       uint32_t (&b)[NC][2])
{
    const uint32_t *src = bfrag + ((pass * KS + s) * 32 + lane) * (2 * NC);
    if (NC == 2) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src);
        b[0][0] = v.x;
        b[0][1] = v.y;
        b[NC - 1][0] = v.z;
        b[NC - 1][1] = v.w;
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(src);
        b[0][0] = v.x;
        b[0][1] = v.y;
    }
}

// The logits of one 16-token tile for this block's query rows, NC n-tiles per pass: per scale
// group an accumulator of the group's K-steps, the scales applied in group order, the pass's
// logits stored.  With one pass the codes are unpacked word by word as the K-steps need them;
// with several, once for the tile into the A fragments of every K-step (d_h / 4 registers).
template <int DH, int G, int NT>
__device__ __forceinline__ void score_tile(const TileRegs<DH, G> &R, const ScoresParams &p,
                                           const uint32_t *bfrag, const int64_t *rowoff,
                                           uint32_t tile, int lane)
{
    constexpr int KS = DH / 16, NG = DH / G, LW = G / 32, KSG = G / 16;
    constexpr int NC = NT < 2 ? NT : 2;  // n-tiles per pass
    constexpr bool ONE_PASS = NT == NC;
    const int gq = lane >> 2, t = lane & 3;
    // A fragments: K-step s = g * KSG + 2 i + h of group g takes word i of the lane's part of
    // the group, pairs 2h (K indices 2t, 2t + 1) and 2h + 1 (2t + 8, 2t + 9)
    uint32_t a[ONE_PASS ? 1 : KS][4];
    if (!ONE_PASS) {
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int i = 0; i < LW; ++i) {
                uint32_t x0[4], x1[4];  // rows gq and gq + 8
                unpack_codes(R.w[0][g * LW + i], x0);
                unpack_codes(R.w[1][g * LW + i], x1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = g * KSG + 2 * i + h;
                    a[ONE_PASS ? 0 : s][0] = x0[2 * h];
                    a[ONE_PASS ? 0 : s][1] = x1[2 * h];
                    a[ONE_PASS ? 0 : s][2] = x0[2 * h + 1];
                    a[ONE_PASS ? 0 : s][3] = x1[2 * h + 1];
                }
            }
    }
#pragma unroll 1  // a real loop: unrolled, the compiler keeps every pass's fragments live
    for (int pass = 0; pass < NT / NC; ++pass) {
        float S[NC][4];
#pragma unroll
        for (int n = 0; n < NC; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) S[n][e] = 0.0f;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            // with one n-tile, even and odd K-steps go to two accumulators (two independent
            // MMA chains), added before the scale
            float D[NC][4], E[NC][4];
#pragma unroll
            for (int i = 0; i < LW; ++i) {
                uint32_t x0[4], x1[4];
                if (ONE_PASS) {
                    unpack_codes(R.w[0][g * LW + i], x0);
                    unpack_codes(R.w[1][g * LW + i], x1);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = g * KSG + 2 * i + h;
                    uint32_t b[NC][2];
                    load_b<NC>(bfrag, pass, s, KS, lane, b);
                    const uint32_t a0 = ONE_PASS ? x0[2 * h] : a[ONE_PASS ? 0 : s][0];
                    const uint32_t a1 = ONE_PASS ? x1[2 * h] : a[ONE_PASS ? 0 : s][1];
                    const uint32_t a2 = ONE_PASS ? x0[2 * h + 1] : a[ONE_PASS ? 0 : s][2];
                    const uint32_t a3 = ONE_PASS ? x1[2 * h + 1] : a[ONE_PASS ? 0 : s][3];
#pragma unroll
                    for (int n = 0; n < NC; ++n) {
                        float(&acc)[4] = (NC == 1 && h == 1) ? E[n] : D[n];
                        if (i == 0 && (h == 0 || NC == 1))
                            mma_16816_first(acc, a0, a1, a2, a3, b[n][0], b[n][1]);
                        else
                            mma_16816(acc, a0, a1, a2, a3, b[n][0], b[n][1]);
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < NC; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float d = NC == 1 ? __fadd_rn(D[n][e], E[n][e]) : D[n][e];
                    S[n][e] = __fmaf_rn(R.s[e >> 1][g], d, S[n][e]);
                }
        }
        // this lane's query rows of the pass: (n, c) -> logits offset, [pass][t][n][c]
        int64_t off[NC][2];
        const int64_t *ro = rowoff + (pass * 4 + t) * (2 * NC);
        if (NC == 2) {
            const longlong2 u = *reinterpret_cast<const longlong2 *>(ro);
            const longlong2 v = *reinterpret_cast<const longlong2 *>(ro + 2);
            off[0][0] = u.x;
            off[0][1] = u.y;
            off[NC - 1][0] = v.x;
            off[NC - 1][1] = v.y;
        } else {
            const longlong2 u = *reinterpret_cast<const longlong2 *>(ro);
            off[0][0] = u.x;
            off[0][1] = u.y;
        }
        const uint32_t tk0 = tile * 16u + static_cast<uint32_t>(gq);
        const uint32_t Tk = static_cast<uint32_t>(p.Tk);
#pragma unroll
        for (int n = 0; n < NC; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (off[n][c] < 0) continue;
                float *dst = p.scores + off[n][c];
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    if (tk0 + 8u * r < Tk) __stcs(dst + (tk0 + 8u * r), S[n][2 * r + c]);
            }
    }
}

// The logits of MT consecutive 16-token tiles (the staged kernels, n-tiles taken two at a
// time): the tiles' codes unpacked into their A fragments first, then every query-fragment
// load from shared memory feeds the MMAs of all MT tiles (the shared-memory reads of the
// fragments, the busiest path at 16 query tokens, fall by MT).
template <int DH, int G, int NT, int MT>
__device__ __forceinline__ void score_tiles(const TileRegs<DH, G> (&R)[MT], const ScoresParams &p,
                                            const uint32_t *bfrag, const int64_t *rowoff,
                                            uint32_t tile0, int lane)
{
    constexpr int KS = DH / 16, NG = DH / G, LW = G / 32, KSG = G / 16;
    constexpr int NC = 2;
    static_assert(NT % NC == 0, "the staged kernels take n-tiles in pairs");
    const int gq = lane >> 2, t = lane & 3;
    uint32_t a[MT][KS][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int i = 0; i < LW; ++i) {
                uint32_t x0[4], x1[4];
                unpack_codes(R[m].w[0][g * LW + i], x0);
                unpack_codes(R[m].w[1][g * LW + i], x1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = g * KSG + 2 * i + h;
                    a[m][s][0] = x0[2 * h];
                    a[m][s][1] = x1[2 * h];
                    a[m][s][2] = x0[2 * h + 1];
                    a[m][s][3] = x1[2 * h + 1];
                }
            }
    const uint32_t Tk = static_cast<uint32_t>(p.Tk);
#pragma unroll 1  // a real loop: unrolled, the compiler keeps every pass's fragments live
    for (int pass = 0; pass < NT / NC; ++pass) {
        float S[MT][NC][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int n = 0; n < NC; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) S[m][n][e] = 0.0f;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            float D[MT][NC][4];
#pragma unroll
            for (int s = g * KSG; s < (g + 1) * KSG; ++s) {
                uint32_t b[NC][2];
                load_b<NC>(bfrag, pass, s, KS, lane, b);
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int n = 0; n < NC; ++n) {
                        if (s == g * KSG)
                            mma_16816_first(D[m][n], a[m][s][0], a[m][s][1], a[m][s][2], a[m][s][3],
                                            b[n][0], b[n][1]);
                        else
                            mma_16816(D[m][n], a[m][s][0], a[m][s][1], a[m][s][2], a[m][s][3],
                                      b[n][0], b[n][1]);
                    }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int n = 0; n < NC; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        S[m][n][e] = __fmaf_rn(R[m].s[e >> 1][g], D[m][n][e], S[m][n][e]);
        }
        int64_t off[NC][2];
        const int64_t *ro = rowoff + (pass * 4 + t) * (2 * NC);
        const longlong2 u = *reinterpret_cast<const longlong2 *>(ro);
        const longlong2 v = *reinterpret_cast<const longlong2 *>(ro + 2);
        off[0][0] = u.x;
        off[0][1] = u.y;
        off[1][0] = v.x;
        off[1][1] = v.y;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint32_t tk0 = (tile0 + m) * 16u + static_cast<uint32_t>(gq);
#pragma unroll
            for (int n = 0; n < NC; ++n)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (off[n][c] < 0) continue;
                    float *dst = p.scores + off[n][c];
#pragma unroll
                    for (int r = 0; r < 2; ++r)
                        if (tk0 + 8u * r < Tk) __stcs(dst + (tk0 + 8u * r), S[m][n][2 * r + c]);
                }
        }
    }
}

// Where a warp keeps the tiles in flight: in shared memory (a ring of cp.async stages, three
// tiles ahead) when several n-tiles make each tile's compute long, in registers (the next
// tile) for one n-tile or group 32, where the register ring measured faster (one decode token
// over a 131072-token 8B cache: 24.3 vs 25.2 us at group 128, 33.5 vs 40.8 us at group 32;
// four tokens 36.5 vs 30.6 us, sixteen 92.4 vs 89.3 us at group 128).
__host__ __device__ constexpr bool asm_staged(int nt, int g) { return nt > 1 && g >= 64; }
// tiles a warp scores per turn: staged with four or more n-tiles and one scale group a row,
// two sharing each query-fragment load (16 query tokens over a 131072-token 8B cache:
// 75.5 vs 89.0 us; with two n-tiles 34.3 vs 30.4 us, and with two groups the second tile's
// accumulators spill)
__host__ __device__ constexpr int asm_unit(int nt, int dh, int g)
{
    return asm_staged(nt, g) && nt >= 4 && g == dh ? 2 : 1;
}
// tiles in the ring: staged, four units (one scored, three in flight) of one tile or three
// of two; else two tiles in registers
__host__ __device__ constexpr int asm_depth(int nt, int dh, int g)
{
    return !asm_staged(nt, g) ? 2 : asm_unit(nt, dh, g) == 2 ? 6 : 4;
}
// resident CTAs per SM the register budget is sized for
constexpr int asm_min_ctas(int nt, int dh, int g)
{
    return nt > 1 ? 2 : (g == dh || dh == 64) ? 4 : dh == 2 * g ? 3 : 2;
}
template <int DH>
__host__ __device__ constexpr int asm_stage_bytes(int nt, int g)
{
    return asm_staged(nt, g) ? ASM_WARPS * asm_depth(nt, DH, g) * stage_words<DH>() * 4 : 0;
}

template <int DH, int G, int NT>
__global__ void __launch_bounds__(ASM_WARPS * 32, asm_min_ctas(NT, DH, G)) k_attention_scores_mma(const ScoresParams p, int qb,
                                                                     uint32_t tiles_per_cta)
{
    constexpr int KS = DH / 16, KSG = G / 16, LW = G / 32, WPG = G / 8;
    constexpr int NC = NT < 2 ? NT : 2;
    // query fragments: [pass][K-step][lane][n-tile of the pass][2 registers]; logits row
    // offsets [pass][quad position t][n-tile of the pass][column 2t + c] (-1: padding)
    __shared__ __align__(16) uint32_t bfrag[NT * KS * 64];
    __shared__ __align__(16) int64_t rowoff[NT * 8];
    wait_prior_grid();  // the queries may be the previous kernel's output
    const uint32_t hk = blockIdx.y;
    const int qpk = p.Hq / p.Hkv;
    const int64_t tq0 = static_cast<int64_t>(blockIdx.z) * qb;
    const int nq = p.Tq - tq0 < qb ? static_cast<int>(p.Tq - tq0) : qb;
    const int rows = nq * qpk;
    for (int i = threadIdx.x; i < NT * KS * 64; i += ASM_WARPS * 32) {
        const int reg = i & 1, nn = (i >> 1) % NC, lane = (i / (2 * NC)) & 31;
        const int s = (i / (64 * NC)) % KS, pass = i / (64 * NC * KS);
        const int m = (pass * NC + nn) * 8 + (lane >> 2), t = lane & 3;
        const int g = s / KSG, u = s % KSG;
        // the A side's channels for K indices (2t, 2t + 1) [reg 0] or (2t + 8, 2t + 9) [reg 1]
        const int c = 8 * (g * WPG + t * LW + (u >> 1)) + 2 * (u & 1) + reg;
        uint32_t v = 0;
        if (m < rows) {
            const uint16_t *qr = p.q + ((tq0 + m / qpk) * p.Hq + hk * qpk + m % qpk) * DH;
            v = static_cast<uint32_t>(qr[c]) | (static_cast<uint32_t>(qr[c + 4]) << 16);
        }
        bfrag[i] = v;
    }
    for (int i = threadIdx.x; i < NT * 8; i += ASM_WARPS * 32) {
        const int c = i & 1, nn = (i >> 1) % NC, t = (i / (2 * NC)) & 3, pass = i / (8 * NC);
        const int m = (pass * NC + nn) * 8 + 2 * t + c;
        rowoff[i] = m < rows ? ((tq0 + m / qpk) * p.Hq + hk * qpk + m % qpk) * p.Tk : -1;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;
    const uint32_t n_tiles = static_cast<uint32_t>((p.Tk + 15) / 16);
    const uint32_t first = blockIdx.x * tiles_per_cta;
    const uint32_t end = first + tiles_per_cta < n_tiles ? first + tiles_per_cta : n_tiles;
    constexpr int DEPTH = asm_depth(NT, DH, G);
    if constexpr (asm_staged(NT, G)) {
        // a ring of DEPTH tile stages per warp, taken MT at a time (a unit): unit k is copied
        // UD - 1 turns ahead, into the stages scored (and so freed) in the turn before; one
        // copy group per turn, empty or not
        constexpr int MT = asm_unit(NT, DH, G), UD = DEPTH / MT;
        extern __shared__ __align__(16) uint32_t stage_mem[];
        const uint32_t *my_stages = stage_mem + warp * DEPTH * stage_words<DH>();
        const uint32_t stage0 = static_cast<uint32_t>(__cvta_generic_to_shared(my_stages));
        float sc[DEPTH][2][DH / G];
        auto issue_unit = [&](int slot, uint32_t tl) {  // tiles tl .. tl + MT - 1 into unit slot
#pragma unroll
            for (int m = 0; m < MT; ++m)
                issue_tile<DH, G>(stage0 + 4u * (slot * MT + m) * stage_words<DH>(), sc[slot * MT + m],
                                  p, hk, tl + m, gq, t, lane);
        };
        constexpr uint32_t STEP = MT * ASM_WARPS;  // tiles between a warp's consecutive units
#pragma unroll
        for (int d = 0; d < UD - 1; ++d) {
            const uint32_t tl = first + MT * warp + d * STEP;
            if (tl < end) issue_unit(d, tl);
            cp_async_commit();
        }
        for (uint32_t base = first + MT * warp; base < end; base += UD * STEP) {
#pragma unroll
            for (int d = 0; d < UD; ++d) {
                const uint32_t tl = base + d * STEP;
                if (tl >= end) break;
                constexpr int ahead = UD - 1;
                const int nd = (d + ahead) % UD;
                const uint32_t nx = tl + ahead * STEP;
                if (nx < end) issue_unit(nd, nx);
                cp_async_commit();
                cp_async_wait<UD - 1>();  // this turn's unit has landed
                TileRegs<DH, G> R[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    read_tile<DH, G>(R[m], my_stages + (d * MT + m) * stage_words<DH>(), sc[d * MT + m], lane);
                score_tiles<DH, G, NT, MT>(R, p, bfrag, rowoff, tl, lane);
            }
        }
        cp_async_wait<0>();  // nothing in flight at exit
    } else {
        // a ring of DEPTH tiles in registers: a slot is refilled with the tile DEPTH turns
        // ahead as soon as it has been scored
        TileRegs<DH, G> R[DEPTH];
#pragma unroll
        for (int d = 0; d < DEPTH; ++d) {
            const uint32_t tl = first + warp + d * ASM_WARPS;
            if (tl < end) load_tile<DH, G>(R[d], p, hk, tl, gq, t);
        }
        for (uint32_t base = first + warp; base < end; base += DEPTH * ASM_WARPS) {
#pragma unroll
            for (int d = 0; d < DEPTH; ++d) {
                const uint32_t tl = base + d * ASM_WARPS;
                if (tl >= end) break;
                score_tile<DH, G, NT>(R[d], p, bfrag, rowoff, tl, lane);
                const uint32_t nx = tl + DEPTH * ASM_WARPS;
                if (nx < end) load_tile<DH, G>(R[d], p, hk, nx, gq, t);
            }
        }
    }
    // (no early trigger of the next launch: measured 15 % slower in back-to-back calls)
}

using ScoresMmaKernel = void (*)(ScoresParams, int, uint32_t);

template <int DH, int G>
ScoresMmaKernel pick_nt(int nt)
{
    switch (nt) {
    case 1: return k_attention_scores_mma<DH, G, 1>;
    case 2: return k_attention_scores_mma<DH, G, 2>;
    case 4: return k_attention_scores_mma<DH, G, 4>;
    case 8: return k_attention_scores_mma<DH, G, 8>;
    }
    return nullptr;
}

ScoresMmaKernel pick_mma(int d_h, int group, int nt)
{
    if (d_h == 64) {
        if (group == 32) return pick_nt<64, 32>(nt);
        if (group == 64) return pick_nt<64, 64>(nt);
    } else if (d_h == 128) {
        if (group == 32) return pick_nt<128, 32>(nt);
        if (group == 64) return pick_nt<128, 64>(nt);
        if (group == 128) return pick_nt<128, 128>(nt);
    }
    return nullptr;
}

// Resident CTAs per SM of a kernel with `smem` bytes of dynamic shared memory, from its
// registers (8-register granules), its shared memory (1 KB reserved per CTA) and 2048
// threads per SM; a staged kernel is set up once per (kernel, device) for that much dynamic
// shared memory and the largest shared-memory carveout.  (The occupancy calculator, asked
// the same with the default carveout, answered no resident CTA for the staged kernels.)
cudaError_t ctas_per_sm(ScoresMmaKernel kern, const DeviceInfo &dev, int smem, int *ctas)
{
    struct Entry {
        ScoresMmaKernel kern;
        int ordinal, regs, static_smem;
    };
    static std::mutex mu;
    static constexpr int kSlots = 64;
    static Entry cache[kSlots];
    static int used = 0;
    std::lock_guard<std::mutex> lock(mu);
    int regs = -1, static_smem = 0;
    for (int i = 0; i < used; ++i)
        if (cache[i].kern == kern && cache[i].ordinal == dev.ordinal) {
            regs = cache[i].regs;
            static_smem = cache[i].static_smem;
        }
    if (regs < 0) {
        cudaError_t e = cudaSuccess;
        if (smem > 0) {  // the staged kernels: room for the stages (the others keep their L1)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
        }
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        regs = fa.numRegs > 0 ? fa.numRegs : 1;
        static_smem = static_cast<int>(fa.sharedSizeBytes);
        if (used < kSlots) cache[used++] = {kern, dev.ordinal, regs, static_smem};
    }
    const int per_sm = dev.smem_per_sm > 0 ? dev.smem_per_sm : 228 * 1024;
    int n = 65536 / (ASM_WARPS * 32 * ((regs + 7) / 8 * 8));
    const int by_smem = per_sm / (static_smem + smem + 1024);
    n = n < by_smem ? n : by_smem;
    n = n < 2048 / (ASM_WARPS * 32) ? n : 2048 / (ASM_WARPS * 32);
    if (n < 1) return cudaErrorInvalidConfiguration;
    *ctas = n;
    return cudaSuccess;
}

}  // namespace

cudaError_t attention_scores_mma_launch(const ScoresParams &p, const DeviceInfo &dev, int d_h,
                                        int group, cudaStream_t stream)
{
    if (p.Tq <= 0 || p.Tk <= 0) return cudaSuccess;
    const int qpk = p.Hq / p.Hkv;
    const int qb = ASM_ROWS / qpk;  // query tokens per block: qpk <= 8, so at least 8
    const int64_t nq_first = p.Tq < qb ? p.Tq : qb;
    const int rows = static_cast<int>(nq_first) * qpk;
    const int nt = rows <= 8 ? 1 : rows <= 16 ? 2 : rows <= 32 ? 4 : 8;
    const ScoresMmaKernel kern = pick_mma(d_h, group, nt);
    if (kern == nullptr) return cudaErrorInvalidValue;
    const int smem = d_h == 64 ? asm_stage_bytes<64>(nt, group) : asm_stage_bytes<128>(nt, group);
    int per_sm = 0;
    const cudaError_t e = ctas_per_sm(kern, dev, smem, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t qblocks = (p.Tq + qb - 1) / qb;
    if (qblocks > 65535) return cudaErrorInvalidValue;
    // one wave of CTAs over (tile runs, key heads, query blocks), each warp at least one tile
    const int64_t n_tiles = (p.Tk + 15) / 16;
    const int64_t wave = static_cast<int64_t>(dev.num_sms) * per_sm;
    const int64_t runs_target = (wave + p.Hkv * qblocks - 1) / (p.Hkv * qblocks);
    int64_t per_cta = (n_tiles + runs_target - 1) / runs_target;
    const int unit = asm_unit(nt, d_h, group);
    per_cta = per_cta < ASM_WARPS * unit ? ASM_WARPS * unit : per_cta;
    per_cta = (per_cta + unit - 1) / unit * unit;  // units never straddle two CTAs
    const int64_t runs = (n_tiles + per_cta - 1) / per_cta;
    if (runs > 0x7fffffff || p.Tk * p.Hkv > 0xffffffffll) return cudaErrorInvalidValue;
    return launch_after_prior(kern, dim3(static_cast<unsigned>(runs), static_cast<unsigned>(p.Hkv),
                                         static_cast<unsigned>(qblocks)),
                              dim3(ASM_WARPS * 32), smem, stream, p, qb, static_cast<uint32_t>(per_cta));
}

}  // namespace qkq

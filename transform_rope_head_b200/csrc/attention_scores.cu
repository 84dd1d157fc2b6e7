// KV4 consumer: attention logits of transformed queries against the int4 key cache,
// read straight from the packed codes and fp16 scales.
//
// With Q~ = RoPE(Q) M and K~ = RoPE(K) M for an orthogonal mixing M, Q~ K~^T = RoPE(Q) RoPE(K)^T
// ("LLM旋转量化笔记" §3.2.1: the online rotation cancels in the score product), so the
// attention logits can be taken against the quantised K~ directly:
//   S[tq][h][tk] = sum_c Q~[tq][h][c] * scale[tk][h_kv][g(c)] * code[tk][h_kv][c],
// h_kv = h / (Hq / Hkv) (grouped-query heads share a key head).  No softmax scale is applied.
//
// One thread per (cache token, key head), or two cached tokens a block apart for a single
// query token (consecutive threads, consecutive tokens: coalesced score stores); a block
// holds, for up to four query tokens, the query heads of one key head in shared memory as
// fp32.  Codes become floats with one byte permutation
// each (2^23 + c + 8, then an exact subtraction) and serve all of those query rows; per
// group a row's products q * code (exact) are summed in fp32, even and odd channels in the
// two halves of packed fp32x2 multiply-adds, then scale * (even + odd) is added.  Bound
// against the exact sum: (d_h + groups + 2) * 2^-24 * sum |q| |scale * code|.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "kv4_codes.cuh"

namespace qkq {

namespace {

constexpr int AS_THREADS = 256;

constexpr int AS_TQ_MAX = 4;  // query tokens per block: each decoded code serves all of them
// cached tokens per thread for a single query token (tuning macro): 46 vs 54 us (1) and
// 57 us (4, 148 registers) for one query over a 131072-token 8B cache at group 128
#ifndef QKQ_AS_TPT
#define QKQ_AS_TPT 2
#endif
constexpr int AS_TPT = QKQ_AS_TPT;

template <int DH, int G, int QPK, int AS_TQ, int TPT>
__global__ void __launch_bounds__(AS_THREADS) k_attention_scores(const ScoresParams p)
{
    constexpr int NG = DH / G;
    constexpr int WPG = G / 8;  // 32-bit code words per group
    // [AS_TQ query tokens][QPK query heads of this key head][DH]
    __shared__ __align__(16) float qs[AS_TQ * QPK * DH];
    const int64_t tq0 = static_cast<int64_t>(blockIdx.y) * AS_TQ;
    const int nt = p.Tq - tq0 < AS_TQ ? static_cast<int>(p.Tq - tq0) : AS_TQ;
    const int hk = blockIdx.z;
    for (int i = threadIdx.x; i < AS_TQ * QPK * DH; i += AS_THREADS) {
        const int t = i / (QPK * DH), rest = i % (QPK * DH);
        const int tt = t < nt ? t : nt - 1;  // missing tokens repeat the last (not stored)
        const uint16_t *qrow = p.q + ((tq0 + tt) * p.Hq + hk * QPK) * DH;
        qs[i] = __uint_as_float(static_cast<uint32_t>(qrow[rest]) << 16);
    }
    __syncthreads();
    // TPT cached tokens per thread, AS_THREADS apart (coalesced score stores); each query
    // value read from shared memory serves all of them
    const int64_t tk0 = static_cast<int64_t>(blockIdx.x) * AS_THREADS * TPT + threadIdx.x;
    if (tk0 >= p.Tk) return;
    uint32_t w[TPT][DH / 8];
    int64_t r[TPT];
#pragma unroll
    for (int u = 0; u < TPT; ++u) {
        const int64_t tk = tk0 + u * AS_THREADS;
        r[u] = (tk < p.Tk ? tk : p.Tk - 1) * p.Hkv + hk;  // ragged tail: a real row, not stored
        const uint4 *crow = reinterpret_cast<const uint4 *>(p.k_codes + r[u] * (DH / 2));
#pragma unroll
        for (int i = 0; i < DH / 32; ++i) {
            const uint4 v = __ldg(crow + i);
            w[u][4 * i] = v.x;
            w[u][4 * i + 1] = v.y;
            w[u][4 * i + 2] = v.z;
            w[u][4 * i + 3] = v.w;
        }
    }
    float acc[TPT][AS_TQ][QPK];
#pragma unroll
    for (int u = 0; u < TPT; ++u)
#pragma unroll
        for (int t = 0; t < AS_TQ; ++t)
#pragma unroll
            for (int j = 0; j < QPK; ++j) acc[u][t][j] = 0.0f;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        float sg[TPT];
#pragma unroll
        for (int u = 0; u < TPT; ++u)
            sg[u] = __half2float(__ushort_as_half(__ldg(p.k_scales + r[u] * NG + g)));
        // per query row and cached token: even- and odd-channel partial sums of q * code
        // (packed fp32x2)
        float2 part[TPT][AS_TQ][QPK];
#pragma unroll
        for (int u = 0; u < TPT; ++u)
#pragma unroll
            for (int t = 0; t < AS_TQ; ++t)
#pragma unroll
                for (int j = 0; j < QPK; ++j) part[u][t][j] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int x = 0; x < WPG; ++x) {
            const int word = g * WPG + x;
            float2 c[TPT][4];
#pragma unroll
            for (int u = 0; u < TPT; ++u) codes_to_float2(w[u][word], c[u]);
#pragma unroll
            for (int t = 0; t < AS_TQ; ++t) {
                if (t >= nt) break;  // the same for every thread of the block
#pragma unroll
                for (int j = 0; j < QPK; ++j) {
                    const float *qh = qs + (t * QPK + j) * DH + word * 8;
                    const float4 q0 = *reinterpret_cast<const float4 *>(qh);
                    const float4 q1 = *reinterpret_cast<const float4 *>(qh + 4);
#pragma unroll
                    for (int u = 0; u < TPT; ++u) {
                        float2 a = part[u][t][j];
                        a = __ffma2_rn(make_float2(q0.x, q0.y), c[u][0], a);
                        a = __ffma2_rn(make_float2(q0.z, q0.w), c[u][1], a);
                        a = __ffma2_rn(make_float2(q1.x, q1.y), c[u][2], a);
                        a = __ffma2_rn(make_float2(q1.z, q1.w), c[u][3], a);
                        part[u][t][j] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < TPT; ++u)
#pragma unroll
            for (int t = 0; t < AS_TQ; ++t)
#pragma unroll
                for (int j = 0; j < QPK; ++j)
                    acc[u][t][j] = __fmaf_rn(sg[u], __fadd_rn(part[u][t][j].x, part[u][t][j].y),
                                             acc[u][t][j]);
    }
#pragma unroll
    for (int u = 0; u < TPT; ++u) {
        const int64_t tk = tk0 + u * AS_THREADS;
        if (tk >= p.Tk) break;
#pragma unroll
        for (int t = 0; t < AS_TQ; ++t)
            if (t < nt)
#pragma unroll
                for (int j = 0; j < QPK; ++j)
                    p.scores[((tq0 + t) * p.Hq + hk * QPK + j) * p.Tk + tk] = acc[u][t][j];
    }
}

using ScoresKernel = void (*)(ScoresParams);

template <int DH, int G, int TQB, int TPT>
ScoresKernel pick_group(int qpk)
{
    switch (qpk) {
    case 1: return k_attention_scores<DH, G, 1, TQB, TPT>;
    case 2: return k_attention_scores<DH, G, 2, TQB, TPT>;
    case 3: return k_attention_scores<DH, G, 3, TQB, TPT>;
    case 4: return k_attention_scores<DH, G, 4, TQB, TPT>;
    case 6: return k_attention_scores<DH, G, 6, TQB, TPT>;
    case 8: return k_attention_scores<DH, G, 8, TQB, TPT>;
    }
    return nullptr;
}

// single-token decode: one query token per block, AS_TPT cached tokens per thread; else up
// to AS_TQ_MAX query tokens per block, one cached token per thread
template <int DH, int G>
ScoresKernel pick_tokens(int qpk, int64_t Tq)
{
    return Tq == 1 ? pick_group<DH, G, 1, AS_TPT>(qpk) : pick_group<DH, G, AS_TQ_MAX, 1>(qpk);
}

}  // namespace

cudaError_t attention_scores_launch(const ScoresParams &p, int d_h, int group, cudaStream_t stream)
{
    if (p.Tq <= 0 || p.Tk <= 0) return cudaSuccess;
    const int qpk = p.Hq / p.Hkv;
    ScoresKernel kern = nullptr;
    if (d_h == 64) {
        if (group == 32) kern = pick_tokens<64, 32>(qpk, p.Tq);
        if (group == 64) kern = pick_tokens<64, 64>(qpk, p.Tq);
    } else if (d_h == 128) {
        if (group == 32) kern = pick_tokens<128, 32>(qpk, p.Tq);
        if (group == 64) kern = pick_tokens<128, 64>(qpk, p.Tq);
        if (group == 128) kern = pick_tokens<128, 128>(qpk, p.Tq);
    }
    const int tqb = p.Tq == 1 ? 1 : AS_TQ_MAX;
    const int tpt = p.Tq == 1 ? AS_TPT : 1;
    if (kern == nullptr) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>((p.Tk + AS_THREADS * tpt - 1) / (AS_THREADS * tpt)),
                    static_cast<unsigned>((p.Tq + tqb - 1) / tqb), static_cast<unsigned>(p.Hkv));
    kern<<<grid, AS_THREADS, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace qkq

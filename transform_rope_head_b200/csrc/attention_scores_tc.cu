// KV4 consumer on the tensor cores: attention logits of a block of transformed queries
// against the int4 key cache, one GEMM per key head.
//
// The logits are S[tq][h][tk] = sum_g scale[tk][h_kv][g] * sum_{c in g} Q~[tq][h][c] * code[tk][h_kv][c]
// (the online rotation cancels in Q~ K~^T: "LLM旋转量化笔记" §3.2.1).  For one key head the
// inner sums are a dense contraction over the channels of a group,
//   D_g[tk][m] = sum_{c in g} code[tk][c] * Qrow_m[c],   m = (query token, query head of the group),
// which the 5th-generation tensor cores compute exactly in their products: the codes
// (-7 .. 7) and the bf16 queries are both bf16 operands, every product is exact and the
// accumulator is fp32.  A tile is M = 128 cached tokens (A: their codes as bf16, one row per
// token) by N query rows (B: the block's transformed queries, loaded once per CTA), with one
// accumulator of N columns per scale group in tensor memory.  The epilogue reads thread t's
// TMEM lane (cached token t of the tile) and adds the groups in order,
//   S = fma(scale_g, D_g, S)  (g = 0, 1, ...),
// as the CUDA-core kernel does, then stores each query row's logit: consecutive threads,
// consecutive cached tokens, so the stores coalesce.
//
// Numerics: the products are exact; the tensor cores add the products of a group in fp32 in
// an order of their own, so a score is within 2 (d_h + d_h/group + 2) 2^-24 sum_c |q_c|
// |scale code_c| of the exact value (twice the CUDA-core kernel's bound, allowing each
// addition one ulp instead of half of one).
//
// One CTA of 4 or 8 warps per (key head, run of tiles): thread t (with 8 warps threads t and
// t + 128, a half each) loads cached token t's codes (16-byte loads, one tile ahead) and
// unpacks them into the 128-byte-swizzled K-major A operand, one elected thread issues the
// MMAs and commits them to an mbarrier, all threads wait (time-bounded) and run the
// epilogue (with 8 warps, warps w and w + 4 read the same 32 TMEM lanes and take alternate
// 32-column chunks).  8 warps when the accumulators fill 256 TMEM columns (two CTAs per
// SM), 4 otherwise (more CTAs per SM).  No TMA, no multicast.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "kv4_codes.cuh"
#include "tcgen05.cuh"

namespace qkq {

namespace {

constexpr int AST_M = 128;         // cached tokens per tile, one per TMEM lane
constexpr int AST_NMAX = 256;     // query rows per launch (the MMA's N, a multiple of 32)
constexpr int AST_TMEM_COLS = 512;

// Shared memory: [A: 128 x d_h bf16 | B: N x d_h bf16 | mbarrier, tmem slot | the logits'
// row offsets, N x int64], 1024-aligned.
__host__ __device__ constexpr int ast_a_bytes(int dh) { return AST_M * dh * 2; }
__host__ __device__ constexpr int ast_b_bytes(int dh, int n) { return n * dh * 2; }
__host__ __device__ constexpr int ast_smem_bytes(int dh, int n)
{
    return 1024 + ast_a_bytes(dh) + ast_b_bytes(dh, n) + 16 + 8 * n;
}

template <int DH, int G, int TH>
__global__ void __launch_bounds__(TH) k_attention_scores_tc(const ScoresParams p, int64_t tq0, int nq,
                                                            int N, int tmem_cols)
{
    constexpr int HALVES = TH / AST_M;  // threads per cached token
    constexpr int NG = DH / G;
    constexpr int KS = DH / 16;  // MMA K-steps of 16 channels
    constexpr int KSG = G / 16;  // K-steps per scale group
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *a_op = smem;
    uint8_t *b_op = smem + ast_a_bytes(DH);
    uint64_t *bar = reinterpret_cast<uint64_t *>(b_op + ast_b_bytes(DH, N));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(b_op + ast_b_bytes(DH, N) + 8);
    // query row m's logits start at scores + rowoff[m] (-1: a padding row)
    int64_t *rowoff = reinterpret_cast<int64_t *>(b_op + ast_b_bytes(DH, N) + 16);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & (AST_M - 1), half = tid >> 7;  // cached token row, part of its channels
    const int hk = blockIdx.y;
    const int qpk = p.Hq / p.Hkv;
    const int rows = nq * qpk;  // valid query rows of B
    int flags = 0;

    // B: query row m = (token tq0 + m / qpk, head hk * qpk + m % qpk); rows past the block zero
    for (int i = tid; i < N * (DH / 8); i += TH) {
        const int m = i / (DH / 8), c8 = i % (DH / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m < rows) {
            const int64_t qrow = (tq0 + m / qpk) * p.Hq + hk * qpk + m % qpk;
            v = __ldg(reinterpret_cast<const uint4 *>(p.q + qrow * DH) + c8);
        }
        *reinterpret_cast<uint4 *>(b_op + sw128_offset_rows(N, m, c8 * 8)) = v;
    }
    for (int m = tid; m < N; m += TH)
        rowoff[m] = m < rows ? ((tq0 + m / qpk) * p.Hq + hk * qpk + m % qpk) * p.Tk : -1;
    if (tid == 0) {
        mbar_init(smem_addr(bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), static_cast<uint32_t>(tmem_cols));
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // B written by the generic proxy, read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t a_s = smem_addr(a_op), b_s = smem_addr(b_op);
    const uint32_t idesc = idesc_bf16(N);

    const int64_t n_tiles = (p.Tk + AST_M - 1) / AST_M;
    // this thread's cached token of a tile (clamped into range for the ragged tail: its
    // codes are read and multiplied, its logits not stored)
    auto token_of = [&](int64_t tile) {
        const int64_t tk = tile * AST_M + row;
        return tk < p.Tk ? tk : p.Tk - 1;
    };
    constexpr int HW = DH / 32 / HALVES;  // 16-byte words of codes per thread
    uint4 cw[HW];  // this thread's part of the token's code bytes, loaded one tile ahead
    auto load_codes = [&](int64_t tile) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.k_codes + (token_of(tile) * p.Hkv + hk) * (DH / 2)) + half * HW;
#pragma unroll
        for (int i = 0; i < HW; ++i) cw[i] = __ldg(src + i);
    };
    if (static_cast<int64_t>(blockIdx.x) < n_tiles) load_codes(blockIdx.x);

    uint32_t phase = 0;
    bool failed = false;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t tk = tile * AST_M + row;
        const int64_t tkc = token_of(tile);
        // A row `row`, this half of its channels: the codes as bf16 (exact), 8 channels per
        // 16-byte chunk
#pragma unroll
        for (int i = 0; i < HW; ++i) {
            const uint32_t w[4] = {cw[i].x, cw[i].y, cw[i].z, cw[i].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t c[4];
                codes_to_bf16x2(w[u], c);
                const uint4 v = make_uint4(c[0], c[1], c[2], c[3]);
                const int ch = half * (DH / HALVES) + 32 * i + 8 * u;
                *reinterpret_cast<uint4 *>(a_op + sw128_offset<AST_M>(row, ch)) = v;
            }
        }
        float sg[NG];
#pragma unroll
        for (int g = 0; g < NG; ++g)
            sg[g] = __half2float(__ushort_as_half(__ldg(p.k_scales + (tkc * p.Hkv + hk) * NG + g)));
        fence_proxy_async_smem();  // A written by this thread, read by the tensor cores
        tc_fence_before();         // (and the previous tile's TMEM reads done)
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
                for (int s = 0; s < KSG; ++s) {
                    // K-step ks: K-block ks / 4 (64 channels), 32 bytes further per step inside it
                    const int ks = g * KSG + s;
                    const uint32_t aoff = (ks >> 2) * (AST_M * 128) + (ks & 3) * 32;
                    const uint32_t boff = (ks >> 2) * (N * 128) + (ks & 3) * 32;
                    mma_bf16(tmem + static_cast<uint32_t>(g * N), sw128_desc(a_s + aoff),
                             sw128_desc(b_s + boff), idesc, s ? 1u : 0u);
                }
            mma_commit(smem_addr(bar));
        }
        static_assert(KS == NG * KSG, "groups tile the channels");
        // the next tile's codes are read while the tensor cores run and the epilogue stores
        if (tile + gridDim.x < n_tiles) load_codes(tile + gridDim.x);
        const bool ok = mbar_wait_bounded(smem_addr(bar), phase);
        phase ^= 1u;
        if (__syncthreads_or(!ok)) {
            flags |= ST_TIMEOUT;
            failed = true;
            break;
        }
        tc_fence_after();

        // epilogue: thread tid reads TMEM lane `row` (cached token tk), its share of the
        // 32-column chunks, N columns per group
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        for (int c0 = 32 * half; c0 < N; c0 += 32 * HALVES) {
            float acc[32];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                float v[32];
                tmem_ld32(lane_addr + static_cast<uint32_t>(g * N + c0), v);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = __fmaf_rn(sg[g], v[i], g ? acc[i] : 0.0f);
            }
            if (tk < p.Tk) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int m = c0 + i;
                    const int64_t ro = rowoff[m];  // the same for the whole warp
                    if (ro >= 0) {
                        p.scores[ro + tk] = acc[i];
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (failed) {
        // the MMAs did not complete in time: one more bounded wait before the tensor memory
        // is released
        mbar_wait_bounded(smem_addr(bar), phase ^ 1u);
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, static_cast<uint32_t>(tmem_cols));
    }
    if (flags && p.status) atomicOr(p.status, flags);
}

using ScoresTcKernel = void (*)(ScoresParams, int64_t, int, int, int);

template <int TH>
ScoresTcKernel pick_tc(int d_h, int group)
{
    if (d_h == 64) {
        if (group == 32) return k_attention_scores_tc<64, 32, TH>;
        if (group == 64) return k_attention_scores_tc<64, 64, TH>;
    } else if (d_h == 128) {
        if (group == 32) return k_attention_scores_tc<128, 32, TH>;
        if (group == 64) return k_attention_scores_tc<128, 64, TH>;
        if (group == 128) return k_attention_scores_tc<128, 128, TH>;
    }
    return nullptr;
}

// Registers per thread of a kernel instance; the first call for it on a device also raises its
// dynamic shared-memory limit to the device's opt-in maximum.  Cached per (kernel, device).
cudaError_t tc_kernel_regs(ScoresTcKernel kern, const DeviceInfo &dev, int smem_cap, int *regs)
{
    struct Entry {
        ScoresTcKernel kern;
        int ordinal, regs;
    };
    constexpr int kCache = 64;
    static std::mutex mu;
    static Entry cache[kCache];
    static int used = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].kern == kern && cache[i].ordinal == dev.ordinal) {
            *regs = cache[i].regs;
            return cudaSuccess;
        }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_cap);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    *regs = fa.numRegs > 0 ? fa.numRegs : 1;
    if (used < kCache) cache[used++] = {kern, dev.ordinal, *regs};
    return cudaSuccess;
}

int pow2_at_least(int x)
{
    int v = 32;
    while (v < x) v <<= 1;
    return v;
}

}  // namespace

// Blocks of query tokens of at most AST_NMAX / groups query rows (the accumulators of two
// CTAs then fit in an SM's 512 TMEM columns), one launch each.  As many CTAs share an SM as
// registers, shared memory and TMEM columns allow (fewer query rows: more CTAs to hide the
// latency of each tile's loads, MMAs and stores); the shared-memory request is padded so
// that no more than that become resident, each then holding its TMEM columns.
cudaError_t attention_scores_tc_launch(const ScoresParams &p, int d_h, int group,
                                       const DeviceInfo &dev, cudaStream_t stream)
{
    if (p.Tq <= 0 || p.Tk <= 0) return cudaSuccess;
    if (pick_tc<128>(d_h, group) == nullptr) return cudaErrorInvalidValue;
    const int qpk = p.Hq / p.Hkv, ng = d_h / group;
    const int nmax = AST_NMAX / ng;
    const int tokens_per_block = nmax / qpk;  // >= 1: qpk <= 8, nmax >= 64
    if (tokens_per_block < 1) return cudaErrorInvalidValue;
    const int per_sm = dev.smem_per_sm > 0 ? dev.smem_per_sm : 228 * 1024;
    const int smem_cap = dev.smem_per_block_optin > 0 ? dev.smem_per_block_optin : 227 * 1024;
    const int64_t n_tiles = (p.Tk + AST_M - 1) / AST_M;
    for (int64_t tq0 = 0; tq0 < p.Tq; tq0 += tokens_per_block) {
        const int nq = static_cast<int>(p.Tq - tq0 < tokens_per_block ? p.Tq - tq0 : tokens_per_block);
        const int N = (nq * qpk + 31) / 32 * 32;
        // 8 warps when the accumulators take 256 TMEM columns (two CTAs per SM), else 4 (more
        // CTAs): 16 query tokens x 4 heads over a 131072-token cache 223 vs 259 us at group 128
        // (64 columns), 222 vs 304 us at group 32 (4 x 64 columns)
        const int th = ng * N >= 256 ? 256 : 128;
        const ScoresTcKernel kern = th == 256 ? pick_tc<256>(d_h, group) : pick_tc<128>(d_h, group);
        int regs = 0;
        cudaError_t e = tc_kernel_regs(kern, dev, smem_cap, &regs);
        if (e != cudaSuccess) return e;
        const int cols = pow2_at_least(ng * N);
        const int need = ast_smem_bytes(d_h, N);
        // CTAs per SM: registers (8-register granules per thread), shared memory (1 KB
        // reserved per CTA), TMEM columns, and at most 8
        int ctas = 65536 / (th * ((regs + 7) / 8 * 8));
        const int by_smem = per_sm / (need + 1024);
        const int by_tmem = AST_TMEM_COLS / cols;
        ctas = ctas < by_smem ? ctas : by_smem;
        ctas = ctas < by_tmem ? ctas : by_tmem;
        ctas = ctas < 8 ? ctas : 8;
        if (ctas < 1) return cudaErrorInvalidValue;
        // pad the request so that shared memory admits no more than `ctas` CTAs
        const int floor_req = per_sm / (ctas + 1) - 1024 + 1;
        const int req = need > floor_req ? need : floor_req;
        if (req > smem_cap) return cudaErrorInvalidValue;
        const int64_t per_head = (static_cast<int64_t>(dev.num_sms) * ctas + p.Hkv - 1) / p.Hkv;
        const unsigned gx = static_cast<unsigned>(n_tiles < per_head ? n_tiles : per_head);
        kern<<<dim3(gx, static_cast<unsigned>(p.Hkv)), th, req, stream>>>(p, tq0, nq, N, cols);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qkq

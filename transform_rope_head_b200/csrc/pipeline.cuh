// Per-warp token pipeline shared by the streaming kernels.
//
// Each warp owns S shared-memory stages; a stage holds one token: its Hq query rows
// and Hkv key rows (each block contiguous in HBM, so one bulk copy each) followed by
// the token's cos and sin table rows (two rows each for a split table) and, for a
// kernel that asks, one more per-token block such as the packed codes.  Lane 0 issues the bulk copies (cp.async.bulk,
// no multicast) S tokens ahead onto the stage's mbarrier; all lanes wait on it with a
// time bound (on a timeout it records ST_TIMEOUT, waits, bounded again, for its copies in
// flight, and stops).  Tokens are dealt to the warps of a persistent grid round-robin
// (token = gw + n * nw for the warp's n-th token).  Positions are read 32 tokens at a
// time, one per lane, two blocks ahead, so a table row address never waits on a load.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace qkq {

// Launch shape of a pipelined kernel: stages per warp, dynamic shared memory, and a
// persistent grid of the CTAs that are resident at once (CTAs per SM x SMs, as the
// occupancy calculator gives them for the kernel's registers and shared memory; fewer
// when there are fewer tokens than warps, or when the caller caps them).
struct PipeLaunch {
    int stages;
    size_t smem;
    int grid;
};

// Tuning overrides, read once from the environment (unset: the planner's choice):
//   QKQ_PIPE_STAGES = stages per warp (1 .. max_stages), QKQ_PIPE_CTAS = CTAs per SM cap.
inline int pipe_env(const char *name)
{
    const char *v = getenv(name);
    return v ? atoi(v) : 0;
}

// Resident CTAs per SM of kern at `threads` threads and `smem` bytes of dynamic shared
// memory on device `ordinal`.  The first call for a kernel on a device raises its
// dynamic shared memory limit to the device's opt-in maximum and asks for the largest
// shared-memory carveout; results are cached.
inline cudaError_t resident_ctas(const void *kern, int threads, size_t smem, const DeviceInfo &dev,
                                 int *per_sm)
{
    struct Entry {
        const void *kern;
        int ordinal, threads;
        size_t smem;
        int per_sm;  // -1: only the attribute has been set
    };
    constexpr int kCache = 512;
    static std::mutex mu;
    static Entry cache[kCache];
    static int used = 0;
    std::lock_guard<std::mutex> lock(mu);
    bool attr_set = false;
    for (int i = 0; i < used; ++i) {
        const Entry &e = cache[i];
        if (e.kern != kern || e.ordinal != dev.ordinal) continue;
        attr_set = true;
        if (e.threads == threads && e.smem == smem && e.per_sm >= 0) {
            *per_sm = e.per_sm;
            return cudaSuccess;
        }
    }
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             dev.smem_per_block_optin);
        if (e != cudaSuccess) return e;
        // the whole unified L1 / shared array as shared memory, so that the occupancy the
        // calculator reports (and the grid is sized for) is the one the launch gets
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (used < kCache) cache[used++] = Entry{kern, dev.ordinal, 0, 0, -1};
    }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (used < kCache) cache[used++] = Entry{kern, dev.ordinal, threads, smem, n};
    *per_sm = n;
    return cudaSuccess;
}

// Plan a launch of kern (warps x 32 threads).  Shared memory = fixed_smem + the stage
// area, which is at least min_area bytes (a kernel that reuses it after its loop asks for
// room there).  Stages: the most (up to max_stages) that still let want_ctas CTAs share
// an SM's shared memory.
template <class Kern>
inline cudaError_t plan_pipeline(Kern kern, int warps, int stage_bytes, size_t fixed_smem,
                                 size_t min_area, int max_stages, int want_ctas, int64_t T,
                                 int max_ctas, const DeviceInfo &dev, PipeLaunch *out)
{
    static const int env_stages = pipe_env("QKQ_PIPE_STAGES");
    static const int env_ctas = pipe_env("QKQ_PIPE_CTAS");
    const size_t reserve = 1024;  // per-CTA shared memory the runtime keeps
    auto smem_of = [&](int s) {
        const size_t area = static_cast<size_t>(warps) * s * stage_bytes;
        return fixed_smem + (area > min_area ? area : min_area);
    };
    int stages = max_stages;
    if (env_stages > 0) {
        stages = env_stages < max_stages ? env_stages : max_stages;
    } else {
        while (stages > 1 &&
               static_cast<size_t>(want_ctas) * (smem_of(stages) + reserve) > static_cast<size_t>(dev.smem_per_sm))
            --stages;
    }
    const size_t smem = smem_of(stages);
    if (smem > static_cast<size_t>(dev.smem_per_block_optin)) return cudaErrorInvalidConfiguration;
    int per_sm = 0;
    cudaError_t e = resident_ctas(reinterpret_cast<const void *>(kern), warps * 32, smem, dev, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (env_ctas > 0 && env_ctas < per_sm) per_sm = env_ctas;
    const int64_t need = (T + warps - 1) / warps;
    int64_t grid = static_cast<int64_t>(dev.num_sms) * per_sm;
    if (grid > max_ctas) grid = max_ctas;
    if (grid > need) grid = need;
    out->stages = stages;
    out->smem = smem;
    out->grid = static_cast<int>(grid);
    return cudaSuccess;
}

// Table rows a stage holds: cos and sin of the position, or with a split table cos and
// sin of its low row and of its high row.
__host__ __device__ inline int table_rows(bool split) { return split ? 4 : 2; }

// Bytes of one stage (a multiple of 128): Q rows (unless the kernel skips them, Hq = 0
// here), K rows, the table rows, and an optional per-token block of extra_bytes.
__host__ __device__ inline int token_stage_bytes(int Hq, int Hkv, int d_h, bool split, int extra_bytes = 0)
{
    const long b = static_cast<long>(Hq + Hkv) * d_h * 2 +
                   static_cast<long>(d_h / 2) * 4 * table_rows(split) + extra_bytes;
    return static_cast<int>((b + 127) / 128 * 128);
}

struct TokenPipe {
    uint8_t *stages;     // this warp's S stages
    uint32_t bar0;       // shared address of this warp's first mbarrier (8 bytes apart)
    int S, SB;
    int64_t gw, nw, ntok;
    // reverse: tokens are taken from the last one down (a kernel that follows one reading the
    // same tokens in order then starts on those still in L2); tlast = T - 1
    bool rev = false;
    int64_t tlast = 0;
    uint32_t qbytes, kbytes, tbytes, ebytes;
    bool split;
    // Row-split units (set by start; 1 = one unit per token): a token's query rows in
    // parts of 8 rows, then one part with all its key rows (and the extra block).
    int np = 1, nqp = 0, hq = 0;
    uint32_t rowb = 0;
    const uint8_t *qsrc, *ksrc, *esrc;
    const float *cos_t, *sin_t;
    const int32_t *pos;
    int max_pos;
    int lane;
    int64_t pos_blk;
    int pos_cur, pos_nxt;

    __device__ int load_pos_block(int64_t blk) const
    {
        const int64_t n = blk * 32 + lane;
        return n < ntok ? __ldg(pos + unit_token(gw + n * nw)) : 0;
    }

    // Set up: barriers (lane 0), position prefetch, and the first S copies.
    __device__ void start(uint8_t *my_stages, uint64_t *my_bars, int n_stages, int stage_bytes,
                          int64_t warp_global, int64_t warps_total, int64_t T, int Hq, int Hkv,
                          int d_h, const void *q, const void *k, const float *ct, const float *st,
                          const int32_t *p, int mp, bool split_tab, int &flags,
                          bool copy_q = true, const void *extra = nullptr,
                          uint32_t extra_bytes = 0, int parts = 1, bool reverse = false)
    {
        split = split_tab;
        np = parts;
        hq = Hq;
        rowb = static_cast<uint32_t>(d_h) * 2;
        nqp = parts > 1 ? (Hq + 7) / 8 : 0;
        stages = my_stages;
        bar0 = smem_addr(my_bars);
        S = n_stages;
        SB = stage_bytes;
        gw = warp_global;
        nw = warps_total;
        rev = reverse;
        tlast = T - 1;
        const int64_t units = T * parts;
        ntok = units > gw ? (units - gw + nw - 1) / nw : 0;
        qbytes = copy_q ? static_cast<uint32_t>(Hq) * d_h * 2 : 0u;
        kbytes = static_cast<uint32_t>(Hkv) * d_h * 2;
        tbytes = static_cast<uint32_t>(d_h / 2) * 4;
        qsrc = static_cast<const uint8_t *>(q);
        ksrc = static_cast<const uint8_t *>(k);
        esrc = static_cast<const uint8_t *>(extra);
        ebytes = extra ? extra_bytes : 0u;
        cos_t = ct;
        sin_t = st;
        pos = p;
        max_pos = mp;
        lane = threadIdx.x & 31;
        if (lane == 0) {
            for (int s = 0; s < S; ++s) mbar_init(bar0 + 8 * s, 1);
            fence_mbar_init();
        }
        __syncwarp();
        pos_blk = 0;
        pos_cur = load_pos_block(0);
        pos_nxt = load_pos_block(1);
        for (int s = 0; s < S && s < ntok; ++s) issue(s, s, flags);
    }

    // Copies of this warp's n-th token into stage s.  Warp-uniform call, n increasing by 1.
    __device__ void issue(int64_t n, int s, int &flags)
    {
        const int64_t blk = n >> 5;
        if (blk != pos_blk) {
            pos_cur = pos_nxt;
            pos_nxt = load_pos_block(blk + 1);
            pos_blk = blk;
        }
        const int m = __shfl_sync(FULL_MASK, pos_cur, static_cast<int>(n & 31));
        if (lane == 0) {
            const int64_t u = gw + n * nw;
            const int64_t tf = unit_token_fwd(u);
            const int part = static_cast<int>(u - tf * np);
            const int64_t t = rev ? tlast - tf : tf;
            const int64_t mc = clamp_pos(m, max_pos, flags);
            const int P = static_cast<int>(tbytes / 4);
            const uint32_t bar = bar0 + 8 * s;
            const uint32_t dst = smem_addr(stages + static_cast<size_t>(s) * SB);
            // rows of this unit: every Q and K row (one unit per token), 8 Q rows of a Q part,
            // or every K row of the key part
            const uint32_t rb = unit_row_bytes(part);
            const uint32_t eb = (np == 1 || part == nqp) ? ebytes : 0u;
            const uint32_t tab = dst + rb;
            fence_proxy_async_smem();
            // the unit's token, its table rows and the staged bytes must stay in range: the
            // bounds-checking build skips the copies (and completes the stage's phase with no
            // bytes, so nothing waits for them) if they do not
            const int64_t trows = split ? 64 + (static_cast<int64_t>(max_pos) + 63) / 64 : max_pos;
            const int64_t row_hi = split ? 64 + (mc >> 6) : mc;
            if (!(QKQ_IN_BOUNDS(t >= 0 && t <= tlast && mc >= 0 && row_hi < trows &&
                                    rb + table_rows(split) * tbytes + eb <= static_cast<uint32_t>(SB) &&
                                    part >= 0 && part < np, flags))) {
                mbar_arrive(bar);
                return;
            }
            mbar_arrive_expect_tx(bar, rb + table_rows(split) * tbytes + eb);
            if (np == 1) {
                if (qbytes) bulk_copy_g2s(dst, qsrc + t * qbytes, qbytes, bar);
                bulk_copy_g2s(dst + qbytes, ksrc + t * kbytes, kbytes, bar);
            } else if (part < nqp) {
                bulk_copy_g2s(dst, qsrc + t * qbytes + static_cast<int64_t>(part) * 8 * rowb, rb, bar);
            } else {
                bulk_copy_g2s(dst, ksrc + t * kbytes, kbytes, bar);
            }
            if (split) {  // low row m % 64, then high row 64 + m / 64
                const int64_t lo = mc & 63, hi = 64 + (mc >> 6);
                bulk_copy_g2s(tab, cos_t + lo * P, tbytes, bar);
                bulk_copy_g2s(tab + tbytes, sin_t + lo * P, tbytes, bar);
                bulk_copy_g2s(tab + 2 * tbytes, cos_t + hi * P, tbytes, bar);
                bulk_copy_g2s(tab + 3 * tbytes, sin_t + hi * P, tbytes, bar);
            } else {
                bulk_copy_g2s(tab, cos_t + mc * P, tbytes, bar);
                bulk_copy_g2s(tab + tbytes, sin_t + mc * P, tbytes, bar);
            }
            if (eb) bulk_copy_g2s(tab + table_rows(split) * tbytes, esrc + t * ebytes, eb, bar);
        }
    }

    // Bytes of the rows a unit stages (before its table rows).
    __host__ __device__ uint32_t unit_row_bytes(int part) const
    {
        if (np == 1) return qbytes + kbytes;
        if (part < nqp) {
            const int r = hq - part * 8;
            return static_cast<uint32_t>(r < 8 ? r : 8) * rowb;
        }
        return kbytes;
    }

    // Wait for this warp's n-th token; returns its stage, or nullptr if the bounded wait
    // gave up (every lane then leaves together and ST_TIMEOUT is recorded).
    __device__ const uint8_t *wait(int64_t n, int &flags)
    {
        const int s = static_cast<int>(n % S);
        const uint32_t parity = static_cast<uint32_t>((n / S) & 1);
        if (!__all_sync(FULL_MASK, mbar_wait_bounded(bar0 + 8 * s, parity))) {
            flags |= ST_TIMEOUT;
            drain(n, n + S);
            return nullptr;
        }
        return stages + static_cast<size_t>(s) * SB;
    }

    // After a timeout: wait, again with the time bound, for the copies of the issued
    // tokens first .. end - 1 that may still be in flight, so that none lands in this
    // warp's stages after it has moved on.
    __device__ void drain(int64_t first, int64_t end) const
    {
        for (int64_t m = first; m < end && m < ntok; ++m)
            mbar_wait_bounded(bar0 + 8 * static_cast<uint32_t>(m % S), static_cast<uint32_t>((m / S) & 1));
    }

    // The stage of token n has been read by every lane: refill it with token n + S.
    __device__ void release(int64_t n, int &flags)
    {
        __syncwarp();
        if (n + S < ntok) issue(n + S, static_cast<int>(n % S), flags);
    }

    // Token of unit u in unit order.  Row-split units are only planned while T * parts < 2^31
    // (a few units per resident warp), so a 32-bit division serves; whole tokens need none.
    __device__ int64_t unit_token_fwd(int64_t u) const
    {
        return np == 1 ? u : static_cast<int64_t>(static_cast<uint32_t>(u) / static_cast<uint32_t>(np));
    }
    // The token unit u works on (from the last one down when reversed).
    __device__ int64_t unit_token(int64_t u) const
    {
        const int64_t t = unit_token_fwd(u);
        return rev ? tlast - t : t;
    }
    __device__ int64_t token(int64_t n) const { return unit_token(gw + n * nw); }
    __device__ int part(int64_t n) const
    {
        const int64_t u = gw + n * nw;
        return static_cast<int>(u - unit_token_fwd(u) * np);
    }

    // Offsets inside a stage: the table rows, and the extra block after them.
    __device__ uint32_t table_offset() const { return qbytes + kbytes; }
    __device__ uint32_t extra_offset() const { return qbytes + kbytes + table_rows(split) * tbytes; }
    // the same for a unit's part (row-split units)
    __device__ uint32_t unit_table_offset(int part) const { return unit_row_bytes(part); }
    __device__ uint32_t unit_extra_offset(int part) const
    {
        return unit_row_bytes(part) + table_rows(split) * tbytes;
    }
};

}  // namespace qkq

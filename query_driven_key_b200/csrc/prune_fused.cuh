// prune_fused.cuh -- the whole prune step of one layer (channel scores, top-T
// selection, thinner key cache) for a bf16 key cache in one persistent kernel
// that reads K from HBM about once.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): score every key channel against the query window,
// sort the channels, drop the least relevant ones, keep the thinner key cache.
//
// Scoring needs every token of a head before the head's channels can be
// chosen, so K is read twice: once to score, once to compact.  This kernel
// makes the second read an L2 hit:
//   - The heads are taken in rounds of about 2,000 64-token tiles (about
//     34 MB of bf16 keys), each head cut into runs of s_tiles tiles (the round
//     split plan; the score kernels give the same bits on that plan).  Run j
//     of a round belongs to block j % gridDim.x, in every round, for both its
//     score and its compaction, so a run is compacted on the SM that scored
//     it, about one round later, while its tiles are still in L2.
//   - One block per SM, five warp roles that never wait for one another
//     except through shared-memory rings:
//       * score producer (one thread): streams the block's score tiles of
//         every round by TMA through its own ring (`s_stages` x 16 KB); before
//         round r >= lag it waits until this block has compacted round
//         r - lag, so at most `lag` rounds are scored ahead of the compaction;
//       * eight score warps: add the squares of each tile (the thread map of
//         score_tma_kernel), add each run's row-group partials in row order
//         and queue the run partial (8 slots) for the merge warps, so that a
//         merge warp busy with a group or head merge does not stall scoring;
//       * four merge warps (one thread per channel): window-query energies,
//         the run partial, and the two-level merge of score_run_end (group and
//         head tickets); the block that completes a head forms its scores,
//         selects the top T and raises the head's ready flag.  Fences and
//         atomics stall only these warps;
//       * compact producer (one thread): streams the block's tiles again, in
//         the same order, through a second ring (`c_stages` x 16 KB);
//       * eight compact warps: wait (bounded) for the head's ready flag,
//         transpose each tile (ldmatrix.trans, then a 4x4 word transpose inside
//         each group of four lanes) and store each kept channel's 8-token runs
//         as 16-byte writes.
//     The ready flag of round r depends only on score work of round r, which
//     no block delays behind its compaction of round r or later, and every
//     block of the grid is resident (the grid is launched cooperatively, so
//     the runtime starts it only when all its blocks fit at once), so every
//     wait ends.
// Every wait is bounded; after the first one that runs out the block stops
// waiting (abort flag), still passes every barrier, and the producers let
// their loads in flight land before the block ends.
#pragma once

#include "prune_kernels.cuh"
#include "think.h"

namespace think {

constexpr int kPfTile = 64;                       // tokens per K tile
constexpr int kPfGroupThreads = 256;              // score warps, compact warps: 8 warps each
constexpr int kPfWarpScoreProd = 16, kPfWarpCompactProd = 17, kPfWarpMerge0 = 18;
constexpr int kPfMergeThreads = 128;              // merge warps: one thread per channel
constexpr int kPfThreads = 22 * 32;
constexpr int kPfMaxStages = 12;                  // score + compact stages
constexpr uint32_t kPfHalfBytes = 64u * 64u * 2u;   // 64 tokens x 64 channels x bf16
constexpr uint32_t kPfTileBytes = 2u * kPfHalfBytes;
constexpr uint32_t kPfRedBytes = 16u * kD * 8u;   // [16][128] fp64 row-group partials of one run
constexpr int kPfHandSlots = 8;                   // run partials queued for the merge warps
constexpr uint32_t kPfHandBytes = kPfHandSlots * kD * 8u;
constexpr uint32_t kPfSvBytes = 4u * kD * 8u;     // [4][128] score bits, one row per merge warp
constexpr uint32_t kPfMiscBytes = 128u;           // abort, compact rounds done, exit flag, merge flag,
                                                  // compact flag, wcnt[4]

inline size_t prune_fused_smem_bytes(int s_stages, int c_stages)
{
    return (size_t)(s_stages + c_stages) * kPfTileBytes + kPfRedBytes + kPfHandBytes + kPfSvBytes + kPfMiscBytes +
           8u * (2u * (size_t)(s_stages + c_stages) + 2u * kPfHandSlots) + 1024u;  // + mbarriers, alignment slack
}

enum : int { kPfHintScoreKeep = 1, kPfHintCompactDrop = 2, kPfHintStoreDrop = 4 };

struct PruneFusedArgs {
    ScoreArgs sc;                 // scores: plan (splits, groups), workspace, outputs (scores, idx)
    int G, T;
    int heads, tiles_per_head;
    int s_tiles;                  // tiles per run
    int hpr, rounds;              // heads per round, rounds
    int s_stages, c_stages;       // ring depths
    int hints;                    // kPfHint* bits: L2 eviction priorities
    int lag;                      // round r is scored once round r - lag is compacted (>= 1)
    int prefetch;                 // score tiles prefetched into L2 ahead of the loads
    unsigned *ready;              // [heads] selection written; reset by the last block
    unsigned *exits;              // blocks finished; reset by the last block
    __nv_bfloat16 *kp;            // K' [heads][T][ldk]
    int64_t ldk, N;
};

struct PfRun {
    int head, run, t0, t1;
};

// The runs of round r owned by block blk of nblk: f(run) for each, in order.
template <typename F>
__device__ __forceinline__ void pf_for_each_run(const PruneFusedArgs &a, int r, int blk, int nblk, F &&f)
{
    const int R = a.sc.splits;
    const int h0 = r * a.hpr;
    const int nruns = min(a.hpr, a.heads - h0) * R;
    for (int j = blk; j < nruns; j += nblk) {
        PfRun x;
        x.head = h0 + j / R;
        x.run = j % R;
        x.t0 = x.run * a.s_tiles;
        x.t1 = min(a.tiles_per_head, x.t0 + a.s_tiles);
        f(x);
    }
}

// The tiles of block blk of nblk in its order (round, run, tile), one at a
// time: start with pf_tile_first, then pf_tile_next until it returns false.
struct PfTile {
    int r, j, t, t1, head;
};

__device__ __forceinline__ bool pf_tile_next(const PruneFusedArgs &a, int nblk, PfTile &c)
{
    if (++c.t < c.t1) return true;
    const int R = a.sc.splits;
    c.j += nblk;
    for (;;) {
        if (c.r >= a.rounds) return false;
        if (c.j < min(a.hpr, a.heads - c.r * a.hpr) * R) break;
        ++c.r;
        c.j -= (c.j / nblk) * nblk;  // back to this block's first run: blk
    }
    c.head = c.r * a.hpr + c.j / R;
    c.t = (c.j % R) * a.s_tiles;
    c.t1 = min(a.tiles_per_head, c.t + a.s_tiles);
    return true;
}

__device__ __forceinline__ bool pf_tile_first(const PruneFusedArgs &a, int blk, int nblk, PfTile &c)
{
    c.r = 0;
    c.j = blk - nblk;
    c.t = c.t1 = 0;
    return pf_tile_next(a, nblk, c);
}

// Wait (bounded) until *flag is non-zero (another block raises it).
__device__ __forceinline__ bool pf_wait_flag(const unsigned *flag, unsigned *status)
{
    if (ld_acquire_gpu(flag)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t spin = 0; spin < kWaitLimitSpins; ++spin) {
        __nanosleep(64);
        if (ld_acquire_gpu(flag)) return true;
        if ((spin & 31u) == 0u && global_ns() - t0 > kWaitLimitNs) break;
    }
    atomicOr(status, THINK_DEVICE_TIMEOUT_READY);
    return false;
}

// Wait (bounded) until the shared word *w reaches at least v (this block).
__device__ __forceinline__ bool pf_wait_smem_ge(const volatile unsigned *w, unsigned v, unsigned *status)
{
    if (*w >= v) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t spin = 0; spin < kWaitLimitSpins; ++spin) {
        __nanosleep(32);
        if (*w >= v) return true;
        if ((spin & 31u) == 0u && global_ns() - t0 > kWaitLimitNs) break;
    }
    atomicOr(status, THINK_DEVICE_TIMEOUT_BARRIER);
    return false;
}

// 8 consecutive tokens of one K' row (x a multiple of 8), with an L2 policy.
__device__ __forceinline__ void store_run8_hint(__nv_bfloat16 *row, int64_t x, int64_t N, const uint32_t (&v)[4],
                                                uint64_t pol)
{
    if (x + 8 <= N) {
        asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(row + x), "r"(v[0]),
                     "r"(v[1]), "r"(v[2]), "r"(v[3]), "l"(pol)
                     : "memory");
    } else {
        store_run8(row, x, N, v);
    }
}

// Shared-memory layout of one block.
struct PfSmem {
    uint32_t ring_s, ring_c;      // shared addresses of the two rings
    double *red;                  // [16][128] score warps' row-group partials
    double *hand;                 // [kPfHandSlots][128] run partials for the merge warps
    unsigned long long *sv;       // [4][128]
    volatile unsigned *abort, *c_done;
    unsigned *last, *mflag, *cflag;
    int *wcnt;
    uint32_t full_s, empty_s, full_c, empty_c, hand_full, hand_free;  // mbarrier arrays (8 bytes apart)
};

__device__ __forceinline__ PfSmem pf_smem(const PruneFusedArgs &a, unsigned char *base)
{
    PfSmem m;
    m.ring_s = smem_addr(base);
    m.ring_c = m.ring_s + (uint32_t)a.s_stages * kPfTileBytes;
    unsigned char *p = base + (size_t)(a.s_stages + a.c_stages) * kPfTileBytes;
    m.red = reinterpret_cast<double *>(p);
    p += kPfRedBytes;
    m.hand = reinterpret_cast<double *>(p);
    p += kPfHandBytes;
    m.sv = reinterpret_cast<unsigned long long *>(p);
    p += kPfSvBytes;
    unsigned *misc = reinterpret_cast<unsigned *>(p);
    m.abort = misc;
    m.c_done = misc + 1;
    m.last = misc + 2;
    m.mflag = misc + 3;
    m.cflag = misc + 4;
    m.wcnt = reinterpret_cast<int *>(misc + 8);
    p += kPfMiscBytes;
    m.full_s = smem_addr(p);
    m.empty_s = m.full_s + 8u * (uint32_t)a.s_stages;
    m.full_c = m.empty_s + 8u * (uint32_t)a.s_stages;
    m.empty_c = m.full_c + 8u * (uint32_t)a.c_stages;
    m.hand_full = m.empty_c + 8u * (uint32_t)a.c_stages;
    m.hand_free = m.hand_full + 8u * kPfHandSlots;
    return m;
}

// A producer thread: every tile of every run of the block, round by round,
// into its ring.  score: before round r >= 2, wait until the block has
// compacted round r - 2.
__device__ __forceinline__ void pf_produce(const PruneFusedArgs &a, const CUtensorMap *tm_k, const PfSmem &m,
                                           bool score)
{
    prefetch_tensormap(tm_k);
    const int stages = score ? a.s_stages : a.c_stages;
    const uint32_t ring = score ? m.ring_s : m.ring_c;
    const uint32_t full0 = score ? m.full_s : m.full_c;
    const uint32_t empty0 = score ? m.empty_s : m.empty_c;
    const bool hint = (a.hints & (score ? kPfHintScoreKeep : kPfHintCompactDrop)) != 0;
    const uint64_t pol = !hint ? l2_policy_evict_normal() : (score ? l2_policy_evict_last() : l2_policy_evict_first());
    // score: L2 prefetches run `prefetch` tiles ahead of the loads, so that
    // more of the stream is in flight than the ring holds
    PfTile pc;
    bool pc_ok = score && a.prefetch > 0 && pf_tile_first(a, blockIdx.x, gridDim.x, pc);
    for (int i = 0; pc_ok && i < a.prefetch; ++i) {
        tma_prefetch_l2_4d(tm_k, 0, pc.t * kPfTile, pc.head % a.sc.Hkv, pc.head / a.sc.Hkv);
        tma_prefetch_l2_4d(tm_k, 64, pc.t * kPfTile, pc.head % a.sc.Hkv, pc.head / a.sc.Hkv);
        pc_ok = pf_tile_next(a, gridDim.x, pc);
    }
    int n = 0;  // tiles put into the ring
    for (int r = 0; r < a.rounds && !*m.abort; ++r) {
        if (score && r >= a.lag && !pf_wait_smem_ge(m.c_done, (unsigned)(r - a.lag + 1), a.sc.status)) {
            *m.abort = 1u;
            break;
        }
        pf_for_each_run(a, r, blockIdx.x, gridDim.x, [&](const PfRun &x) {
            const int b = x.head / a.sc.Hkv, kv = x.head % a.sc.Hkv;
            for (int t = x.t0; t < x.t1; ++t) {
                if (pc_ok) {
                    tma_prefetch_l2_4d(tm_k, 0, pc.t * kPfTile, pc.head % a.sc.Hkv, pc.head / a.sc.Hkv);
                    tma_prefetch_l2_4d(tm_k, 64, pc.t * kPfTile, pc.head % a.sc.Hkv, pc.head / a.sc.Hkv);
                    pc_ok = pf_tile_next(a, gridDim.x, pc);
                }
                const int s = n % stages, f = n / stages;
                if (*m.abort) return;
                if (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)((f - 1) & 1), a.sc.status,
                                                THINK_DEVICE_TIMEOUT_EMPTY)) {
                    *m.abort = 1u;
                    return;
                }
                const uint32_t full = full0 + 8 * s;
                const uint32_t dst = ring + (uint32_t)s * kPfTileBytes;
                mbar_arrive_expect_tx(full, kPfTileBytes);
                tma_load_4d_hint(dst, tm_k, 0, t * kPfTile, kv, b, full, pol);
                tma_load_4d_hint(dst + kPfHalfBytes, tm_k, 64, t * kPfTile, kv, b, full, pol);
                ++n;
            }
        });
    }
    // every load issued lands before the block ends
    for (int k = max(0, n - stages); k < n; ++k)
        mbar_wait_bounded(full0 + 8 * (k % stages), (uint32_t)((k / stages) & 1), a.sc.status,
                          THINK_DEVICE_TIMEOUT_FULL);
}

// Score warps (threads 0..255): squares of each tile; a run's [16][128]
// row-group partials go to red buffer (run count & 1).
__device__ __forceinline__ void pf_score(const PruneFusedArgs &a, const PfSmem &m)
{
    const int tid = threadIdx.x, lane = tid & 31;
    const int cc = tid & 15, rg = tid >> 4;
    const uint32_t s_half = (uint32_t)(cc >> 3) * kPfHalfBytes;
    const uint32_t s_chunk = (uint32_t)(cc & 7);
    const int stages = a.s_stages;
    int n = 0, cnt = 0;  // tiles taken, runs done
    for (int r = 0; r < a.rounds; ++r) {
        pf_for_each_run(a, r, blockIdx.x, gridDim.x, [&](const PfRun &x) {
            double acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0;
            // two tiles per step: both tiles' loads are in flight together
            for (int t = x.t0; t < x.t1; t += 2) {
                const int nt = min(2, x.t1 - t);
                const int n0 = n;
                n += nt;
                if (*m.abort) continue;
                uint4 w[2][4];
                bool ok = true;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i >= nt) break;
                    const int s = (n0 + i) % stages;
                    if (!mbar_wait_bounded(m.full_s + 8 * s, (uint32_t)(((n0 + i) / stages) & 1), a.sc.status,
                                           THINK_DEVICE_TIMEOUT_FULL)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = m.ring_s + (uint32_t)s * kPfTileBytes + s_half;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint32_t row = (uint32_t)(rg + 16 * k4);
                        const uint32_t addr = st + row * 128u + ((s_chunk ^ (row & 7u)) << 4);
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(w[i][k4].x), "=r"(w[i][k4].y), "=r"(w[i][k4].z), "=r"(w[i][k4].w)
                                     : "r"(addr)
                                     : "memory");
                    }
                }
                if (!ok) {
                    *m.abort = 1u;
                    continue;
                }
                add_squares4_bf16(w[0], acc);  // tile order; uses the loaded words: the stages have been read
                if (nt == 2) add_squares4_bf16(w[1], acc);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(m.empty_s + 8 * (n0 % stages));
                    if (nt == 2) mbar_arrive(m.empty_s + 8 * ((n0 + 1) % stages));
                }
            }
            // the run partial: row groups added in row order (threads 0..127,
            // one channel each), queued for the merge warps
            named_barrier(3, kPfGroupThreads);  // the previous run's sums have read red
#pragma unroll
            for (int e = 0; e < 8; ++e) m.red[rg * kD + cc * 8 + e] = acc[e];
            named_barrier(3, kPfGroupThreads);
            if (tid < kD) {
                double p = 0.0;
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) p += m.red[rr * kD + tid];
                const int k = cnt % kPfHandSlots, u = cnt / kPfHandSlots;
                if (u > 0 && !*m.abort &&
                    !mbar_wait_bounded(m.hand_free + 8 * k, (uint32_t)((u - 1) & 1), a.sc.status,
                                       THINK_DEVICE_TIMEOUT_BARRIER))
                    *m.abort = 1u;
                m.hand[k * kD + tid] = p;
                mbar_arrive(m.hand_full + 8 * k);  // threads 0..127 (count 128)
            }
            ++cnt;
        });
    }
}

// Merge warps (128 threads, thread c = channel c): per run of the block, in
// the score warps' order, the window-query energies assigned to the run, the
// run partial (from the score warps' queue) and the two-level merge of
// score_run_end (same additions, same order), then for the block that completes a head its scores, the top T and
// the head's ready flag.  Only one thread per level touches a ticket, with an
// acquire-release fetch-and-add after a merge-group barrier, so a level costs
// about one L2 round trip for the ticket and one for its loads.
__device__ __forceinline__ void pf_merge(const PruneFusedArgs &a, const PfSmem &m)
{
    const int c = threadIdx.x - 32 * kPfWarpMerge0;  // 0..127
    const int lane = c & 31, warp = c >> 5;
    const ScoreArgs &sa = a.sc;
    const int G = a.G, R = sa.splits;
    auto sync = [] { named_barrier(2, kPfMergeThreads); };
    int cnt = 0;
    for (int r = 0; r < a.rounds; ++r) {
        pf_for_each_run(a, r, blockIdx.x, gridDim.x, [&](const PfRun &x) {
            const int head = x.head;
            const int b = head / sa.Hkv, kv = head % sa.Hkv;
            // window-query energies of the query heads g of the group with
            // (head * G + g) % R == run: spread over the blocks of the grid,
            // one run of the head each
            for (int g = (int)(((int64_t)x.run - (int64_t)head * G % R + R) % R); g < G; g += R) {
                const __nv_bfloat16 *qh = static_cast<const __nv_bfloat16 *>(sa.qwin) +
                                          (((int64_t)b * sa.Hq + (int64_t)kv * G + g) * sa.S) * kD + c;
                sa.qn2[((int64_t)head * G + g) * kD + c] = window_energy<__nv_bfloat16>(qh, sa.S);
            }
            // the run partial from the score warps' queue
            const int k = cnt % kPfHandSlots, u = cnt / kPfHandSlots;
            ++cnt;
            if (!*m.abort && !mbar_wait_bounded(m.hand_full + 8 * k, (uint32_t)(u & 1), sa.status,
                                                THINK_DEVICE_TIMEOUT_BARRIER))
                *m.abort = 1u;
            if (THINK_IN_RANGE(head < a.heads && x.run < R, sa.status))
                sa.part[((int64_t)head * R + x.run) * kD + c] = m.hand[k * kD + c];
            __syncwarp();
            if (lane == 0) mbar_arrive(m.hand_free + 8 * k);
            sync();
            // group of kMergeGroup runs: its last run adds the group's partials
            const int grp = x.run / kMergeGroup;
            const int r0 = grp * kMergeGroup, r1 = min(R, r0 + kMergeGroup);
            unsigned *gt = sa.gtickets + (int64_t)head * sa.groups + grp;
            if (c == 0) *m.mflag = (atom_add_acq_rel_gpu(gt, 1u) == (unsigned)(r1 - r0 - 1)) ? 1u : 0u;
            sync();
            if (!*m.mflag) return;
            {
                const double *q = sa.part + ((int64_t)head * R + r0) * kD + c;
                double v[kMergeGroup];
#pragma unroll
                for (int i = 0; i < kMergeGroup; ++i) v[i] = (r0 + i < r1) ? __ldcg(q + (int64_t)i * kD) : 0.0;
                double gs = 0.0;
#pragma unroll
                for (int i = 0; i < kMergeGroup; ++i) gs = __dadd_rn(gs, v[i]);  // + 0.0 past the group is exact
                sa.gpart[((int64_t)head * sa.groups + grp) * kD + c] = gs;
            }
            if (c == 0) *gt = 0u;  // ready for the next call
            sync();
            if (c == 0) *m.mflag = (atom_add_acq_rel_gpu(sa.tickets + head, 1u) == (unsigned)(sa.groups - 1)) ? 1u : 0u;
            sync();
            if (!*m.mflag) return;
            // last group of the head: channel energy, score, top T, ready flag
            double qv[8];
#pragma unroll
            for (int g = 0; g < 8; ++g) qv[g] = (g < G) ? __ldcg(sa.qn2 + ((int64_t)head * G + g) * kD + c) : 0.0;
            const double *gq = sa.gpart + (int64_t)head * sa.groups * kD + c;
            double k2 = 0.0;
            for (int g0 = 0; g0 < sa.groups; g0 += 24) {
                double v[24];
#pragma unroll
                for (int i = 0; i < 24; ++i) v[i] = (g0 + i < sa.groups) ? __ldcg(gq + (int64_t)(g0 + i) * kD) : 0.0;
#pragma unroll
                for (int i = 0; i < 24; ++i) k2 = __dadd_rn(k2, v[i]);
            }
            const double knorm = sqrt(k2);
            double sc = 0.0;
#pragma unroll
            for (int g = 0; g < 8; ++g)
                if (g < G) sc = __dadd_rn(sc, __dmul_rn(sqrt(qv[g]), knorm));
            sa.scores[(int64_t)head * kD + c] = sc;
            m.sv[c] = __double_as_longlong(sc);
            if (c == 0) sa.tickets[head] = 0u;  // ready for the next call
            sync();
            // top T: rank of channel c in (score descending, index ascending)
            const unsigned long long mine = m.sv[c];
            int rank = 0;
#pragma unroll 8
            for (int c2 = 0; c2 < kD; ++c2) {
                const unsigned long long o = m.sv[c2];
                rank += (o > mine) | ((o == mine) & (c2 < c));
            }
            const bool keep = rank < a.T;
            const unsigned ball = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) m.wcnt[warp] = __popc(ball);
            sync();
            if (keep) {
                int base = 0;
                for (int w = 0; w < warp; ++w) base += m.wcnt[w];
                sa.idx[(int64_t)head * a.T + base + __popc(ball & ((1u << lane) - 1u))] = c;
            }
            sync();
            if (c == 0) st_release_gpu(a.ready + head, 1u);  // after the barrier: every thread's selection
        });
    }
}

// Compact warps (threads 256..511): the kept channels of each tile into K'.
__device__ __forceinline__ void pf_compact(const PruneFusedArgs &a, const PfSmem &m)
{
    const int ctid = threadIdx.x - kPfGroupThreads;
    const int warp = ctid >> 5, lane = ctid & 31;
    const int tb0 = 4 * (warp & 1), cw = warp >> 1;
    const uint32_t c_row = (uint32_t)(8 * (tb0 + (lane >> 3)) + (lane & 7));
    const int stages = a.c_stages;
    const uint64_t pol_store = (a.hints & kPfHintStoreDrop) ? l2_policy_evict_first() : l2_policy_evict_normal();
    int cur_head = -1;
    int64_t crow[4];  // K' row (head * T + t) of my four channels, -1 if dropped
#pragma unroll
    for (int k = 0; k < 4; ++k) crow[k] = -1;
    int n = 0;  // tiles taken
    for (int r = 0; r < a.rounds; ++r) {
        pf_for_each_run(a, r, blockIdx.x, gridDim.x, [&](const PfRun &x) {
            if (x.head != cur_head) {
                // one thread of the block polls the head's flag, then the group
                // reads the selection
                if (ctid == 0) *m.cflag = (!*m.abort && pf_wait_flag(a.ready + x.head, a.sc.status)) ? 1u : 0u;
                named_barrier(1, kPfGroupThreads);
                const bool ok = *m.cflag != 0;
                if (!ok) *m.abort = 1u;
                if (ok) kept_rows_of_warp(a.sc.idx + (int64_t)x.head * a.T, a.T, (int64_t)x.head * a.T, cw, lane, crow);
                cur_head = ok ? x.head : -1;
                named_barrier(1, kPfGroupThreads);  // cflag is read before it is rewritten
            }
            // two tiles per step: both tiles' loads are in flight together
            for (int t = x.t0; t < x.t1; t += 2) {
                const int nt = min(2, x.t1 - t);
                const int n0 = n;
                n += nt;
                if (*m.abort) continue;
                uint32_t v[2][4][4];
                bool ok = true;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i >= nt) break;
                    const int s = (n0 + i) % stages;
                    if (!mbar_wait_bounded(m.full_c + 8 * s, (uint32_t)(((n0 + i) / stages) & 1), a.sc.status,
                                           THINK_DEVICE_TIMEOUT_FULL)) {
                        ok = false;
                        break;
                    }
                    compact_tile_load(m.ring_c + (uint32_t)s * kPfTileBytes, c_row, cw, v[i]);
                }
                if (!ok) {
                    *m.abort = 1u;
                    continue;
                }
                compact_tile_transpose(v[0], lane);  // uses the loaded words: the stages have been read
                if (nt == 2) compact_tile_transpose(v[1], lane);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(m.empty_c + 8 * (n0 % stages));
                    if (nt == 2) mbar_arrive(m.empty_c + 8 * ((n0 + 1) % stages));
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i >= nt) break;
                    const int64_t xo = (int64_t)(t + i) * kPfTile + 8 * (tb0 + (lane & 3));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (crow[k] >= 0 && THINK_IN_RANGE(crow[k] < (int64_t)a.heads * a.T, a.sc.status))
                            store_run8_hint(a.kp + crow[k] * a.ldk, xo, a.N, v[i][k], pol_store);
                }
            }
        });
        // this block has compacted round r (the score producer may go on)
        named_barrier(1, kPfGroupThreads);
        if (ctid == 0) *m.c_done = (unsigned)(r + 1);
    }
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prune_fused_kernel(const __grid_constant__ CUtensorMap tm_k, const PruneFusedArgs a)
{
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *base = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);
    const PfSmem m = pf_smem(a, base);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < a.s_stages; ++s) {
            mbar_init(m.full_s + 8 * s, 1);
            mbar_init(m.empty_s + 8 * s, 8);
        }
        for (int s = 0; s < a.c_stages; ++s) {
            mbar_init(m.full_c + 8 * s, 1);
            mbar_init(m.empty_c + 8 * s, 8);
        }
        for (int k = 0; k < kPfHandSlots; ++k) {
            mbar_init(m.hand_full + 8 * k, kD);
            mbar_init(m.hand_free + 8 * k, kPfMergeThreads / 32);
        }
        *m.abort = 0u;
        *m.c_done = 0u;
        *m.last = 0u;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp < 8) {
        pf_score(a, m);
    } else if (warp < 16) {
        pf_compact(a, m);
    } else if (warp >= kPfWarpMerge0) {
        pf_merge(a, m);
    } else {
        if ((tid & 31) == 0) pf_produce(a, &tm_k, m, warp == kPfWarpScoreProd);
        __syncwarp();
    }
    __syncthreads();  // every role is done (all of their waits are bounded)

    // the last block to finish leaves the ready flags and the exit counter at zero
    if (tid == 0) {
        __threadfence();
        *m.last = (atomicAdd(a.exits, 1u) == gridDim.x - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (*m.last) {
        __threadfence();
        for (int h = tid; h < a.heads; h += kPfThreads) a.ready[h] = 0u;
        if (tid == 0) *a.exits = 0u;
    }
}

}  // namespace think

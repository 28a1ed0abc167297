// prune_fused.cuh -- the whole prune step of one layer (channel scores, top-T
// selection, thinner key cache) for a bf16 key cache in one persistent kernel.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): score every key channel against the query window,
// sort the channels, drop the least relevant ones, keep the thinner key cache.
//
// Scoring needs every token of a head before the head's channels can be
// chosen, so K is read twice: once to score, once to compact.  This kernel
// runs the second read of a head as soon as the head's selection is known, so
// that it can find the head's K still in L2:
//   - Two work queues: score items S(h, i) (channel energies of a run of
//     tokens of head h), in head order, and compact items C(h, j) (K' of a run
//     of tokens), in head order.  A block alternates between them: after a
//     score item it takes the next compact item if the selection of that
//     item's head is ready (else another score item), after a compact item the
//     next score item.  When the score queue is empty it waits (bounded) for
//     the front compact head.
//   - The block that finishes the last score item of head h adds the partials,
//     forms the scores, selects the top T and raises ready[h].  Compact items
//     are only taken for heads that are ready, so no consumer ever waits for
//     another block, and a producer waits only when every score item is
//     already taken (and so will finish).
//   - One block per SM: a producer warp streams 64-token tiles of K (16 KB, two
//     64-channel halves with the 128-byte swizzle) by TMA through a 12-stage
//     ring (score tiles with an L2 keep hint, compact tiles with an evict
//     hint); eight consumer warps either add squares (S) or transpose the tile
//     (C: ldmatrix.trans, then a 4x4 word transpose inside each group of four
//     lanes, so that every lane holds 8 consecutive tokens of one channel) and
//     write the kept channels to K' as 64-byte runs.  Compact tiles need no
//     block barrier: each warp finds the kept channels' rows from a bit mask
//     of the head's selection that it builds itself.
// The scores are those of score_kernel bit for bit (same split plan, same
// per-thread order of additions, same fixed-order merges); the selection is
// select_top_t_warp; K' is a pure copy.  Every wait is bounded; the block
// barriers inside the loop are mbarriers with bounded waits.
#pragma once

#include "prune_kernels.cuh"
#include "think.h"

namespace think {

constexpr int kPfTile = 64;                       // tokens per K tile
constexpr int kPfConsumerWarps = 8;
constexpr int kPfConsumers = 32 * kPfConsumerWarps;
constexpr int kPfThreads = kPfConsumers + 32;     // + one producer warp
constexpr int kPfStages = 12;
constexpr uint32_t kPfHalfBytes = 64u * 64u * 2u;   // 64 tokens x 64 channels x bf16
constexpr uint32_t kPfTileBytes = 2u * kPfHalfBytes;

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kPfRedOff = kPfStages * kPfTileBytes;      // [16][128] fp64
constexpr uint32_t kPfSvOff = kPfRedOff + 16u * kD * 8u;      // [128] score bits
constexpr uint32_t kPfKhalfOff = kPfSvOff + kD * 8u;          // [128] fp64
constexpr uint32_t kPfMetaOff = kPfKhalfOff + kD * 8u;        // [stages] int4
constexpr uint32_t kPfBarOff = kPfMetaOff + kPfStages * 16u;  // full[], empty[], block barrier
constexpr uint32_t kPfFlagOff = kPfBarOff + (2u * kPfStages + 1u) * 8u;
constexpr size_t kPfSmemBytes = kPfFlagOff + 16u + 1024u;     // + alignment slack

enum : int { kPfScore = 0, kPfCompact = 1, kPfStop = 2, kPfFirst = 4, kPfLast = 8 };

struct PruneFusedArgs {
    const __nv_bfloat16 *qwin;    // [B][Hq][S][128]
    int Hq, Hkv, S, G, T;
    int heads, tiles_per_head;
    int s_tiles, s_items;         // tiles per score item, score items per head
    int c_tiles, c_items;         // the same for compact items
    int l2_hints;                 // 1: score loads evict_last, compact loads and K' stores evict_first
    long long s_total;            // heads * s_items
    double *part;                 // [heads][s_items][128] partial channel energies
    double *qn2;                  // [heads][G][128]       window-query energies
    unsigned *tickets;            // [heads] S items done; reset by the finalize
    unsigned *ready;              // [heads] selection written; reset by the last block
    unsigned *status;             // device status word
    unsigned long long *s_next;   // next score item; reset by the last block
    unsigned *c_front;            // head whose compact items are being handed out; reset by the last block
    unsigned *c_cnt;              // [heads] compact items of the head handed out; reset by the last block
    unsigned *exits;              // blocks finished; reset by the last block
    double *scores;               // [heads][128]
    int32_t *idx;                 // [heads][T]
    __nv_bfloat16 *kp;            // K' [heads][T][ldk]
    int64_t ldk, N;
};

struct PfItem {
    int kind, head, part;
};

// Barrier of the consumer warps on an mbarrier (one arrival per warp, after
// the warp's own sync) with a bounded wait.
__device__ __forceinline__ bool pf_bar(uint32_t bar, uint32_t &phase, unsigned *status)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = mbar_wait_bounded(bar, phase, status, THINK_DEVICE_TIMEOUT_BARRIER);
    phase ^= 1u;
    return ok;
}

// Wait (bounded) until another block has raised *flag.
__device__ __forceinline__ bool pf_wait_flag(const unsigned *flag, unsigned *status)
{
    if (ld_acquire_gpu(flag)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t spin = 0; spin < kWaitLimitSpins; ++spin) {
        __nanosleep(128);
        if (ld_acquire_gpu(flag)) return true;
        if ((spin & 31u) == 0u && global_ns() - t0 > kWaitLimitNs) break;
    }
    atomicOr(status, THINK_DEVICE_TIMEOUT_READY);
    return false;
}

__device__ __forceinline__ void pf_item_tiles(const PruneFusedArgs &a, const PfItem &it, int &t0, int &t1)
{
    if (it.kind == kPfScore) {
        t0 = it.part * a.s_tiles;
        t1 = min(a.tiles_per_head, t0 + a.s_tiles);
    } else if (it.kind == kPfCompact) {
        t0 = it.part * a.c_tiles;
        t1 = min(a.tiles_per_head, t0 + a.c_tiles);
    } else {
        t0 = 0;  // one stop marker
        t1 = 1;
    }
}

// Next item for this block.  After a score item (want_c) the next compact
// item of the front compact head if that head's selection is ready, else a
// score item; after a compact item a score item.  With no score item left: the
// next compact item, waiting (bounded) for its head if needed (every score
// item is then taken, so the head's selection will come).  Stop when both
// queues are empty.  Compact items are handed out by a per-head fetch-and-add;
// the front head moves on when its items are gone.
__device__ __forceinline__ PfItem pf_claim(const PruneFusedArgs &a, bool &s_left, bool &want_c)
{
    for (;;) {
        unsigned h = *reinterpret_cast<volatile unsigned *>(a.c_front);
        if (want_c || !s_left) {
            while (h < (unsigned)a.heads && ld_acquire_gpu(a.ready + h)) {
                const unsigned i = atomicAdd(a.c_cnt + h, 1u);
                if (i < (unsigned)a.c_items) {
                    want_c = false;
                    return PfItem{kPfCompact, (int)h, (int)i};
                }
                atomicCAS(a.c_front, h, h + 1u);
                h = *reinterpret_cast<volatile unsigned *>(a.c_front);
            }
        }
        if (s_left) {
            const unsigned long long i = atomicAdd(a.s_next, 1ull);
            if (i < (unsigned long long)a.s_total) {
                want_c = true;
                return PfItem{kPfScore, (int)(i / (unsigned long long)a.s_items),
                              (int)(i % (unsigned long long)a.s_items)};
            }
            s_left = false;
            continue;
        }
        if (h >= (unsigned)a.heads) return PfItem{kPfStop, 0, 0};
        if (!pf_wait_flag(a.ready + h, a.status)) return PfItem{kPfStop, 0, 0};
    }
}

// Producer (one thread): claim items, stream their tiles into the ring.
__device__ __forceinline__ void pf_produce(const PruneFusedArgs &a, const CUtensorMap *tm_k,
                                           uint32_t ring, int4 *meta, uint32_t full0,
                                           uint32_t empty0, volatile unsigned *abort)
{
    prefetch_tensormap(tm_k);
    const uint64_t pol_keep = a.l2_hints ? l2_policy_evict_last() : l2_policy_evict_normal();
    const uint64_t pol_drop = a.l2_hints ? l2_policy_evict_first() : l2_policy_evict_normal();
    long long n = 0;  // tiles and stop markers put into the ring
    bool ok = true, s_left = true, want_c = false;
    for (bool stop = false; !stop && ok;) {
        const PfItem it = pf_claim(a, s_left, want_c);
        stop = it.kind == kPfStop;
        int t0, t1;
        pf_item_tiles(a, it, t0, t1);
        const int b = it.head / a.Hkv, kv = it.head % a.Hkv;
        for (int t = t0; t < t1; ++t) {
            const int s = (int)(n % kPfStages);
            const long long f = n / kPfStages;
            if (*abort || (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)((f - 1) & 1),
                                                       a.status, THINK_DEVICE_TIMEOUT_EMPTY))) {
                ok = false;
                break;
            }
            meta[s] = make_int4(it.kind | (t == t0 ? kPfFirst : 0) | (t == t1 - 1 ? kPfLast : 0),
                                it.head, it.part, t);
            const uint32_t full = full0 + 8 * s;
            if (stop) {
                mbar_arrive(full);
            } else {
                mbar_arrive_expect_tx(full, kPfTileBytes);
                const uint32_t dst = ring + (uint32_t)s * kPfTileBytes;
                const uint64_t pol = it.kind == kPfScore ? pol_keep : pol_drop;
                tma_load_4d_hint(dst, tm_k, 0, t * kPfTile, kv, b, full, pol);
                tma_load_4d_hint(dst + kPfHalfBytes, tm_k, 64, t * kPfTile, kv, b, full, pol);
            }
            ++n;
        }
    }
    if (!ok) {  // let the loads already issued land before the block exits
        for (long long m = n > kPfStages ? n - kPfStages : 0; m < n; ++m)
            mbar_wait_bounded(full0 + 8 * (int)(m % kPfStages), (uint32_t)((m / kPfStages) & 1),
                              a.status, THINK_DEVICE_TIMEOUT_FULL);
    }
}

// End of a score item (all consumer threads): block partial -> part, and the
// last item of the head finalizes it (scores, top-T, ready flag).
__device__ __forceinline__ bool pf_score_item_end(const PruneFusedArgs &a, int head, int part,
                                                  const double (&acc)[8], unsigned char *smem,
                                                  uint32_t bar, uint32_t &phase, unsigned *flags)
{
    const int tid = threadIdx.x;
    const int cc = tid & 15, rg = tid >> 4;
    double *red = reinterpret_cast<double *>(smem + kPfRedOff);
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rg * kD + cc * 8 + e] = acc[e];
    if (!pf_bar(bar, phase, a.status)) return false;
    if (tid < kD) {
        double s = 0.0;
#pragma unroll 4
        for (int rr = 0; rr < 16; ++rr) s += red[rr * kD + tid];
        a.part[((int64_t)head * a.s_items + part) * kD + tid] = s;
        __threadfence();
    }
    if (!pf_bar(bar, phase, a.status)) return false;
    if (tid == 0) flags[1] = (atomicAdd(a.tickets + head, 1u) == (unsigned)(a.s_items - 1)) ? 1u : 0u;
    if (!pf_bar(bar, phase, a.status)) return false;
    if (!flags[1]) return true;

    // ------------------------------------------ last score item of the head
    __threadfence();
    unsigned long long *sv = reinterpret_cast<unsigned long long *>(smem + kPfSvOff);
    double *khalf = reinterpret_cast<double *>(smem + kPfKhalfOff);
    const int c = tid & (kD - 1), hp = tid >> 7;
    double k0 = 0.0;
    {
        const double *p = a.part + (int64_t)head * a.s_items * kD + c;
        for (int s = hp; s < a.s_items; s += 32) {
            double v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int s2 = s + 2 * u;
                v[u] = (s2 < a.s_items) ? __ldcg(p + (int64_t)s2 * kD) : 0.0;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) k0 = __dadd_rn(k0, v[u]);
        }
    }
    if (hp == 1) khalf[c] = k0;
    if (!pf_bar(bar, phase, a.status)) return false;
    if (tid < kD) {
        k0 = __dadd_rn(k0, khalf[tid]);
        const double knorm = sqrt(k0);
        double sc = 0.0;
        for (int g = 0; g < a.G; ++g)
            sc = __dadd_rn(sc, __dmul_rn(sqrt(__ldcg(a.qn2 + ((int64_t)head * a.G + g) * kD + tid)), knorm));
        a.scores[(int64_t)head * kD + tid] = sc;
        sv[tid] = __double_as_longlong(sc);
    }
    if (tid == 0) a.tickets[head] = 0u;  // ready for the next call
    if (!pf_bar(bar, phase, a.status)) return false;
    if (tid < 32) {
        select_top_t_warp(sv, a.T, a.idx + (int64_t)head * a.T, tid);
        __threadfence();
        __syncwarp();
        if (tid == 0) st_release_gpu(a.ready + head, 1u);
    }
    return true;
}

// Window-query energies of query heads g = part, part + s_items, ... of the
// group (threads 0..127, one channel each), as in score_kernel.
__device__ __forceinline__ void pf_window_energies(const PruneFusedArgs &a, int head, int part)
{
    const int tid = threadIdx.x;
    if (tid >= kD) return;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    for (int g = part; g < a.G; g += a.s_items) {
        const int64_t h = (int64_t)kv * a.G + g;
        const __nv_bfloat16 *qh = a.qwin + (((int64_t)b * a.Hq + h) * a.S) * kD + tid;
        a.qn2[((int64_t)head * a.G + g) * kD + tid] = window_energy<__nv_bfloat16>(qh, a.S);
    }
}

__device__ __forceinline__ void pf_consume(const PruneFusedArgs &a, unsigned char *smem, uint32_t full0,
                                           uint32_t empty0, uint32_t bar, unsigned *flags)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t ring = smem_addr(smem);
    const int4 *meta = reinterpret_cast<const int4 *>(smem + kPfMetaOff);
    volatile unsigned *abort = flags;

    // score: this thread's 16-byte chunk (channels 8cc..8cc+7) and row group
    const int cc = tid & 15, rg = tid >> 4;
    const uint32_t s_half = (uint32_t)(cc >> 3) * kPfHalfBytes;
    const uint32_t s_chunk = (uint32_t)(cc & 7);
    // compact: this warp's token half (blocks tb0..tb0+3 of 8 tokens) and its
    // channel chunks cw + 4k (k = 0..3) of 8 channels; this lane's ldmatrix row
    const int tb0 = 4 * (warp & 1), cw = warp >> 1;
    const uint32_t c_row = (uint32_t)(8 * (tb0 + (lane >> 3)) + (lane & 7));

    uint32_t phase = 0;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    int cur_head = -1;
    int64_t crow[4];  // compact: K' row (head * T + t) of my four channels, -1 if dropped
#pragma unroll
    for (int k = 0; k < 4; ++k) crow[k] = -1;

    for (long long k = 0;; ++k) {
        const int s = (int)(k % kPfStages);
        if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((k / kPfStages) & 1), a.status,
                               THINK_DEVICE_TIMEOUT_FULL)) {
            *abort = 1u;
            break;
        }
        const int4 m = meta[s];
        const int kind = m.x & 3;
        if (kind == kPfStop) break;
        const int head = m.y, part = m.z, tile = m.w;
        const uint32_t st = ring + (uint32_t)s * kPfTileBytes;

        if (kind == kPfScore) {
            if (m.x & kPfFirst) {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.0;
                pf_window_energies(a, head, part);
            }
            uint4 w[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const uint32_t row = (uint32_t)(rg + 16 * k4);
                const uint32_t addr = st + s_half + row * 128u + ((s_chunk ^ (row & 7u)) << 4);
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[k4].x), "=r"(w[k4].y), "=r"(w[k4].z), "=r"(w[k4].w)
                             : "r"(addr)
                             : "memory");
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
            add_squares4_bf16(w, acc);
            if ((m.x & kPfLast) && !pf_score_item_end(a, head, part, acc, smem, bar, phase, flags)) {
                *abort = 1u;
                break;
            }
        } else {
            if (head != cur_head) {
                // kept-channel rows of the head (every warp builds its own)
                if (lane == 0) (void)ld_acquire_gpu(a.ready + head);
                __syncwarp();
                kept_rows_of_warp(a.idx + (int64_t)head * a.T, a.T, (int64_t)head * a.T, cw, lane, crow);
                cur_head = head;
            }
            uint32_t v[4][4];
            compact_tile_load(st, c_row, cw, v);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
            compact_tile_store(v, lane, crow, a.kp, a.ldk, (int64_t)tile * kPfTile + 8 * (tb0 + (lane & 3)), a.N);
        }
    }

}

__global__ void __launch_bounds__(kPfThreads, 1)
    prune_fused_kernel(const __grid_constant__ CUtensorMap tm_k, const PruneFusedArgs a)
{
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);
    int4 *meta = reinterpret_cast<int4 *>(smem + kPfMetaOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kPfBarOff);
    unsigned *flags = reinterpret_cast<unsigned *>(smem + kPfFlagOff);  // abort, last-of-head, last block
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = full0 + 8u * kPfStages;
    const uint32_t bar = empty0 + 8u * kPfStages;

    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kPfConsumerWarps);
        }
        mbar_init(bar, kPfConsumerWarps);
        flags[0] = flags[1] = flags[2] = 0u;
        fence_barrier_init();
    }
    __syncthreads();

    if (tid >= kPfConsumers) {
        if (tid == kPfConsumers) pf_produce(a, &tm_k, smem_addr(smem), meta, full0, empty0, flags);
        __syncwarp();
    } else {
        pf_consume(a, smem, full0, empty0, bar, flags);
    }
    __syncthreads();  // every role is done (all of their waits are bounded)

    // the last block to finish leaves the list counter and the flags at zero
    if (tid == 0) {
        __threadfence();
        flags[2] = (atomicAdd(a.exits, 1u) == gridDim.x - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (flags[2]) {
        __threadfence();
        for (int h = tid; h < a.heads; h += kPfThreads) {
            a.ready[h] = 0u;
            a.c_cnt[h] = 0u;
        }
        if (tid == 0) {
            *a.s_next = 0ull;
            *a.c_front = 0u;
            *a.exits = 0u;
        }
    }
}

}  // namespace think

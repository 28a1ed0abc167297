// prune_kernels.cuh -- channel scoring, top-T selection and key compaction.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): rate each key channel's relevance to the query,
// sort the channels, drop the least relevant ones, keep a thinner key cache.
#pragma once

#include "ptx.cuh"

namespace think {

// Top-T of the kD channel scores held in shared memory, by one warp:
// rank(c) = #channels before c in the order (score descending, index
// ascending); c is kept if rank(c) < T; kept channels are written ascending.
// Scores are non-negative doubles, whose bit patterns order like their values.
__device__ __forceinline__ void select_top_t_warp(const unsigned long long *sv, int T,
                                                  int32_t *__restrict__ idx_out, int lane)
{
    unsigned long long mine[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) mine[j] = sv[lane + 32 * j];
    int base = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = lane + 32 * j;
        int rank = 0;
#pragma unroll 8
        for (int c2 = 0; c2 < kD; ++c2) {
            const unsigned long long u = sv[c2];
            rank += (u > mine[j]) | ((u == mine[j]) & (c2 < c));
        }
        const bool keep = rank < T;
        const unsigned ball = __ballot_sync(0xffffffffu, keep);
        if (keep) idx_out[base + __popc(ball & ((1u << lane) - 1u))] = c;
        base += __popc(ball);
    }
}

// Barrier policies of the score merge: the whole block, or the 256 consumer
// threads of a warp-specialised block whose producer warp keeps running.
struct BlockSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct ConsumerSync {
    __device__ __forceinline__ void operator()() const { named_barrier(1, 256); }
};

// The same selection (same rule, same output) by the first 256 threads of a
// block; every thread taking part in `sync` calls it.  Thread t ranks channel
// t/2 against half t%2 of the channels and the pair adds its two counts, so
// each thread makes 64 comparisons instead of 512.  wcnt: 8 ints of shared
// memory.
template <typename Sync>
__device__ __forceinline__ void select_top_t_block(const unsigned long long *sv, int T,
                                                   int32_t *__restrict__ idx_out, int *wcnt, Sync sync)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool on = tid < 2 * kD;
    const int c = (tid >> 1) & (kD - 1), h = tid & 1;
    int rank = 0;
    if (on) {
        const unsigned long long mine = sv[c];
#pragma unroll 8
        for (int j = 0; j < kD / 2; ++j) {
            const int c2 = h * (kD / 2) + j;
            const unsigned long long u = sv[c2];
            rank += (u > mine) | ((u == mine) & (c2 < c));
        }
    }
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    const bool keep = on && h == 0 && rank < T;
    const unsigned ball = __ballot_sync(0xffffffffu, keep);
    if (on && lane == 0) wcnt[warp] = __popc(ball);
    sync();
    if (keep) {
        int base = 0;
        for (int w = 0; w < warp; ++w) base += wcnt[w];
        idx_out[base + __popc(ball & ((1u << lane) - 1u))] = c;
    }
}

// Window-query energy of one channel: sum over s of q[s][c]^2 in fp64, in row
// order; q points at the channel's element of row 0, rows kD apart.  The loads
// go out 32 at a time (the sum itself is sequential), so that the blocks that
// compute these energies start streaming keys soon after the others.
template <typename TIn>
__device__ __forceinline__ double window_energy(const TIn *q, int S)
{
    double q2 = 0.0;
    int s = 0;
    for (; s + 32 <= S; s += 32) {
        float x[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) x[u] = Elem<TIn>::to_float(q[(int64_t)(s + u) * kD]);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const double xd = (double)x[u];
            q2 = __dadd_rn(q2, __dmul_rn(xd, xd));
        }
    }
    for (; s + 8 <= S; s += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = Elem<TIn>::to_float(q[(int64_t)(s + u) * kD]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const double xd = (double)x[u];
            q2 = __dadd_rn(q2, __dmul_rn(xd, xd));
        }
    }
    for (; s < S; ++s) {
        const double x = (double)Elem<TIn>::to_float(q[(int64_t)s * kD]);
        q2 = __dadd_rn(q2, __dmul_rn(x, x));
    }
    return q2;
}

struct ScoreArgs {
    const void *k;
    int64_t sb, sh, sn;        // element strides of K (batch, head, token)
    const void *qwin;          // [B][Hq][S][D]
    int Hq, Hkv, S;
    int64_t N, rows_per_split;
    int splits;
    double *part;              // [heads][splits][D]   partial channel energies of the runs
    double *gpart;             // [heads][groups][D]   sums of groups of kMergeGroup runs
    double *qn2;               // [heads][G][D]        window-query channel energies
    unsigned *gtickets;        // [heads][groups] runs of the group done; zero between calls
    unsigned *tickets;         // [heads] groups of the head done; zero between calls
    int groups;                // ceil(splits / kMergeGroup)
    double *scores;            // [heads][D]
    int T;                     // > 0: also select the top T into idx
    int32_t *idx;              // [heads][T]
    unsigned *status;          // device status word (bounded waits of score_tma_kernel)
    int stages;                // score_tma_kernel: ring stages
};

// ---------------------------------------------------------------------------
// Score.  Block (split, head) sums K[n,c]^2 over its run of tokens with
// 16-byte loads (bf16: 16 threads x 8 channels per row, 16 rows per pass, 8
// passes in flight); blocks split < G also sum the window-query energies of
// query head kv*G + split.  The last block of the head to finish (ticket
// counter) adds the partials in a fixed order (even and odd splits in two
// halves of the block, then the halves) and forms
//     s[c] = sum_g sqrt(qn2[g][c]) * sqrt(kn2[c])
// with each operation rounded as written, then optionally selects the top T.
// fp32 keys: every square is exact in fp64 and only the order of the fp64
// additions differs from a sequential sum.  bf16 keys: four-row fp32 partials
// (add_squares4_bf16), then fp64.  The order of all additions is fixed by the
// split plan, so the result is deterministic.
// ---------------------------------------------------------------------------
// fp32 keys: the square of an fp32 value is exact in fp64; one FMA per element.
__device__ __forceinline__ void add_squares_f32(const uint4 &w, double *acc)
{
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const double x = (double)__uint_as_float(ww[e]);
        acc[e] = fma(x, x, acc[e]);
    }
}

// bf16: the squares of one thread's four rows of a 64-token tile (rows r,
// r+16, r+32, r+48; 8 channels each) are added in fp32 (FFMA2 on channel
// pairs; each product is exact, three roundings of at most 2^-24 relative),
// then the four-term partial of each channel is added to its fp64 running sum.
// So every channel energy carries a relative error below 3 * 2^-24 = 1.8e-7,
// for keys of magnitude in [2^-63, 2^64) (outside it the fp32 square
// underflows or overflows).  Rows past the end of the keys are passed as zero
// words, which add nothing.
__device__ __forceinline__ void add_squares4_bf16(const uint4 (&w)[4], double *acc)
{
    float2 p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = make_float2(__uint_as_float(ww[e] << 16), __uint_as_float(ww[e] & 0xffff0000u));
            p[e] = __ffma2_rn(x, x, p[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)p[e].x;
        acc[2 * e + 1] += (double)p[e].y;
    }
}

// Window-query energies of the group's query heads g = split, split +
// splits, ... (threads 0..127, one channel each): qn2[g][c] = sum_s q[s,c]^2
// in fp64, in token order.
template <typename TIn>
__device__ __forceinline__ void score_window_energies(const ScoreArgs &a, int head, int split)
{
    const int tid = threadIdx.x;
    if (tid >= kD) return;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int G = a.Hq / a.Hkv;
    for (int g = split; g < G; g += a.splits) {
        const int64_t h = (int64_t)kv * G + g;
        const TIn *qh = static_cast<const TIn *>(a.qwin) + (((int64_t)b * a.Hq + h) * a.S) * kD + tid;
        a.qn2[((int64_t)head * G + g) * kD + tid] = window_energy<TIn>(qh, a.S);
    }
}

// Runs of a head merged by one block before the head's total is formed.
constexpr int kMergeGroup = 16;

// End of a score run (called by every thread taking part in `sync`; threads
// 0..255 do the work).  The run's partial part[head][split][c] is the sum of
// the ROWS rows of red[][c] in row order.  The partials are then added in a
// fixed two-level order: the last block of each group of kMergeGroup runs
// (group ticket) adds the group's partials in run order into gpart; the last
// group of the head (head ticket) adds the group sums in group order, forms
//     s[c] = sum_g sqrt(qn2[g][c]) * sqrt(kn2[c])
// with each operation rounded as written, resets the tickets and, for T > 0,
// selects the top T.  Every sum starts at 0 and runs in ascending order, so
// the result depends only on the split plan.  Shared memory: flag (1 word), sv
// (kD words), wcnt (8 ints).  Returns true (uniformly) in the block that
// formed the head's scores.
template <int ROWS, typename Sync>
__device__ __forceinline__ bool score_run_end(const ScoreArgs &a, int head, int split, const double *red,
                                              unsigned *flag, unsigned long long *sv, int *wcnt, Sync sync)
{
    const int tid = threadIdx.x;
    const int G = a.Hq / a.Hkv;
    if (tid < kD) {
        double s = 0.0;
#pragma unroll 4
        for (int rr = 0; rr < ROWS; ++rr) s += red[rr * kD + tid];
        if (THINK_IN_RANGE(split < a.splits, a.status))
            a.part[((int64_t)head * a.splits + split) * kD + tid] = s;
    }
    __threadfence();
    sync();
    const int grp = split / kMergeGroup;
    const int r0 = grp * kMergeGroup, r1 = min(a.splits, r0 + kMergeGroup);
    unsigned *gt = a.gtickets + (int64_t)head * a.groups + grp;
    if (tid == 0) *flag = (atomicAdd(gt, 1u) == (unsigned)(r1 - r0 - 1)) ? 1u : 0u;
    sync();
    if (!*flag) return false;

    // ------------------------------------------ last run of the group
    __threadfence();
    if (tid < kD) {
        const double *p = a.part + ((int64_t)head * a.splits + r0) * kD + tid;
        double v[kMergeGroup];
#pragma unroll
        for (int u = 0; u < kMergeGroup; ++u) v[u] = (r0 + u < r1) ? __ldcg(p + (int64_t)u * kD) : 0.0;
        double s = 0.0;
#pragma unroll
        for (int u = 0; u < kMergeGroup; ++u) s = __dadd_rn(s, v[u]);  // + 0.0 past the group is exact
        if (THINK_IN_RANGE(grp < a.groups, a.status)) a.gpart[((int64_t)head * a.groups + grp) * kD + tid] = s;
    }
    if (tid == 0) *gt = 0u;  // ready for the next call
    __threadfence();
    sync();
    if (tid == 0) *flag = (atomicAdd(a.tickets + head, 1u) == (unsigned)(a.groups - 1)) ? 1u : 0u;
    sync();
    if (!*flag) return false;

    // ------------------------------------------ last group of the head
    __threadfence();
    if (tid < kD) {
        const double *p = a.gpart + (int64_t)head * a.groups * kD + tid;
        double k2 = 0.0;
        for (int g0 = 0; g0 < a.groups; g0 += 16) {
            double v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (g0 + u < a.groups) ? __ldcg(p + (int64_t)(g0 + u) * kD) : 0.0;
#pragma unroll
            for (int u = 0; u < 16; ++u) k2 = __dadd_rn(k2, v[u]);
        }
        const double knorm = sqrt(k2);
        double sc = 0.0;
        for (int g = 0; g < G; ++g)
            sc = __dadd_rn(sc, __dmul_rn(sqrt(__ldcg(a.qn2 + ((int64_t)head * G + g) * kD + tid)), knorm));
        a.scores[(int64_t)head * kD + tid] = sc;
        sv[tid] = __double_as_longlong(sc);
    }
    if (tid == 0) a.tickets[head] = 0u;  // ready for the next call
    if (a.T > 0) {
        sync();
        select_top_t_block(sv, a.T, a.idx + (int64_t)head * a.T, wcnt, sync);
    }
    return true;
}

// score_run_end for the score kernels (the whole block takes part).
template <int ROWS>
__device__ __forceinline__ void score_block_end(const ScoreArgs &a, int head, int split, const double *red)
{
    __shared__ unsigned flag;
    __shared__ unsigned long long sv[kD];
    __shared__ int wcnt[8];
    (void)score_run_end<ROWS>(a, head, split, red, &flag, sv, wcnt, BlockSync{});
}

template <typename TIn>
__global__ void __launch_bounds__(256, 3) score_kernel(const ScoreArgs a)
{
    constexpr int VEC = 16 / sizeof(TIn);  // channels per 16-byte load
    constexpr int TPR = kD / VEC;          // threads per row
    constexpr int RPP = 256 / TPR;         // rows per pass
    constexpr int UNROLL = 4;              // 16-byte loads per batch (two batches in flight)
    __shared__ double red[RPP][kD];

    const int head = blockIdx.y;
    const int split = blockIdx.x;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int tid = threadIdx.x;
    const int cg = tid % TPR;
    const int r = tid / TPR;
    const int64_t n0 = (int64_t)split * a.rows_per_split;
    const int64_t n1 = min(a.N, n0 + a.rows_per_split);
    const TIn *base = static_cast<const TIn *>(a.k) + (int64_t)b * a.sb + (int64_t)kv * a.sh + cg * VEC;

    score_window_energies<TIn>(a, head, split);

    double acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
    // Software pipeline: the loads of the next batch of UNROLL rows are issued
    // before the squares of the current batch are added, so about 2 * UNROLL
    // 16-byte loads per thread stay in flight.
    int64_t n = n0 + r;
    const int64_t step = (int64_t)RPP * UNROLL;
    uint4 cur[UNROLL];
    bool have = n + (int64_t)(UNROLL - 1) * RPP < n1;
    if (have) {
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
            cur[u] = __ldg(reinterpret_cast<const uint4 *>(base + (n + (int64_t)u * RPP) * a.sn));
    }
    while (have) {
        const int64_t nn = n + step;
        const bool have_next = nn + (int64_t)(UNROLL - 1) * RPP < n1;
        uint4 nxt[UNROLL];
        if (have_next) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                nxt[u] = __ldg(reinterpret_cast<const uint4 *>(base + (nn + (int64_t)u * RPP) * a.sn));
        }
        if constexpr (sizeof(TIn) == 2) {
            add_squares4_bf16(cur, acc);
        } else {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) add_squares_f32(cur[u], acc);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) cur[u] = nxt[u];
        n = nn;
        have = have_next;
    }
    if constexpr (sizeof(TIn) == 2) {
        if (n < n1) {  // the rows of the last, partial tile
#pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                cur[u] = (n + (int64_t)u * RPP < n1)
                             ? __ldg(reinterpret_cast<const uint4 *>(base + (n + (int64_t)u * RPP) * a.sn))
                             : make_uint4(0u, 0u, 0u, 0u);
            add_squares4_bf16(cur, acc);
        }
    } else {
        for (; n < n1; n += RPP) add_squares_f32(__ldg(reinterpret_cast<const uint4 *>(base + n * a.sn)), acc);
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[r][cg * VEC + e] = acc[e];
    __syncthreads();
    score_block_end<RPP>(a, head, split, &red[0][0]);
}

// ---------------------------------------------------------------------------
// Select (stand-alone): one warp per head.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    select_kernel(const double *__restrict__ scores, int heads, int T, int32_t *__restrict__ idx)
{
    __shared__ unsigned long long sv[4][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x * 4 + warp;
    if (head >= heads) return;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        sv[warp][lane + 32 * j] = __double_as_longlong(scores[(int64_t)head * kD + lane + 32 * j]);
    __syncwarp();
    select_top_t_warp(sv[warp], T, idx + (int64_t)head * T, lane);
}

// ---------------------------------------------------------------------------
// Adaptive kept width (ThinK method section, key design 3: the pruning ratio
// adapts to the query and the cache).  One block does every head: a warp per
// head ranks the channels (score descending, index ascending; scores are
// non-negative doubles, ordered by their bits), and lane 0 adds the squared
// scores in rank order (fp64, each product and sum rounded as written) to
// find the shortest prefix holding tau of the total:
//     T_h = min { k in [T_min, T_max] : cum_k >= tau * E }, else T_max;
//     T_h = T_min when E == 0.
// The padded widths (multiples of 16) are then scanned into the heads' first
// rows, and the kept channels are written ascending at idx[rowoff[h] ..].
// ---------------------------------------------------------------------------
__device__ __forceinline__ int rank_of(const unsigned long long *sv, unsigned long long mine, int c)
{
    int rank = 0;
#pragma unroll 8
    for (int c2 = 0; c2 < kD; ++c2) {
        const unsigned long long u = sv[c2];
        rank += (u > mine) | ((u == mine) & (c2 < c));
    }
    return rank;
}

__global__ void __launch_bounds__(1024)
    select_adaptive_kernel(const double *__restrict__ scores, int heads, double tau, int T_min, int T_max,
                           int32_t *__restrict__ Th, int32_t *__restrict__ rowoff, int32_t *__restrict__ idx)
{
    __shared__ unsigned long long sv[32][kD];
    __shared__ unsigned char order[32][kD];   // channel at each rank
    __shared__ int32_t wsum[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- widths
    for (int h = warp; h < heads; h += 32) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            sv[warp][lane + 32 * j] = __double_as_longlong(scores[(int64_t)h * kD + lane + 32 * j]);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = lane + 32 * j;
            order[warp][rank_of(sv[warp], sv[warp][c], c)] = (unsigned char)c;
        }
        __syncwarp();
        if (lane == 0) {
            double E = 0.0;
            for (int i = 0; i < kD; ++i) {
                const double x = __longlong_as_double(sv[warp][order[warp][i]]);
                E = __dadd_rn(E, __dmul_rn(x, x));
            }
            int T = T_max;
            if (E == 0.0) {
                T = T_min;
            } else {
                const double target = __dmul_rn(tau, E);
                double cum = 0.0;
                for (int k = 1; k <= T_max; ++k) {
                    const double x = __longlong_as_double(sv[warp][order[warp][k - 1]]);
                    cum = __dadd_rn(cum, __dmul_rn(x, x));
                    if (k >= T_min && cum >= target) {
                        T = k;
                        break;
                    }
                }
            }
            Th[h] = T;
        }
        __syncwarp();
    }
    __syncthreads();

    // ---- first rows: exclusive scan of the padded widths over the heads
    const int per = (heads + 1023) / 1024;
    const int h0 = min(heads, (int)threadIdx.x * per), h1 = min(heads, h0 + per);
    int32_t local = 0;
    for (int h = h0; h < h1; ++h) local += (Th[h] + 15) & ~15;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;  // inclusive sums over warps
    }
    __syncthreads();
    int32_t run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
    for (int h = h0; h < h1; ++h) {
        rowoff[h] = run;
        run += (Th[h] + 15) & ~15;
    }
    if (threadIdx.x == 1023) rowoff[heads] = run;
    __syncthreads();

    // ---- kept channels, ascending
    for (int h = warp; h < heads; h += 32) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            sv[warp][lane + 32 * j] = __double_as_longlong(scores[(int64_t)h * kD + lane + 32 * j]);
        __syncwarp();
        const int T = Th[h];
        int base = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = lane + 32 * j;
            const bool keep = rank_of(sv[warp], sv[warp][c], c) < T;
            const unsigned ball = __ballot_sync(0xffffffffu, keep);
            if (keep) idx[rowoff[h] + base + __popc(ball & ((1u << lane) - 1u))] = c;
            base += __popc(ball);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// Compact: K'^T[t][col0 + n] = K[n][idx[t]] for a tile of 64 tokens of one
// head (col0 = 0 for a whole cache, the current length when new tokens'
// keys are appended).
// Each thread loads a 4-token x 8-channel block (four 16-byte loads, one per
// token row), regroups it in registers into 8 channel runs of 4 tokens, and
// stores those transposed into shared memory (channel-major, padded pitch).
// Every kept channel is then one contiguous run of tokens, copied out with
// 16-byte stores.  A pure copy: bit-exact.
// ---------------------------------------------------------------------------
template <typename TIn> struct Transpose4;
// bf16: four 16-byte rows (tokens) of 8 channels -> 8 channel runs of 4 tokens (8 bytes)
template <> struct Transpose4<__nv_bfloat16> {
    static constexpr int CH = 8;
    static __device__ __forceinline__ void run(const uint4 w[4], uint2 out[CH])
    {
        const uint32_t r[4][4] = {{w[0].x, w[0].y, w[0].z, w[0].w}, {w[1].x, w[1].y, w[1].z, w[1].w},
                                  {w[2].x, w[2].y, w[2].z, w[2].w}, {w[3].x, w[3].y, w[3].z, w[3].w}};
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // channel pair (2i, 2i+1)
            out[2 * i] = make_uint2(__byte_perm(r[0][i], r[1][i], 0x5410), __byte_perm(r[2][i], r[3][i], 0x5410));
            out[2 * i + 1] = make_uint2(__byte_perm(r[0][i], r[1][i], 0x7632), __byte_perm(r[2][i], r[3][i], 0x7632));
        }
    }
};
// fp32: four 16-byte rows (tokens) of 4 channels -> 4 channel runs of 4 tokens (16 bytes)
template <> struct Transpose4<float> {
    static constexpr int CH = 4;
    static __device__ __forceinline__ void run(const uint4 w[4], uint4 out[CH])
    {
        out[0] = make_uint4(w[0].x, w[1].x, w[2].x, w[3].x);
        out[1] = make_uint4(w[0].y, w[1].y, w[2].y, w[3].y);
        out[2] = make_uint4(w[0].z, w[1].z, w[2].z, w[3].z);
        out[3] = make_uint4(w[0].w, w[1].w, w[2].w, w[3].w);
    }
};

// ---------------------------------------------------------------------------
// Compaction of one 64-token K tile held in shared memory as two 64-channel
// halves with the 128-byte swizzle (as TMA writes them), by the 8 warps of a
// block: warp w takes the token half tb0 = 4 * (w % 2) (token blocks tb0 ..
// tb0 + 3 of 8 tokens) and the channel chunks cw + 4k (k = 0..3, 8 channels
// each) with cw = w / 2.  ldmatrix.trans gives each lane two tokens of one
// channel per register; a word transpose inside each group of four lanes then
// gives lane j of the group 8 consecutive tokens of its channel, which go to
// the channel's K' row as one 16-byte store (64 bytes per group of four).
// ---------------------------------------------------------------------------
// 4x4 transpose of 32-bit words inside each group of four lanes: lane j of
// the group ends with word j of every lane of the group, in lane order.
__device__ __forceinline__ void quad_transpose(uint32_t (&a)[4], int j)
{
    const bool o1 = j & 1, o2 = j & 2;
    uint32_t t0 = o1 ? a[0] : a[1], t1 = o1 ? a[2] : a[3];
    t0 = __shfl_xor_sync(0xffffffffu, t0, 1);
    t1 = __shfl_xor_sync(0xffffffffu, t1, 1);
    if (o1) {
        a[0] = t0;
        a[2] = t1;
    } else {
        a[1] = t0;
        a[3] = t1;
    }
    uint32_t u0 = o2 ? a[0] : a[2], u1 = o2 ? a[1] : a[3];
    u0 = __shfl_xor_sync(0xffffffffu, u0, 2);
    u1 = __shfl_xor_sync(0xffffffffu, u1, 2);
    if (o2) {
        a[0] = u0;
        a[1] = u1;
    } else {
        a[2] = u0;
        a[3] = u1;
    }
}

// 8 consecutive tokens of one K' row starting at token x (x a multiple of 8);
// only tokens < N are written.
__device__ __forceinline__ void store_run8(__nv_bfloat16 *row, int64_t x, int64_t N, const uint32_t (&v)[4])
{
    if (x + 8 <= N) {
        *reinterpret_cast<uint4 *>(row + x) = make_uint4(v[0], v[1], v[2], v[3]);
    } else if (x < N) {
        unsigned short *r = reinterpret_cast<unsigned short *>(row + x);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (x + i < N) r[i] = (unsigned short)(v[i >> 1] >> (16 * (i & 1)));
    }
}

// K' rows of this warp's four channel chunks: crow[k] = row0 + rank of
// channel 8 * (cw + 4k) + lane / 4 among the kept channels, or -1 if the
// channel is dropped.  idx holds the T kept channels of the head.
__device__ __forceinline__ void kept_rows_of_warp(const int32_t *idx, int T, int64_t row0, int cw, int lane,
                                                  int64_t (&crow)[4])
{
    uint32_t mk[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = lane + 32 * i;
        if (t < T) {
            const int c = __ldcg(idx + t);
            if ((unsigned)c < (unsigned)kD) {
                const uint32_t bitv = 1u << (c & 31);
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) mk[wd] |= (c >> 5) == wd ? bitv : 0u;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) mk[i] = __reduce_or_sync(0xffffffffu, mk[i]);
    // channel 8*(cw+4k) + lane/4 lies in mask word k (k = c / 32)
    int before = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int bit = (8 * cw + (lane >> 2)) & 31;
        crow[k] = ((mk[k] >> bit) & 1u) ? row0 + before + __popc(mk[k] & ((1u << bit) - 1u)) : -1;
        before += __popc(mk[k]);
    }
}

// The warp's part of the tile at shared address st into registers: register m
// of load k holds channel 8 * (cw + 4k) + lane / 4, tokens 8 * (tb0 + m) +
// 2 * (lane % 4) + {0, 1}; c_row = 8 * (tb0 + lane / 8) + lane % 8 is the
// token row this lane addresses.
__device__ __forceinline__ void compact_tile_load(uint32_t st, uint32_t c_row, int cw, uint32_t (&v)[4][4])
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t chunk = (uint32_t)(cw + 4 * k);
        const uint32_t addr = st + (chunk >> 3) * (64u * 64u * 2u) + c_row * 128u + (((chunk & 7u) ^ (c_row & 7u)) << 4);
        ldsm_x4_trans(addr, v[k][0], v[k][1], v[k][2], v[k][3]);
    }
}

// The 4x4 word transposes of a loaded tile part: afterwards register m of
// v[k] holds tokens 2m, 2m + 1 of this lane's 8-token run of its channel.
__device__ __forceinline__ void compact_tile_transpose(uint32_t (&v)[4][4], int lane)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) quad_transpose(v[k], lane & 3);
}

// Store the kept channels' runs: x = first token of this lane's run (a
// multiple of 8).
__device__ __forceinline__ void compact_tile_store_kept(const uint32_t (&v)[4][4], const int64_t (&crow)[4],
                                                        __nv_bfloat16 *kp, int64_t ldk, int64_t x, int64_t N)
{
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (crow[k] >= 0) store_run8(kp + crow[k] * ldk, x, N, v[k]);
}

template <typename TIn> struct CompactTokens { static constexpr int value = 64; };

template <typename TIn>
__global__ void __launch_bounds__(256)
    compact_kernel(const TIn *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int Hkv, int64_t N,
                   const int32_t *__restrict__ idx, int T, TIn *__restrict__ kp, int64_t ldk, int64_t col0,
                   const int32_t *__restrict__ Th, const int32_t *__restrict__ rowoff)
{
    constexpr int BNC = CompactTokens<TIn>::value;  // tokens per block
    constexpr int VEC = 16 / sizeof(TIn);         // elements per 16 bytes (channels per load)
    constexpr int PITCH = BNC + VEC;              // padded smem row, elements (16-byte multiple)
    constexpr int CGROUPS = kD / VEC;             // channel groups of one row: 16 (bf16), 32 (fp32)
    constexpr int TGROUPS = 256 / CGROUPS;        // token groups of 4 per pass: 16 (bf16), 8 (fp32)
    constexpr int PASSES = BNC / (4 * TGROUPS);   // 1 (bf16), 2 (fp32)
    constexpr int LPR = BNC / VEC;                // lanes per output row
    constexpr int RPI = 32 / LPR;                 // output rows per warp instruction
    using Run = typename std::conditional<sizeof(TIn) == 2, uint2, uint4>::type;
    __shared__ __align__(16) TIn sT[kD][PITCH];

    const int head = blockIdx.y;
    const int b = head / Hkv, h = head % Hkv;
    const int64_t n0 = (int64_t)blockIdx.x * BNC;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // lane -> (token group, channel group); the 16 lanes of a half-warp cover
    // 16 token groups of one channel group, so their shared stores form one
    // contiguous 128-byte run per channel.
    const int tg = (CGROUPS == 16) ? (lane & 15) : (lane & 7);
    const int cgi = (CGROUPS == 16) ? (warp * 2 + (lane >> 4)) : (warp * 4 + (lane >> 3));
    const TIn *kh = k + (int64_t)b * sb + (int64_t)h * sh + cgi * VEC;

    uint4 w[PASSES][4];  // every load of the block is issued before the first is used
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int row0 = (pass * TGROUPS + tg) * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t n = n0 + row0 + i;
            w[pass][i] = (n < N) ? __ldg(reinterpret_cast<const uint4 *>(kh + n * sn)) : make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const int row0 = (pass * TGROUPS + tg) * 4;
        Run runs[Transpose4<TIn>::CH];
        Transpose4<TIn>::run(w[pass], runs);
#pragma unroll
        for (int c = 0; c < Transpose4<TIn>::CH; ++c)
            *reinterpret_cast<Run *>(&sT[cgi * VEC + c][row0]) = runs[c];
    }
    __syncthreads();

    const int seg = lane % LPR;
    const int tok = seg * VEC;
    const bool vec_ok = (col0 % VEC) == 0;  // 16-byte aligned output runs
    // ragged (Th set): this head keeps Th[head] rows from rowoff[head], then
    // zero rows up to a multiple of 16
    const int Tk = Th ? min(max(Th[head], 0), T) : T;
    const int Tw = Th ? ((Tk + 15) & ~15) : T;
    const int64_t r0 = Th ? (int64_t)rowoff[head] : (int64_t)head * T;
    if (Th && (r0 < 0 || r0 + Tw > (int64_t)gridDim.y * ((T + 15) & ~15))) return;  // not from the selection
    for (int t = warp * RPI + lane / LPR; t < Tw; t += 8 * RPI) {
        const int c = t < Tk ? idx[r0 + t] : -1;
        uint4 val = make_uint4(0, 0, 0, 0);
        if ((unsigned)c < (unsigned)kD) val = *reinterpret_cast<const uint4 *>(&sT[c][tok]);
        TIn *out = kp + (r0 + t) * ldk + col0 + n0 + tok;
        if (vec_ok && n0 + tok + VEC <= N) {
            *reinterpret_cast<uint4 *>(out) = val;
        } else {
            const TIn *e = reinterpret_cast<const TIn *>(&val);
            for (int i = 0; i < VEC; ++i)
                if (n0 + tok + i < N) out[i] = e[i];
        }
    }
}

}  // namespace think

// evict.cuh -- token eviction by observation-window attention mass, to be
// composed with the channel pruning (the prune then runs on the kept tokens).
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", abstract and
// experiments: ThinK is compared with and combined with KV-cache eviction;
// the Keyformer page keeps the "key tokens" that receive the most attention.
// Reading used here, for each (b, h_kv) and cached token n:
//     mass[n] = sum over the group's query heads g and window rows s of
//               softmax_n( scale * Qwin[b,g,s,:] . K[b,h_kv,n,:] )
// and each head keeps the M tokens of largest mass (ties to the lower index),
// in ascending order.
//
// The mass is an attention of R = G * S_obs query rows over the N keys,
// computed in two passes on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate): pass 1 the row statistics (max and sum of exponentials,
// per split, merged by the last block of the head), pass 2 the column sums of
// the normalised weights.  K streams through a TMA ring as 128-token tiles
// (two 64-channel halves, 128-byte swizzle); the window queries stay in
// shared memory (same swizzle) for the whole block.
#pragma once

#include "decode_mma.cuh"

namespace think {

constexpr int kMassWarps = 8;
constexpr int kMassThreads = kMassWarps * 32 + 32;  // + TMA producer warp
constexpr int kMassRowsMax = 512;                   // G * S_obs

struct MassArgs {
    const __nv_bfloat16 *qwin;  // [B][Hq][S][128]
    int Hq, Hkv, S, G, R, r_pad;  // R = G * S rows; r_pad = 8 * kMassWarps * NTW >= R
    int64_t N;
    int tiles_per_split, splits, stages;
    float scale_log2;           // scale * log2(e)
    float2 *part;               // [heads][splits][R] (max, sum) of each split (pass 1)
    float2 *stats;              // [heads][R] (max, 1 / sum) (written by pass 1, read by pass 2)
    unsigned *tickets;          // [heads], zero between calls
    unsigned *status;           // device status word
    float *mass;                // [heads][N] (pass 2)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// shared memory: stages x K tile (32 KB), the window queries (two 64-channel
// halves of r_pad rows x 128 B), pass 2's row statistics and per-warp token
// sums, barriers, a flag
__host__ __device__ inline size_t mass_smem_bytes(int r_pad, int stages)
{
    return (size_t)stages * 32768u + (size_t)2 * r_pad * 128u + (size_t)r_pad * 8u +
           (size_t)kMassWarps * kBN * 4u + (size_t)2 * stages * 8u + 16u + 1024u;
}

// Pass 1's end: the block's per-row (max, sum) partials are in a.part; the
// head's last block (ticket) merges the splits in split order into
// (max, 1 / sum) per row.  NT threads (tid < NT) take part, barrier 1.
template <int NT>
__device__ __forceinline__ void mass_merge_splits(const MassArgs &a, int head, int tid, unsigned *flag)
{
    __threadfence();
    named_barrier(1, NT);
    if (tid == 0) *flag = (atomicAdd(a.tickets + head, 1u) == (unsigned)(a.splits - 1)) ? 1u : 0u;
    named_barrier(1, NT);
    if (*flag == 0u) return;
    __threadfence();
    for (int r = tid; r < a.R; r += NT) {
        float M = -INFINITY;
        for (int s = 0; s < a.splits; ++s) M = fmaxf(M, __ldcg(a.part + ((int64_t)head * a.splits + s) * a.R + r).x);
        float L = 0.f;
        for (int s = 0; s < a.splits; ++s) {
            const float2 p = __ldcg(a.part + ((int64_t)head * a.splits + s) * a.R + r);
            if (p.x != -INFINITY) L = fmaf(p.y, exp2_approx(p.x - M), L);
        }
        a.stats[(int64_t)head * a.R + r] = make_float2(M, L > 0.f ? 1.f / L : 0.f);
    }
    if (tid == 0) a.tickets[head] = 0u;
}

// NTW: 8-row query groups per warp (r_pad = 64 * NTW).  With NTW <= 4 a warp
// keeps the B fragments of its rows in registers for the whole block.
template <int PASS, int NTW>
__global__ void __launch_bounds__(kMassThreads)
    token_mass_kernel(const __grid_constant__ CUtensorMap tm_k, const MassArgs a)
{
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);
    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int stages = a.stages;
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);
    const uint32_t q_half = (uint32_t)a.r_pad * 128u;

    unsigned char *qs = smem + (size_t)stages * 32768u;                 // queries, swizzled
    float2 *rstat = reinterpret_cast<float2 *>(qs + 2u * q_half);        // [r_pad] (max, 1/sum)
    float *tsum = reinterpret_cast<float *>(rstat + a.r_pad);            // [warps][128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(tsum + kMassWarps * kBN);
    unsigned *flag = reinterpret_cast<unsigned *>(bars + 2 * stages);
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + stages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kMassWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kMassWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            int issued = 0;
            bool ok = true;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % stages, f = it / stages;
                if (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (f - 1) & 1, a.status,
                                                THINK_DEVICE_TIMEOUT_EMPTY)) {
                    ok = false;
                    break;
                }
                const uint32_t full = full0 + 8 * s;
                mbar_arrive_expect_tx(full, 32768u);
                const int x = (int)((tile0 + it) * kBN);
                const uint32_t st = smem_addr(smem + (size_t)s * 32768u);
                tma_load_4d(st, &tm_k, 0, x, kv, b, full);
                tma_load_4d(st + 16384u, &tm_k, 64, x, kv, b, full);
                ++issued;
            }
            if (!ok) {
                for (int it = max(0, issued - stages); it < issued; ++it)
                    mbar_wait_bounded(full0 + 8 * (it % stages), (it / stages) & 1, a.status,
                                      THINK_DEVICE_TIMEOUT_FULL);
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    constexpr int NT = kMassWarps * 32;
    // the window queries of the group, row r = g * S + s (rows >= R zero), in
    // two 64-channel halves with the 128-byte swizzle
    for (int i = tid; i < a.r_pad * 16; i += NT) {
        const int r = i >> 4, c16 = i & 15;  // row, 16-byte chunk (8 channels)
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < a.R) {
            const int g = r / a.S, s = r % a.S;
            v = *reinterpret_cast<const uint4 *>(
                a.qwin + (((int64_t)b * a.Hq + (int64_t)kv * a.G + g) * a.S + s) * kD + 8 * c16);
        }
        *reinterpret_cast<uint4 *>(qs + (c16 >> 3) * q_half + (uint32_t)r * 128u +
                                   ((((uint32_t)c16 & 7u) ^ ((uint32_t)r & 7u)) << 4)) = v;
    }
    if (PASS == 2) {
        for (int r = tid; r < a.r_pad; r += NT)
            rstat[r] = r < a.R ? __ldcg(a.stats + (int64_t)head * a.R + r) : make_float2(0.f, 0.f);
    }
    named_barrier(1, NT);

    const int q4 = lane & 3, r8 = lane >> 2;
    const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix index, row within it
    const uint32_t qbase = smem_addr(qs);
    constexpr bool kBRegs = NTW <= 4;
    // B fragments (k = channel, n = query row) of the warp's row groups
    // warp, warp + 8, ...: two registers per 16-channel step
    uint32_t bq[kBRegs ? NTW : 1][8][2];
    if (kBRegs) {
#pragma unroll
        for (int j = 0; j < (kBRegs ? NTW : 1); ++j) {
            const uint32_t n = (uint32_t)(8 * (warp + kMassWarps * j) + rr);
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                const uint32_t chunk = (uint32_t)(4 * kp + mi);
                ldsm_x4(qbase + (chunk >> 3) * q_half + n * 128u + (((chunk & 7u) ^ (n & 7u)) << 4),
                        bq[j][2 * kp][0], bq[j][2 * kp][1], bq[j][2 * kp + 1][0], bq[j][2 * kp + 1][1]);
            }
        }
    }
    // pass 1: this lane's running (max, sum of 2^(z - max)) over the tokens it
    // sees, for the 2 rows of each of its row groups
    float rm[NTW][2], rl[NTW][2];
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rm[j][h] = -INFINITY;
            rl[j][h] = 0.f;
        }

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (it / stages) & 1, a.status, THINK_DEVICE_TIMEOUT_FULL)) break;
        const uint32_t kb = smem_addr(smem + (size_t)s * 32768u);
        const int64_t tok0 = (tile0 + it) * kBN;
#pragma unroll 1
        for (int mt = 0; mt < 8; ++mt) {
            // A fragments: tokens 16 mt .. +15, all 8 channel steps
            uint32_t af[8][4];
            const uint32_t tok = (uint32_t)(16 * mt + (mi & 1) * 8 + rr);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t chunk = (uint32_t)(2 * ks + (mi >> 1));
                ldsm_x4(kb + (chunk >> 3) * 16384u + tok * 128u + (((chunk & 7u) ^ (tok & 7u)) << 4), af[ks][0],
                        af[ks][1], af[ks][2], af[ks][3]);
            }
            const bool v0 = tok0 + 16 * mt + r8 < a.N, v1 = tok0 + 16 * mt + 8 + r8 < a.N;
            float tacc[2] = {0.f, 0.f};  // pass 2: this lane's sums for tokens 16 mt + r8, + 8
#pragma unroll
            for (int j = 0; j < NTW; ++j) {
                const int nt = warp + kMassWarps * j;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                if (kBRegs) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        wmma16::mma_bf16(c, af[ks][0], af[ks][1], af[ks][2], af[ks][3], bq[kBRegs ? j : 0][ks][0],
                                         bq[kBRegs ? j : 0][ks][1]);
                } else {
                    const uint32_t n = (uint32_t)(8 * nt + rr);
#pragma unroll
                    for (int kp = 0; kp < 4; ++kp) {
                        uint32_t b0, b1, b2, b3;
                        const uint32_t chunk = (uint32_t)(4 * kp + mi);
                        ldsm_x4(qbase + (chunk >> 3) * q_half + n * 128u + (((chunk & 7u) ^ (n & 7u)) << 4), b0,
                                b1, b2, b3);
                        wmma16::mma_bf16(c, af[2 * kp][0], af[2 * kp][1], af[2 * kp][2], af[2 * kp][3], b0, b1);
                        wmma16::mma_bf16(c, af[2 * kp + 1][0], af[2 * kp + 1][1], af[2 * kp + 1][2],
                                         af[2 * kp + 1][3], b2, b3);
                    }
                }
                // c[0], c[1]: token 16 mt + r8, rows 8 nt + 2 q4 (+1); c[2], c[3]: token + 8
                if (PASS == 1) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float z0 = v0 ? c[h] * a.scale_log2 : -INFINITY;
                        const float z1 = v1 ? c[2 + h] * a.scale_log2 : -INFINITY;
                        const float mnew = fmaxf(rm[j][h], fmaxf(z0, z1));
                        const float mref = mnew == -INFINITY ? 0.f : mnew;
                        rl[j][h] = rl[j][h] * exp2_approx(rm[j][h] - mref) + exp2_approx(z0 - mref) +
                                   exp2_approx(z1 - mref);
                        rm[j][h] = mnew;
                    }
                } else {
                    const float2 s0 = rstat[8 * nt + 2 * q4], s1 = rstat[8 * nt + 2 * q4 + 1];
                    tacc[0] += exp2_approx(c[0] * a.scale_log2 - s0.x) * s0.y +
                               exp2_approx(c[1] * a.scale_log2 - s1.x) * s1.y;
                    tacc[1] += exp2_approx(c[2] * a.scale_log2 - s0.x) * s0.y +
                               exp2_approx(c[3] * a.scale_log2 - s1.x) * s1.y;
                }
            }
            if (PASS == 2) {
                // the warp's rows for these 16 tokens (the 4 lanes of a token)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float x = tacc[h];
                    x += __shfl_xor_sync(0xffffffffu, x, 1);
                    x += __shfl_xor_sync(0xffffffffu, x, 2);
                    if (q4 == 0) tsum[warp * kBN + 16 * mt + 8 * h + r8] = x;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (PASS == 2) {
            // the warps' row groups in order: the tile's masses
            named_barrier(1, NT);
            if (tid < kBN && tok0 + tid < a.N) {
                float m = 0.f;
#pragma unroll
                for (int w = 0; w < kMassWarps; ++w) m += tsum[w * kBN + tid];
                a.mass[(int64_t)head * a.N + tok0 + tid] = m;
            }
            named_barrier(1, NT);
        }
    }
    if constexpr (PASS == 1) {
        // ---- pass 1: the block's row statistics, then the last block of the head merges
#pragma unroll
        for (int j = 0; j < NTW; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // merge the 8 lanes that saw the other tokens of these rows
                float m = rm[j][h], l = rl[j][h];
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
                    const float mm = fmaxf(m, mo);
                    const float mref = mm == -INFINITY ? 0.f : mm;
                    l = l * exp2_approx(m - mref) + lo * exp2_approx(mo - mref);
                    m = mm;
                }
                const int r = 8 * (warp + kMassWarps * j) + 2 * q4 + h;
                if (r8 == 0 && r < a.R)
                    a.part[((int64_t)head * a.splits + split) * a.R + r] = make_float2(m, l);
            }
        mass_merge_splits<NT>(a, head, tid, flag);
    }
}

// ---------------------------------------------------------------------------
// Top-M tokens of each head by mass: the M-th largest key K* (masses are
// non-negative floats, whose bit patterns order like their values), then
// every token with key > K* and the lowest-indexed `ties` tokens with key ==
// K*, written ascending.  Spread over the whole GPU: each head's keys are cut
// into chunks of 256 * kpt keys (a block per chunk and head, kpt consecutive
// keys per thread), and
//   select_hist_kernel<P> (P = 0..3): a radix pass on the 8-bit digit P from
//     the top: each block replays passes 0..P-1 from the global histograms
//     (the same digit choice in every block), then adds its chunk's keys that
//     match the prefix so far into hist[P][head];
//   select_count_kernel: replays all four passes (K*, ties) and counts each
//     chunk's keys above K* and equal to K*;
//   select_write_kernel: each chunk's first output position from the counts of
//     the chunks before it, then the chunk's kept tokens in index order (two
//     block scans).
// Workspace: hist [4][heads][256], sel [heads][2], cnt [heads][chunks][2]
// (int32); hist is zero between calls (pass 0 clears hist[1..3] of the
// previous call, the write kernel clears hist[0]).
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 256;

struct SelectArgs {
    const float *mass;  // [heads][N]
    int64_t N;
    int M, kpt, chunks;
    int *hist;          // [4][heads][256]
    int *sel;           // [heads][2]: K* bits, ties
    int *cnt;           // [heads][chunks][2]: keys > K*, keys == K*
    int32_t *kept;      // [heads][M]
    int heads;
};

// A thread's keys are handled in batches of kSelBatch consecutive keys, every
// load of a batch issued before the first is used (kpt is a multiple of it).
constexpr int kSelBatch = 16;

__device__ __forceinline__ void select_load_batch(const uint32_t *key, int64_t n, int64_t N,
                                                  uint32_t (&kk)[kSelBatch], unsigned &valid)
{
    valid = 0u;
#pragma unroll
    for (int e = 0; e < kSelBatch; ++e) {
        const bool in = n + e < N;
        kk[e] = in ? __ldcg(key + n + e) : 0u;
        valid |= in ? (1u << e) : 0u;
    }
}

// Radix digit choice of one pass (warp 0; h = the pass's 256-bin histogram in
// shared memory): the largest digit dg with sum_{d >= dg} h[d] >= need (else
// 0), and need minus the keys of the digits above dg.  Lane l holds bins
// 255 - 8l down to 248 - 8l.
__device__ __forceinline__ void select_pick_digit(const int *h, int lane, int &need, int &dg)
{
    int v[8], s = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        v[e] = h[255 - 8 * lane - e];
        s += v[e];
    }
    int cum = s;  // inclusive over lanes 0..lane (the higher digits first)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, cum >= need);
    int d = 0, left = need;
    if (hit) {
        const int L = __ffs(hit) - 1;
        const int before = __shfl_sync(0xffffffffu, cum - s, L);  // keys of the lanes before L
        int run = before, pick = 0, rest = need - before;
        bool found = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int ve = __shfl_sync(0xffffffffu, v[e], L);
            if (!found) {
                if (run + ve >= need) {
                    pick = 255 - 8 * L - e;
                    rest = need - run;
                    found = true;
                } else {
                    run += ve;
                }
            }
        }
        d = pick;
        left = rest;
    } else {
        // fewer matching keys than need (not reached for 1 <= M <= N): digit 0
        // after every higher digit, as a sequential scan would end
        d = 0;
        left = need - (__shfl_sync(0xffffffffu, cum, 31) - h[0]);
    }
    dg = d;
    need = left;
}

// Replay passes 0..P-1 of this head: prefix and mask of the digits chosen so
// far and the keys still to take among those matching them.  Every thread
// of the block calls it; sh: 256 shared ints; sv: 3 shared ints.
__device__ __forceinline__ void select_replay(const SelectArgs &a, int head, int P, int *sh, int *sv,
                                              uint32_t &prefix, uint32_t &mask, int &need)
{
    const int tid = threadIdx.x;
    if (tid == 0) {
        sv[0] = 0;
        sv[1] = 0;
        sv[2] = a.M;
    }
    __syncthreads();
    for (int p = 0; p < P; ++p) {
        sh[tid] = a.hist[((int64_t)p * a.heads + head) * 256 + tid];
        __syncthreads();
        if (tid < 32) {
            int nd = sv[2], dg;
            select_pick_digit(sh, tid, nd, dg);
            if (tid == 0) {
                const int shift = 24 - 8 * p;
                sv[0] = (int)((uint32_t)sv[0] | ((uint32_t)dg << shift));
                sv[1] = (int)((uint32_t)sv[1] | (255u << shift));
                sv[2] = nd;
            }
        }
        __syncthreads();
    }
    prefix = (uint32_t)sv[0];
    mask = (uint32_t)sv[1];
    need = sv[2];
}

template <int P>
__global__ void __launch_bounds__(kSelThreads) select_hist_kernel(const SelectArgs a)
{
    __shared__ int sh[256];
    __shared__ int hloc[256];
    __shared__ int sv[3];
    const int head = blockIdx.y, tid = threadIdx.x;
    uint32_t prefix, mask;
    int need;
    select_replay(a, head, P, sh, sv, prefix, mask, need);
    if (P == 0 && blockIdx.x == 0) {  // the previous call's passes 1..3
        for (int p = 1; p < 4; ++p) a.hist[((int64_t)p * a.heads + head) * 256 + tid] = 0;
    }
    hloc[tid] = 0;
    __syncthreads();
    const int shift = 24 - 8 * P;
    const uint32_t *key = reinterpret_cast<const uint32_t *>(a.mass + (int64_t)head * a.N);
    const int64_t n0 = (int64_t)blockIdx.x * kSelThreads * a.kpt + (int64_t)tid * a.kpt;
    for (int e0 = 0; e0 < a.kpt; e0 += kSelBatch) {
        uint32_t kk[kSelBatch];
        unsigned valid;
        select_load_batch(key, n0 + e0, a.N, kk, valid);
#pragma unroll
        for (int e = 0; e < kSelBatch; ++e)
            if (((valid >> e) & 1u) && (kk[e] & mask) == prefix) atomicAdd(&hloc[(kk[e] >> shift) & 255u], 1);
    }
    __syncthreads();
    if (hloc[tid]) atomicAdd(a.hist + ((int64_t)P * a.heads + head) * 256 + tid, hloc[tid]);
}

__global__ void __launch_bounds__(kSelThreads) select_count_kernel(const SelectArgs a)
{
    __shared__ int sh[256];
    __shared__ int sv[3];
    __shared__ int red[2][kSelThreads / 32];
    const int head = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kth, mask;
    int ties;
    select_replay(a, head, 4, sh, sv, kth, mask, ties);
    const uint32_t *key = reinterpret_cast<const uint32_t *>(a.mass + (int64_t)head * a.N);
    const int64_t n0 = (int64_t)blockIdx.x * kSelThreads * a.kpt + (int64_t)tid * a.kpt;
    int gt = 0, eq = 0;
    for (int e0 = 0; e0 < a.kpt; e0 += kSelBatch) {
        uint32_t kk[kSelBatch];
        unsigned valid;
        select_load_batch(key, n0 + e0, a.N, kk, valid);
#pragma unroll
        for (int e = 0; e < kSelBatch; ++e) {
            const bool in = (valid >> e) & 1u;
            gt += in && kk[e] > kth;
            eq += in && kk[e] == kth;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
        red[0][warp] = gt;
        red[1][warp] = eq;
    }
    __syncthreads();
    if (tid == 0) {
        int g = 0, q = 0;
        for (int w = 0; w < kSelThreads / 32; ++w) {
            g += red[0][w];
            q += red[1][w];
        }
        a.cnt[((int64_t)head * a.chunks + blockIdx.x) * 2] = g;
        a.cnt[((int64_t)head * a.chunks + blockIdx.x) * 2 + 1] = q;
        if (blockIdx.x == 0) {
            a.sel[head * 2] = (int)kth;
            a.sel[head * 2 + 1] = ties;
        }
    }
}

// Exclusive scan of one int per thread over the block (256 threads).
__device__ __forceinline__ int select_block_scan(int x, int *wsum, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const int ws = wsum[w];
        before += w < warp ? ws : 0;
        total += ws;
    }
    __syncthreads();
    return before + incl - x;
}

__global__ void __launch_bounds__(kSelThreads) select_write_kernel(const SelectArgs a)
{
    __shared__ int wsum[kSelThreads / 32];
    __shared__ int red[2][kSelThreads / 32];
    const int head = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const uint32_t kth = (uint32_t)a.sel[head * 2];
    const int ties = a.sel[head * 2 + 1];
    // keys > K* and == K* in the chunks before this one
    int gb = 0, qb = 0;
    for (int j = tid; j < c; j += kSelThreads) {
        gb += a.cnt[((int64_t)head * a.chunks + j) * 2];
        qb += a.cnt[((int64_t)head * a.chunks + j) * 2 + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gb += __shfl_xor_sync(0xffffffffu, gb, o);
        qb += __shfl_xor_sync(0xffffffffu, qb, o);
    }
    if (lane == 0) {
        red[0][warp] = gb;
        red[1][warp] = qb;
    }
    __syncthreads();
    gb = qb = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        gb += red[0][w];
        qb += red[1][w];
    }
    // every count-kernel block has replayed hist[0] of this head: leave it zero
    // (passes 1..3 are cleared by the next call's pass 0)
    if (c == 0) a.hist[(int64_t)head * 256 + tid] = 0;
    const uint32_t *key = reinterpret_cast<const uint32_t *>(a.mass + (int64_t)head * a.N);
    const int64_t n0 = (int64_t)c * kSelThreads * a.kpt + (int64_t)tid * a.kpt;
    // this thread's keys equal to K*, ranked over the chunk in index order
    // (the usual kpt = kSelBatch: one batch, loaded once and kept in registers)
    uint32_t kk[kSelBatch];
    unsigned valid;
    select_load_batch(key, n0, a.N, kk, valid);
    int myeq = 0, mygt = 0;
    for (int e0 = 0; e0 < a.kpt; e0 += kSelBatch) {
        if (e0 > 0) select_load_batch(key, n0 + e0, a.N, kk, valid);
#pragma unroll
        for (int e = 0; e < kSelBatch; ++e) {
            const bool in = (valid >> e) & 1u;
            myeq += in && kk[e] == kth;
            mygt += in && kk[e] > kth;
        }
    }
    int eq_tot;
    const int eq_rank0 = qb + select_block_scan(myeq, wsum, eq_tot);
    // kept: every key above K*, and the keys equal to K* of rank < ties
    const int mykeep = mygt + max(0, min(ties - eq_rank0, myeq));
    int keep_tot;
    int pos = gb + min(qb, ties) + select_block_scan(mykeep, wsum, keep_tot);
    int r = eq_rank0;
    for (int e0 = 0; e0 < a.kpt; e0 += kSelBatch) {
        if (e0 > 0 || a.kpt > kSelBatch) select_load_batch(key, n0 + e0, a.N, kk, valid);
#pragma unroll
        for (int e = 0; e < kSelBatch; ++e) {
            if (!((valid >> e) & 1u)) continue;
            const bool keep = kk[e] > kth || (kk[e] == kth && r++ < ties);
            if (keep && pos < a.M) a.kept[(int64_t)head * a.M + pos++] = (int32_t)(n0 + e0 + e);
        }
    }
}

// ---------------------------------------------------------------------------
// Gather the kept tokens' rows: out[b,h,j,:] = x[b,h,kept[b,h,j],:] (a copy).
// A warp per row (16-byte lanes).
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(256)
    gather_tokens_kernel(const TIn *__restrict__ x, int64_t sb, int64_t sh, int64_t sn, int Hkv, int M,
                         const int32_t *__restrict__ kept, int64_t N, TIn *__restrict__ out)
{
    constexpr int VEC = 16 / sizeof(TIn);
    constexpr int LANES = kD / VEC;  // 16 (bf16) or 32 (fp32) lanes per row
    const int64_t row = (int64_t)blockIdx.x * (256 / LANES) + threadIdx.x / LANES;
    const int head = blockIdx.y;
    if (row >= M) return;
    const int b = head / Hkv, h = head % Hkv;
    const int n = kept[(int64_t)head * M + row];
    const int c = (threadIdx.x % LANES) * VEC;
    uint4 v = make_uint4(0, 0, 0, 0);
    if ((unsigned)n < (unsigned)N) v = *reinterpret_cast<const uint4 *>(x + (int64_t)b * sb + (int64_t)h * sh + (int64_t)n * sn + c);
    *reinterpret_cast<uint4 *>(out + ((int64_t)head * M + row) * kD + c) = v;
}

}  // namespace think

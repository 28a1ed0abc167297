// prune_kernels.cuh -- channel scoring, top-T selection and key compaction.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): rate each key channel's relevance to the query,
// sort the channels, drop the least relevant ones, keep a thinner key cache.
#pragma once

#include "ptx.cuh"

namespace think {

// ---------------------------------------------------------------------------
// Score, stage 1: per (split of the token axis, head) partial channel energy
//   part[head][split][c] = sum_{n in split} K[n,c]^2   (fp64)
// 16-byte loads, 256 threads: for bf16 a row (256 B) is 16 threads x 8
// channels and a pass covers 16 rows.  The square of a bf16 or fp32 value is
// exact in fp64, so every product below is exact and only the order of the
// additions differs from a sequential sum.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(256)
    score_partial_kernel(const TIn *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int Hkv,
                         int64_t N, int64_t rows_per_split, int splits,
                         double *__restrict__ part)
{
    constexpr int VEC = 16 / sizeof(TIn);  // channels per 16-byte load
    constexpr int TPR = kD / VEC;          // threads per row
    constexpr int RPP = 256 / TPR;         // rows per pass
    constexpr int UNROLL = 4;
    __shared__ double red[RPP][kD];

    const int head = blockIdx.y;
    const int split = blockIdx.x;
    const int b = head / Hkv, h = head % Hkv;
    const int cg = threadIdx.x % TPR;
    const int r = threadIdx.x / TPR;
    const int64_t n0 = (int64_t)split * rows_per_split;
    const int64_t n1 = min(N, n0 + rows_per_split);
    const TIn *base = k + (int64_t)b * sb + (int64_t)h * sh + cg * VEC;

    double acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.0;

    for (int64_t n = n0 + r; n < n1; n += (int64_t)RPP * UNROLL) {
        uint4 w[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t nn = n + (int64_t)u * RPP;
            w[u] = (nn < n1) ? __ldg(reinterpret_cast<const uint4 *>(base + nn * sn))
                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
            if constexpr (sizeof(TIn) == 2) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const double lo = (double)bf16lo(ww[e]);
                    const double hi = (double)bf16hi(ww[e]);
                    acc[2 * e] = fma(lo, lo, acc[2 * e]);
                    acc[2 * e + 1] = fma(hi, hi, acc[2 * e + 1]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const double x = (double)__uint_as_float(ww[e]);
                    acc[e] = fma(x, x, acc[e]);
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[r][cg * VEC + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < kD) {
        double s = 0.0;
#pragma unroll 4
        for (int rr = 0; rr < RPP; ++rr) s += red[rr][threadIdx.x];
        part[((int64_t)head * splits + split) * kD + threadIdx.x] = s;
    }
}

// ---------------------------------------------------------------------------
// Score, stage 2: one block per head, one thread per channel.
//   kn2 = sum over splits (fixed order);  qn2_g = sum_s Qwin_g[s,c]^2
//   s[c] = sum_g sqrt(qn2_g) * sqrt(kn2)     (each step rounded as written)
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kD)
    score_finalize_kernel(const double *__restrict__ part, int splits, const TIn *__restrict__ qwin,
                          int Hq, int Hkv, int S, double *__restrict__ scores)
{
    const int head = blockIdx.x;
    const int c = threadIdx.x;
    const int b = head / Hkv, kv = head % Hkv;
    const int G = Hq / Hkv;
    double kn2 = 0.0;
    for (int s = 0; s < splits; ++s) kn2 = __dadd_rn(kn2, part[((int64_t)head * splits + s) * kD + c]);
    const double knorm = sqrt(kn2);
    double sc = 0.0;
    for (int g = 0; g < G; ++g) {
        const int64_t h = (int64_t)kv * G + g;
        const TIn *qh = qwin + (((int64_t)b * Hq + h) * S) * kD + c;
        double qn2 = 0.0;
        for (int s = 0; s < S; ++s) {
            const double x = (double)Elem<TIn>::to_float(qh[(int64_t)s * kD]);
            qn2 = __dadd_rn(qn2, __dmul_rn(x, x));
        }
        sc = __dadd_rn(sc, __dmul_rn(sqrt(qn2), knorm));
    }
    scores[(int64_t)head * kD + c] = sc;
}

// ---------------------------------------------------------------------------
// Select: one warp per head.  Rank of channel c = number of channels that come
// before it in the order (score descending, index ascending); c is kept if
// its rank is below T.  Scores are non-negative doubles, whose bit patterns
// order like their values, so the comparison is done on the 64-bit patterns.
// The kept channels are written in ascending channel order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    select_kernel(const double *__restrict__ scores, int heads, int T, int32_t *__restrict__ idx)
{
    __shared__ unsigned long long sv[4][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x * 4 + warp;
    if (head >= heads) return;
    unsigned long long mine[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        mine[j] = __double_as_longlong(scores[(int64_t)head * kD + lane + 32 * j]);
        sv[warp][lane + 32 * j] = mine[j];
    }
    __syncwarp();
    int base = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = lane + 32 * j;
        int rank = 0;
#pragma unroll 8
        for (int c2 = 0; c2 < kD; ++c2) {
            const unsigned long long u = sv[warp][c2];
            rank += (u > mine[j]) | ((u == mine[j]) & (c2 < c));
        }
        const bool keep = rank < T;
        const unsigned ball = __ballot_sync(0xffffffffu, keep);
        if (keep) idx[(int64_t)head * T + base + __popc(ball & ((1u << lane) - 1u))] = c;
        base += __popc(ball);
    }
}

// ---------------------------------------------------------------------------
// Compact: K'^T[t][n] = K[n][idx[t]] for a tile of 64 tokens of one head.
// The tile is read with 16-byte loads (each lane a 32- or 64-byte run of one
// row) and written transposed into shared memory (channel-major, padded
// pitch), so every kept channel is then one contiguous 16-byte-vector run of
// tokens both in shared memory and in the output.  A pure copy: bit-exact.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(256)
    compact_kernel(const TIn *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int Hkv, int64_t N,
                   const int32_t *__restrict__ idx, int T, TIn *__restrict__ kp, int64_t ldk)
{
    constexpr int BNC = 64;                       // tokens per block
    constexpr int VEC = 16 / sizeof(TIn);         // elements per 16 bytes
    constexpr int PITCH = BNC + VEC;              // padded smem row (16-byte multiple)
    constexpr int CPW = kD / 8;                   // channels per warp (16)
    constexpr int LOADS = CPW / VEC;              // 16-byte loads per lane per row
    constexpr int LPR = BNC / VEC;                // lanes per output row
    constexpr int RPI = 32 / LPR;                 // output rows per warp instruction
    __shared__ __align__(16) TIn sT[kD][PITCH];

    const int head = blockIdx.y;
    const int b = head / Hkv, h = head % Hkv;
    const int64_t n0 = (int64_t)blockIdx.x * BNC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TIn *kh = k + (int64_t)b * sb + (int64_t)h * sh + warp * CPW;

    uint4 w[2][LOADS];
#pragma unroll
    for (int rg = 0; rg < 2; ++rg) {
        const int64_t n = n0 + rg * 32 + lane;
#pragma unroll
        for (int q = 0; q < LOADS; ++q)
            w[rg][q] = (n < N) ? __ldg(reinterpret_cast<const uint4 *>(kh + n * sn + q * VEC))
                               : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int rg = 0; rg < 2; ++rg) {
        const int row = rg * 32 + lane;
#pragma unroll
        for (int q = 0; q < LOADS; ++q) {
            const TIn *e = reinterpret_cast<const TIn *>(&w[rg][q]);
#pragma unroll
            for (int i = 0; i < VEC; ++i) sT[warp * CPW + q * VEC + i][row] = e[i];
        }
    }
    __syncthreads();

    const int seg = lane % LPR;
    const int tok = seg * VEC;
    for (int t = warp * RPI + lane / LPR; t < T; t += 8 * RPI) {
        const int c = idx[(int64_t)head * T + t];
        uint4 val = make_uint4(0, 0, 0, 0);
        if ((unsigned)c < (unsigned)kD) val = *reinterpret_cast<const uint4 *>(&sT[c][tok]);
        TIn *out = kp + ((int64_t)head * T + t) * ldk + n0 + tok;
        if (n0 + tok + VEC <= N) {
            *reinterpret_cast<uint4 *>(out) = val;
        } else {
            const TIn *e = reinterpret_cast<const TIn *>(&val);
            for (int i = 0; i < VEC; ++i)
                if (n0 + tok + i < N) out[i] = e[i];
        }
    }
}

}  // namespace think

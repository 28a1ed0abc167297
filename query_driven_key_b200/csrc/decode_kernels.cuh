// decode_kernels.cuh -- decode attention with the thinner key cache.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework, last step): run inference with the pruned cache.
// For query head h of KV head h/G:  z[n] = scale * q[idx] . K'[:,n],
// out = softmax(z) V, with V at full width.
//
// Split-N flash decoding.  Block (split, head) streams its run of 128-token
// tiles of K'^T ([T][128]) and V ([128][128]) through a ring of shared-memory
// stages filled by TMA (one elected producer thread, mbarrier completion), and
// four consumer warps each own 32 tokens of every tile with their own running
// (max, sum, weighted V) per query head of the group.  The block merges its
// four warps and writes one partial per (head, split, group member); the
// combine kernel merges the splits.  Every mbarrier wait is bounded in time.
#pragma once

#include "ptx.cuh"
#include "think.h"

namespace think {

constexpr int kBN = 128;                  // tokens per tile
constexpr int kConsumerWarps = 4;         // kConsumerWarps * 32 == kBN
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
static_assert(kConsumerWarps * 32 == kBN, "one token per consumer lane per tile");

struct DecodeArgs {
    const void *q;          // [B][Hq][D]
    const int32_t *idx;     // [B][Hkv][T]
    float *part_o;          // [heads][splits][G][D]
    float *part_ml;         // [heads][splits][G][2]  (running max in log2 units, sum)
    unsigned *status;       // device status bits
    int Hq, Hkv, T;
    int64_t N;
    int tiles_per_split, splits, stages;
    float scale_log2;       // scale * log2(e)
    uint32_t stage_bytes;   // bytes per ring stage (multiple of 1024)
    uint32_t v_off;         // offset of the V tile inside a stage
    uint32_t tx_bytes;      // bytes one stage's two TMA loads deliver
};

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename TIn, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    pruned_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a)
{
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int T = a.T;
    const int stages = a.stages;
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);

    float *qs = reinterpret_cast<float *>(smem + (size_t)stages * a.stage_bytes);  // [T][G]
    const int qs_len = ((T * G + 3) / 4) * 4;
    float *pbuf = qs + qs_len;                                                   // [warps][32][G]
    uint64_t *bars = reinterpret_cast<uint64_t *>(pbuf + kConsumerWarps * 32 * G);
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + stages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kConsumerWarps);
        }
        fence_barrier_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    // q' = q[idx] for the G query heads of this KV head, pre-scaled to log2 units.
    {
        const TIn *q = reinterpret_cast<const TIn *>(a.q);
        const int32_t *ih = a.idx + (int64_t)head * T;
        for (int i = tid; i < T * G; i += kDecodeThreads) {
            const int t = i / G, g = i % G;
            const int c = ih[t];
            float x = 0.f;
            if ((unsigned)c < (unsigned)kD)
                x = Elem<TIn>::to_float(q[((int64_t)b * a.Hq + (int64_t)kv * G + g) * kD + c]);
            qs[i] = x * a.scale_log2;
        }
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
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
                mbar_arrive_expect_tx(full, a.tx_bytes);
                const int x = (int)((tile0 + it) * kBN);
                unsigned char *st = smem + (size_t)s * a.stage_bytes;
                tma_load_4d(smem_addr(st), &tm_k, x, 0, kv, b, full);
                tma_load_4d(smem_addr(st + a.v_off), &tm_v, 0, x, kv, b, full);
                ++issued;
            }
            if (!ok) {
                // Let the loads already in flight land before the block exits.
                for (int it = max(0, issued - stages); it < issued; ++it)
                    mbar_wait_bounded(full0 + 8 * (it % stages), (it / stages) & 1, a.status,
                                      THINK_DEVICE_TIMEOUT_FULL);
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    float m[G], l[G], acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;
    }
    const int j = warp * 32 + lane;  // this lane's token inside a tile
    float *pw = pbuf + warp * 32 * G;

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (it / stages) & 1, a.status,
                               THINK_DEVICE_TIMEOUT_FULL))
            break;
        const unsigned char *st = smem + (size_t)s * a.stage_bytes;
        const TIn *kt = reinterpret_cast<const TIn *>(st);
        const TIn *vt = reinterpret_cast<const TIn *>(st + a.v_off);
        const bool valid = (tile0 + it) * kBN + j < a.N;

        // logits of this lane's token for the G heads of the group
        float sc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] = 0.f;
#pragma unroll 4
        for (int t = 0; t < T; ++t) {
            const float kvv = Elem<TIn>::to_float(kt[t * kBN + j]);
            const float *qt = qs + t * G;
#pragma unroll
            for (int g = 0; g < G; ++g) sc[g] = fmaf(qt[g], kvv, sc[g]);
        }
        // online softmax over this warp's 32 tokens
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float x = valid ? sc[g] : -INFINITY;
            const float mnew = fmaxf(m[g], warp_max(x));
            const float alpha = (m[g] == mnew) ? 1.f : exp2_approx(m[g] - mnew);
            const float p = valid ? exp2_approx(x - mnew) : 0.f;
            l[g] = fmaf(l[g], alpha, p);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[g][e] *= alpha;
            m[g] = mnew;
            pw[lane * G + g] = p;
        }
        __syncwarp();
        // weighted V over the same 32 tokens; this lane owns channels 4*lane..4*lane+3
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            const float4 vv = Elem<TIn>::load4(vt + (warp * 32 + jj) * kD + 4 * lane);
            const float *pj = pw + jj * G;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float p = pj[g];
                acc[g][0] = fmaf(p, vv.x, acc[g][0]);
                acc[g][1] = fmaf(p, vv.y, acc[g][1]);
                acc[g][2] = fmaf(p, vv.z, acc[g][2]);
                acc[g][3] = fmaf(p, vv.w, acc[g][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }

    // ------------------------------------------- merge the four warps
#pragma unroll
    for (int g = 0; g < G; ++g) l[g] = warp_sum(l[g]);
    named_barrier(1, kConsumerWarps * 32);  // every consumer is done with the stages
    float *mo = reinterpret_cast<float *>(smem);                 // [warps][G][D]
    float *mml = mo + kConsumerWarps * G * kD;                   // [warps][G][2]
#pragma unroll
    for (int g = 0; g < G; ++g) {
        *reinterpret_cast<float4 *>(mo + (warp * G + g) * kD + 4 * lane) =
            make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
        if (lane == 0) {
            mml[(warp * G + g) * 2] = m[g];
            mml[(warp * G + g) * 2 + 1] = l[g];
        }
    }
    named_barrier(1, kConsumerWarps * 32);
    const int dch = tid;  // 0..127: one output channel per consumer thread
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mml[(w * G + g) * 2]);
        float O = 0.f, L = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = mml[(w * G + g) * 2];
            if (mw == -INFINITY) continue;
            const float sw = exp2_approx(mw - M);
            O = fmaf(mo[(w * G + g) * kD + dch], sw, O);
            L = fmaf(mml[(w * G + g) * 2 + 1], sw, L);
        }
        const int64_t slot = ((int64_t)head * a.splits + split) * G + g;
        a.part_o[slot * kD + dch] = O;
        if (dch == 0) {
            a.part_ml[slot * 2] = M;
            a.part_ml[slot * 2 + 1] = L;
        }
    }
}

// Merge the per-split partials of one query head: out = sum_s O_s 2^(M_s-M)
// / sum_s L_s 2^(M_s-M).  One block per (b, h), one thread per channel.
__global__ void __launch_bounds__(kD)
    decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml,
                          float *__restrict__ out, int Hq, int Hkv, int splits)
{
    const int bh = blockIdx.x;
    const int G = Hq / Hkv;
    const int b = bh / Hq, h = bh % Hq;
    const int head = b * Hkv + h / G, g = h % G;
    const int dch = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s)
        M = fmaxf(M, part_ml[(((int64_t)head * splits + s) * G + g) * 2]);
    float O = 0.f, L = 0.f;
    for (int s = 0; s < splits; ++s) {
        const int64_t slot = ((int64_t)head * splits + s) * G + g;
        const float ms = part_ml[slot * 2];
        if (ms == -INFINITY) continue;
        const float w = exp2_approx(ms - M);
        O = fmaf(part_o[slot * kD + dch], w, O);
        L = fmaf(part_ml[slot * 2 + 1], w, L);
    }
    out[(int64_t)bh * kD + dch] = O / L;
}

}  // namespace think

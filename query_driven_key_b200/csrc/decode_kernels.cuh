// decode_kernels.cuh -- decode attention with the thinner key cache.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework, last step): run inference with the pruned cache.
// For query head h of KV head h/G:  z[n] = scale * q[idx] . K'[:,n],
// out = softmax(z) V, with V at full width.
//
// Split-N flash decoding in one kernel.  Block (split, head) streams its run
// of 128-token tiles of K'^T ([T][128]) and V ([128][128]) through a ring of
// shared-memory stages filled by TMA (one elected producer thread, mbarrier
// completion).  Four consumer warps each own 32 tokens of every tile and keep
// their own running (max, sum, weighted V) for the G query heads of the group:
//   logits   lane = token, fp32 FFMA2 over pairs of query heads;
//   weighted V  each half-warp takes one token at a time, each lane 8 channels,
//            FFMA2 over channel pairs.
// The block merges its warps and writes one partial per (head, split); the
// last block of a head to finish (a ticket counter in the workspace) merges
// the head's partials into the output.  Every mbarrier wait is bounded.
#pragma once

#include "ptx.cuh"
#include "think.h"

namespace think {

constexpr int kBN = 128;                  // tokens per tile
constexpr int kConsumerWarps = 4;         // kConsumerWarps * 32 == kBN
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kDecodeThreads = kConsumerThreads + 32;
static_assert(kConsumerWarps * 32 == kBN, "one token per consumer lane per tile");

struct DecodeArgs {
    const void *q;          // [B][Hq][D]
    const int32_t *idx;     // [B][Hkv][T]
    float *out;             // [B][Hq][D]
    float *part_o;          // [heads][splits][G][D]
    float *part_ml;         // [heads][splits][G][2]  (max in log2 units, sum)
    unsigned *status;       // device status bits
    unsigned *tickets;      // [heads] arrival counters, zero between calls
    int Hq, Hkv, T;
    int64_t N;
    int tiles_per_split, splits, stages;
    int stages_v;           // tcgen05 kernel: V ring slots (stages = K' ring slots)
    int prefetch;           // tiles prefetched into L2 ahead of the TMA loads
    int early;              // 1: the first tiles are prefetched into L2 before the dependency wait
    int staged_merge;       // 1: the split merge copies the partial outputs into shared memory when they fit
    int cluster;            // warp-MMA decode: > 0 when the splits of a head form one thread-block
                            // cluster of that many blocks and merge through distributed shared memory
    float scale_log2;       // scale * log2(e)
    uint32_t stage_bytes;   // bytes per ring stage (multiple of 1024)
    uint32_t v_off;         // offset of the V tile inside a stage
    uint32_t tx_bytes;      // bytes one stage's two TMA loads deliver
    const int32_t *Th;      // kept width per head (ragged thinner cache), or null: T for all
    const int32_t *rowoff;  // first K' row (and idx entry) of each head when Th is set
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

// Logits of one token for the G query heads: s[g] += q'[t][g] * k[t].
template <int G> struct QK;
template <> struct QK<1> {
    float s;
    __device__ __forceinline__ void zero() { s = 0.f; }
    __device__ __forceinline__ void step(const float *q, float k) { s = fmaf(q[0], k, s); }
    __device__ __forceinline__ float get(int) const { return s; }
};
template <> struct QK<2> {
    float2 s;
    __device__ __forceinline__ void zero() { s = make_float2(0.f, 0.f); }
    __device__ __forceinline__ void step(const float *q, float k)
    {
        s = __ffma2_rn(*reinterpret_cast<const float2 *>(q), make_float2(k, k), s);
    }
    __device__ __forceinline__ float get(int g) const { return g ? s.y : s.x; }
};
template <> struct QK<4> {
    float2 s[2];
    __device__ __forceinline__ void zero() { s[0] = s[1] = make_float2(0.f, 0.f); }
    __device__ __forceinline__ void step(const float *q, float k)
    {
        const float4 qq = *reinterpret_cast<const float4 *>(q);
        const float2 kk = make_float2(k, k);
        s[0] = __ffma2_rn(make_float2(qq.x, qq.y), kk, s[0]);
        s[1] = __ffma2_rn(make_float2(qq.z, qq.w), kk, s[1]);
    }
    __device__ __forceinline__ float get(int g) const
    {
        return (g & 1) ? s[g >> 1].y : s[g >> 1].x;
    }
};
template <> struct QK<8> {
    float2 s[4];
    __device__ __forceinline__ void zero() { s[0] = s[1] = s[2] = s[3] = make_float2(0.f, 0.f); }
    __device__ __forceinline__ void step(const float *q, float k)
    {
        const float4 qa = *reinterpret_cast<const float4 *>(q);
        const float4 qb = *reinterpret_cast<const float4 *>(q + 4);
        const float2 kk = make_float2(k, k);
        s[0] = __ffma2_rn(make_float2(qa.x, qa.y), kk, s[0]);
        s[1] = __ffma2_rn(make_float2(qa.z, qa.w), kk, s[1]);
        s[2] = __ffma2_rn(make_float2(qb.x, qb.y), kk, s[2]);
        s[3] = __ffma2_rn(make_float2(qb.z, qb.w), kk, s[3]);
    }
    __device__ __forceinline__ float get(int g) const
    {
        return (g & 1) ? s[g >> 1].y : s[g >> 1].x;
    }
};

// 8 consecutive channels of one V row as 4 float2 pairs.
template <typename TIn> struct V8;
template <> struct V8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float2 v[4])
    {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        v[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
        v[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
        v[2] = make_float2(bf16lo(w.z), bf16hi(w.z));
        v[3] = make_float2(bf16lo(w.w), bf16hi(w.w));
    }
};
template <> struct V8<float> {
    static __device__ __forceinline__ void load(const float *p, float2 v[4])
    {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        const float4 b = *reinterpret_cast<const float4 *>(p + 4);
        v[0] = make_float2(a.x, a.y);
        v[1] = make_float2(a.z, a.w);
        v[2] = make_float2(b.x, b.y);
        v[3] = make_float2(b.z, b.w);
    }
};

// Write this block's partial (O[g][d] for d = tid < 128, max M[g] in log2
// units, sum L[g]) for (head, split); the last block of the head to arrive
// merges every split of the head into `out`.  Called by the NT threads
// 0 .. NT-1 of the block (NT a multiple of 128), which synchronise on named
// barrier `bar`; `scratch` is free shared memory (16-byte aligned) of
// scratch_floats >= (2 * splits * G + 2 * G + (NT / 128) * G * 128) floats,
// `flag` one shared word.  When scratch also holds every partial output of
// the head (splits * G * 128 floats more), the merge copies them in with
// asynchronous 16-byte copies issued together with the (max, sum) loads: one
// round trip in all; otherwise it loads the outputs 8 * NT / 128 splits per
// round trip.  Both add the splits in the same order.
template <int G, int NT>
__device__ __forceinline__ void finish_split(const DecodeArgs &a, int head, int split, int b, int kv,
                                             int tid, const float (&O)[G], const float (&M)[G],
                                             const float (&L)[G], float *scratch, unsigned *flag,
                                             int bar, size_t scratch_floats = 0)
{
    static_assert(NT % 128 == 0, "whole channel rows per thread group");
    constexpr int P = NT / 128;            // thread groups splitting the split axis
    const int64_t slot0 = ((int64_t)head * a.splits + split) * G;
    if (tid < 128 && THINK_IN_RANGE(split < a.splits && head < (int)gridDim.y, a.status)) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            a.part_o[(slot0 + g) * kD + tid] = O[g];
            if (tid == 0) {
                a.part_ml[(slot0 + g) * 2] = M[g];
                a.part_ml[(slot0 + g) * 2 + 1] = L[g];
            }
        }
    }
    __threadfence();
    named_barrier(bar, NT);
    if (tid == 0) {
        const unsigned ticket = atomicAdd(a.tickets + head, 1u);
        *flag = (ticket == (unsigned)(a.splits - 1)) ? 1u : 0u;
    }
    named_barrier(bar, NT);
    if (*flag == 0u) return;
    __threadfence();
    const int S = a.splits;
    const int nsg = S * G;
    float *sw = scratch;            // [splits][G]  max, then weight 2^(M_s - M*)
    float *sl = sw + nsg;           // [splits][G]  sum
    float *smax = sl + nsg;         // [G]
    float *sL = smax + G;           // [G]
    float *sp = sL + G;             // [P][G][128]  per-group output sums
    // [splits][G][128] the head's partial outputs, when they fit
    const size_t so_off = ((size_t)2 * nsg + 2 * G + (size_t)P * G * kD + 3) & ~(size_t)3;
    const bool staged = so_off + (size_t)nsg * kD <= scratch_floats;
    float *so = scratch + so_off;
    if (staged) {
        const uint32_t dst = smem_addr(so);
        const float4 *src = reinterpret_cast<const float4 *>(a.part_o + (int64_t)head * S * G * kD);
        for (int i = tid; i < nsg * (kD / 4); i += NT) cp_async_16(dst + 16u * (uint32_t)i, src + i);
        cp_async_commit();
    }
    const float *pml = a.part_ml + (int64_t)head * S * G * 2;
    for (int i = tid; i < nsg; i += NT) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(pml) + i);
        sw[i] = ml.x;
        sl[i] = ml.y;
    }
    named_barrier(bar, NT);
    if (tid < G) {
        float Mx = -INFINITY;
        for (int s2 = 0; s2 < S; ++s2) Mx = fmaxf(Mx, sw[s2 * G + tid]);
        smax[tid] = Mx;
    }
    named_barrier(bar, NT);
    for (int i = tid; i < nsg; i += NT) {
        const float ms = sw[i];
        sw[i] = (ms == -INFINITY) ? 0.f : exp2_approx(ms - smax[i % G]);
    }
    named_barrier(bar, NT);
    if (tid < G) {
        float Ls = 0.f;
        for (int s2 = 0; s2 < S; ++s2) Ls = fmaf(sl[s2 * G + tid], sw[s2 * G + tid], Ls);
        sL[tid] = Ls;
    }
    // outputs: thread (q, d) sums the splits s = q, q + P, ... for channel d
    const int d = tid & 127, q = tid >> 7;
    const float *po = a.part_o + (int64_t)head * S * G * kD + d;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    if (staged) {
        cp_async_wait_all();
        named_barrier(bar, NT);
        for (int s2 = q; s2 < S; s2 += P) {
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = fmaf(so[(s2 * G + g) * kD + d], sw[s2 * G + g], acc[g]);
        }
    }
    constexpr int CH = 8;
    for (int s0 = staged ? S : q; s0 < S; s0 += P * CH) {
        float v[CH][G];
#pragma unroll
        for (int u = 0; u < CH; ++u) {
            const int s2 = s0 + u * P;
#pragma unroll
            for (int g = 0; g < G; ++g)
                v[u][g] = (s2 < S) ? __ldcg(po + ((int64_t)s2 * G + g) * kD) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < CH; ++u) {
            const int s2 = s0 + u * P;
            if (s2 < S) {
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = fmaf(v[u][g], sw[s2 * G + g], acc[g]);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) sp[(q * G + g) * kD + d] = acc[g];
    named_barrier(bar, NT);
    if (tid < 128) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float o = sp[g * kD + d];
#pragma unroll
            for (int q2 = 1; q2 < P; ++q2) o += sp[(q2 * G + g) * kD + d];
            if (THINK_IN_RANGE((int64_t)b * a.Hq + (int64_t)kv * G + g < (int64_t)gridDim.y / a.Hkv * a.Hq, a.status))
                a.out[((int64_t)b * a.Hq + (int64_t)kv * G + g) * kD + d] = o / sL[g];
        }
        if (tid == 0) a.tickets[head] = 0u;  // ready for the next call
    }
}

template <typename TIn, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    pruned_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a)
{
    extern __shared__ unsigned char smem_dyn[];
    // 1024-byte aligned base, kept as shared-array arithmetic so that every
    // access below compiles to shared-memory loads and stores.
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);

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
    float2 *pdup = reinterpret_cast<float2 *>(qs + qs_len);  // [warps][32 tokens][G] as (p, p)
    uint64_t *bars = reinterpret_cast<uint64_t *>(pdup + kConsumerWarps * 32 * G);
    unsigned *flag = reinterpret_cast<unsigned *>(bars + 2 * stages);
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
    __syncthreads();  // barriers initialised

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        // starts at once; the consumers gather q' meanwhile
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            int issued = 0;
            bool ok = true;
            const int pf = a.prefetch;
            for (int it = 0; it < min(ntiles, pf); ++it) {
                const int x = (int)((tile0 + it) * kBN);
                tma_prefetch_l2_4d(&tm_k, x, 0, kv, b);
                tma_prefetch_l2_4d(&tm_v, 0, x, kv, b);
            }
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % stages, f = it / stages;
                if (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (f - 1) & 1, a.status,
                                                THINK_DEVICE_TIMEOUT_EMPTY)) {
                    ok = false;
                    break;
                }
                if (pf > 0 && it + pf < ntiles) {
                    const int xp = (int)((tile0 + it + pf) * kBN);
                    tma_prefetch_l2_4d(&tm_k, xp, 0, kv, b);
                    tma_prefetch_l2_4d(&tm_v, 0, xp, kv, b);
                }
                const uint32_t full = full0 + 8 * s;
                mbar_arrive_expect_tx(full, a.tx_bytes);
                const int x = (int)((tile0 + it) * kBN);
                const uint32_t st = smem_addr(smem + (size_t)s * a.stage_bytes);
                tma_load_4d(st, &tm_k, x, 0, kv, b, full);
                tma_load_4d(st + a.v_off, &tm_v, 0, x, kv, b, full);
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
    // q' = q[idx] for the G query heads of this KV head, pre-scaled to log2 units.
    {
        const TIn *q = reinterpret_cast<const TIn *>(a.q);
        const int32_t *ih = a.idx + (int64_t)head * T;
        for (int i = tid; i < T * G; i += kConsumerThreads) {
            const int t = i / G, g = i % G;
            const int c = ih[t];
            float x = 0.f;
            if ((unsigned)c < (unsigned)kD)
                x = Elem<TIn>::to_float(q[((int64_t)b * a.Hq + (int64_t)kv * G + g) * kD + c]);
            qs[i] = x * a.scale_log2;
        }
    }
    named_barrier(1, kConsumerThreads);
    float m[G], l[G];
    float2 acc[G][4];  // channels 8*(lane&15) .. +7 of the tokens of half-warp lane>>4
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] = make_float2(0.f, 0.f);
    }
    const int j = warp * 32 + lane;  // this lane's token inside a tile (logits)
    const int half = lane >> 4;      // token parity this lane takes in the weighted sum
    const int dch = 8 * (lane & 15); // first of this lane's 8 channels
    float2 *pw = pdup + warp * 32 * G;

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (it / stages) & 1, a.status,
                               THINK_DEVICE_TIMEOUT_FULL))
            break;
        const unsigned char *st = smem + (size_t)s * a.stage_bytes;
        const TIn *kt = reinterpret_cast<const TIn *>(st);
        const TIn *vt = reinterpret_cast<const TIn *>(st + a.v_off);
        const bool valid = (tile0 + it) * kBN + j < a.N;

        QK<G> sc;
        sc.zero();
#pragma unroll 4
        for (int t = 0; t < T; ++t) sc.step(qs + t * G, Elem<TIn>::to_float(kt[t * kBN + j]));

        // online softmax over this warp's 32 tokens
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float x = valid ? sc.get(g) : -INFINITY;
            const float mnew = fmaxf(m[g], warp_max(x));
            const float alpha = (m[g] == mnew) ? 1.f : exp2_approx(m[g] - mnew);
            const float p = valid ? exp2_approx(x - mnew) : 0.f;
            l[g] = fmaf(l[g], alpha, p);
            const float2 al = make_float2(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[g][e] = __fmul2_rn(acc[g][e], al);
            m[g] = mnew;
            pw[lane * G + g] = make_float2(p, p);
        }
        __syncwarp();
        // weighted V: half-warp `half` takes tokens 2*jj + half of this warp's 32
        const TIn *vrow = vt + (size_t)(warp * 32 + half) * kD + dch;
#pragma unroll 4
        for (int jj = 0; jj < 16; ++jj) {
            float2 v[4];
            V8<TIn>::load(vrow + (size_t)(2 * jj) * kD, v);
            const float2 *pp = pw + (2 * jj + half) * G;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float2 p2 = pp[g];
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[g][e] = __ffma2_rn(v[e], p2, acc[g][e]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }

    // ------------------------------------------- merge the four warps
#pragma unroll
    for (int g = 0; g < G; ++g) {
        l[g] = warp_sum(l[g]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, 16);
            acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, 16);
        }
    }
    named_barrier(1, kConsumerThreads);  // every consumer is done with the stages
    float *mo = reinterpret_cast<float *>(smem);                 // [warps][G][D]
    float *mml = mo + kConsumerWarps * G * kD;                   // [warps][G][2]
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (half == 0) {
            float4 *dst = reinterpret_cast<float4 *>(mo + (warp * G + g) * kD + dch);
            dst[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
            dst[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
        }
        if (lane == 0) {
            mml[(warp * G + g) * 2] = m[g];
            mml[(warp * G + g) * 2 + 1] = l[g];
        }
    }
    named_barrier(1, kConsumerThreads);
    const int d = tid;  // 0..127: one output channel per consumer thread
    float O[G], M[G], L[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        M[g] = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M[g] = fmaxf(M[g], mml[(w * G + g) * 2]);
        O[g] = 0.f;
        L[g] = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = mml[(w * G + g) * 2];
            if (mw == -INFINITY) continue;
            const float sw = exp2_approx(mw - M[g]);
            O[g] = fmaf(mo[(w * G + g) * kD + d], sw, O[g]);
            L[g] = fmaf(mml[(w * G + g) * 2 + 1], sw, L[g]);
        }
    }
    named_barrier(1, kConsumerThreads);  // merge scratch below overwrites mo/mml
    finish_split<G, kConsumerThreads>(a, head, split, b, kv, d, O, M, L, reinterpret_cast<float *>(smem),
                                      flag, 1);
}

}  // namespace think

// decode_mma.cuh -- decode attention with the thinner key cache, tensor-core
// contractions issued per warp (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework, last step): run inference with the pruned cache.
//
// Same split-N structure as the CUDA-core kernel (producer warp + four
// consumer warps, TMA stage ring, each warp owns 32 tokens of every 128-token
// tile and keeps its own online-softmax state), but each warp runs its two
// small contractions on the tensor cores:
//   logits  S[tok][g]  = K'[tok][t] q'[g][t]^T   m16n8k16: M = 16 tokens, N = 8
//                                                 query heads (G <= 8), K = 16 channels
//   values  O^T[c][g] += V[tok][c]^T P[g][tok]^T  M = 16 channels, N = 8, K = 16 tokens
// K' and V tiles arrive by TMA with the 128-byte swizzle and are read with
// ldmatrix.trans (conflict-free); the softmax weights are transposed from the
// logits' accumulator layout to the values' operand layout in registers with
// movmatrix, split into a bf16 high and low part (two MMAs; p = hi + lo keeps
// the weights to about 2^-17 relative).  No block-wide barrier in the loop;
// every mbarrier wait is bounded.
#pragma once

#include "decode_kernels.cuh"

namespace think {

namespace wmma16 {

using ::think::ldsm_x4_trans;

// D = A * B + D, A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8x8 16-bit matrix held one row per group of 4 lanes -> its transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// (lo, hi) floats -> bf16x2 with `lo` in the low half (round to nearest even).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace wmma16

struct MmaLayout {
    uint32_t t_pad;   // T rounded up to 16
    uint32_t k_half;  // one 64-token half of a K' tile: t_pad rows x 128 B
    uint32_t v_off;   // V tile (two 64-channel halves of 128 tokens x 128 B) inside a stage
    uint32_t stage;   // bytes per stage
};

__host__ __device__ inline MmaLayout mma_layout(int T)
{
    MmaLayout L;
    L.t_pad = (uint32_t)((T + 15) & ~15);
    L.k_half = L.t_pad * 128u;
    L.v_off = 2u * L.k_half;
    L.stage = L.v_off + 32768u;
    return L;
}

// shared memory after the stages: q' [16 rows][t_pad] bf16, per-warp merge
// area [CW warps][G][128] + [CW warps][G][2] floats, barriers, a flag
__host__ __device__ inline size_t mma_smem_bytes(int T, int G, int stages, int CW = kConsumerWarps)
{
    const MmaLayout L = mma_layout(T);
    return (size_t)stages * L.stage + 32u * L.t_pad + (size_t)CW * G * 130 * 4 +
           (size_t)2 * stages * 8 + 16 + 1024;
}

// q' = q[idx] of the group's query heads as [16 rows (g)][t_pad] bf16 (rows
// g >= G and columns t >= T zero), by the consumer threads (NT of them; every
// one calls it).  One round of global loads: the group's G query rows (16-byte
// loads) and the T kept channels go to scratch together (the per-warp merge
// area, unused until the end), then q' is gathered from shared memory.
template <int G, int NT>
__device__ __forceinline__ void mma_stage_q(const DecodeArgs &a, unsigned char *qsm, uint32_t t_pad, int T,
                                            const int32_t *ih, int b, int kv, int tid, unsigned char *scratch)
{
    constexpr int QV = G * (kD / 8);  // 16-byte words of the group's q rows
    static_assert(QV + kD <= 2 * NT, "at most two loads per thread");
    uint4 *qraw = reinterpret_cast<uint4 *>(scratch);       // [G][128] bf16
    int *is = reinterpret_cast<int *>(scratch + G * kD * 2);  // [T]
    const uint4 *qg = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                                      ((int64_t)b * a.Hq + (int64_t)kv * G) * kD);
    // both of a thread's loads are issued before either is stored
    uint4 qv[2];
    int iv[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = tid + r * NT;
        if (i < QV)
            qv[r] = __ldcg(qg + i);
        else if (i < QV + T)
            iv[r] = __ldcg(ih + (i - QV));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = tid + r * NT;
        if (i < QV)
            qraw[i] = qv[r];
        else if (i < QV + T)
            is[i - QV] = iv[r];
    }
    named_barrier(1, NT);
    const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(qraw);
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(qsm);
    for (int i = tid; i < 16 * (int)t_pad; i += NT) {
        const int g = i / (int)t_pad, t = i % (int)t_pad;
        __nv_bfloat16 x = __float2bfloat16(0.f);
        if (g < G && t < T) {
            const int c = is[t];
            if ((unsigned)c < (unsigned)kD) x = qr[g * kD + c];
        }
        qs[g * t_pad + t] = x;
    }
}

// q' as the B operand of the logits MMA (k = channel, n = query head): per
// 16-channel step two registers, channels 2*q4, 2*q4+1 and +8 of head r8
// (q' rows t_pad apart; ksteps 16-channel steps used).
__device__ __forceinline__ void mma_load_qb(const unsigned char *qsm, uint32_t t_pad, int ksteps, int lane,
                                            uint32_t (&qb)[kD / 16][2])
{
    const int q4 = lane & 3, r8 = lane >> 2;
    const uint32_t *qs32 = reinterpret_cast<const uint32_t *>(qsm);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
        if (ks < ksteps) {
            qb[ks][0] = qs32[(r8 * t_pad + 16 * ks + 2 * q4) >> 1];
            qb[ks][1] = qs32[(r8 * t_pad + 16 * ks + 8 + 2 * q4) >> 1];
        } else {
            qb[ks][0] = qb[ks][1] = 0u;
        }
    }
}

// Online-softmax state of one consumer warp: running max (log2 units) and sum
// for query heads 2*q4, 2*q4+1, and O^T (channel rows 16*md + r8 (+8), head
// columns 2*q4 (+1)).
struct MmaState {
    float m[2], l[2];
    float acc[8][4];
};

// One 128-token tile for one consumer warp (its TPW = 32 or 16 tokens):
// logits from the K' tile (two 64-token halves of t_pad channel rows x 128 B,
// 128-byte swizzle, starting at kbase), online softmax, values from the V
// tile (two 64-channel halves of 128 tokens x 128 B, swizzled, at vbase).
template <int TPW>
__device__ __forceinline__ void mma_tile(uint32_t kbase, uint32_t k_half, uint32_t vbase,
                                         const uint32_t (&qb)[kD / 16][2], int ksteps, int warp, int lane,
                                         int64_t tok_base, int64_t N, float scale_log2, MmaState &S)
{
    static_assert(TPW == 32 || TPW == 16, "one or two 16-token m-tiles per warp");
    constexpr int KS_MAX = kD / 16;
    constexpr int MT = TPW / 16;
    const int q4 = lane & 3, r8 = lane >> 2;
    const int jm = lane >> 3, jr = lane & 7;  // ldmatrix: matrix index, row within it

    // ---- logits for this warp's tokens: MT 16-token m-tiles
    float sc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
        const int tok = warp * TPW + mt * 16 + (jm & 1) * 8;   // first token of this lane's 8x8 block
        const uint32_t kh = kbase + (uint32_t)(tok >> 6) * k_half;
        const uint32_t chunk = (uint32_t)((tok & 63) >> 3);
#pragma unroll
        for (int ks = 0; ks < KS_MAX; ++ks) {
            if (ks < ksteps) {
                const uint32_t t = (uint32_t)(16 * ks + (jm >> 1) * 8 + jr);
                uint32_t a0, a1, a2, a3;
                wmma16::ldsm_x4_trans(kh + t * 128u + ((chunk ^ (t & 7u)) << 4), a0, a1, a2, a3);
                wmma16::mma_bf16(sc[mt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            }
        }
    }
    // ---- online softmax per query head over the warp's tokens
    // sc[mt][0..1]: token 16*mt + r8, heads 2*q4, 2*q4+1; sc[mt][2..3]: token +8
    float alpha[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        float xm = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int64_t n = tok_base + mt * 16 + hr * 8 + r8;
                const float x = (n < N) ? sc[mt][hr * 2 + h2] * scale_log2 : -INFINITY;
                sc[mt][hr * 2 + h2] = x;
                xm = fmaxf(xm, x);
            }
        xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, 4));
        xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, 8));
        xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, 16));
        const float mnew = fmaxf(S.m[h2], xm);
        alpha[h2] = (S.m[h2] == mnew) ? 1.f : exp2_approx(S.m[h2] - mnew);
        float ps = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const float x = sc[mt][hr * 2 + h2];
                const float p = (x == -INFINITY) ? 0.f : exp2_approx(x - mnew);
                sc[mt][hr * 2 + h2] = p;
                ps += p;
            }
        S.l[h2] = fmaf(S.l[h2], alpha[h2], ps);
        S.m[h2] = mnew;
    }
#pragma unroll
    for (int md = 0; md < 8; ++md) {
        S.acc[md][0] *= alpha[0];
        S.acc[md][1] *= alpha[1];
        S.acc[md][2] *= alpha[0];
        S.acc[md][3] *= alpha[1];
    }
    // ---- weights as the B operand of the values MMA (k = token, n = head),
    // high and low bf16 parts; one 16-token k-step per logits m-tile
    uint32_t pbh[MT][2], pbl[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const float p0 = sc[mt][hr * 2], p1 = sc[mt][hr * 2 + 1];
            const uint32_t hi = wmma16::pack_bf16x2(p0, p1);
            const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
            const uint32_t lo = wmma16::pack_bf16x2(p0 - h0, p1 - h1);
            pbh[mt][hr] = wmma16::movmatrix_trans(hi);
            pbl[mt][hr] = wmma16::movmatrix_trans(lo);
        }
    // ---- values: O^T[c][g] += V^T[c][tok] P^T[tok][g] over the warp's tokens
#pragma unroll
    for (int ks = 0; ks < MT; ++ks) {
        const uint32_t tok = (uint32_t)(warp * TPW + ks * 16 + (jm >> 1) * 8 + jr);
#pragma unroll
        for (int md = 0; md < 8; ++md) {
            const uint32_t c0 = (uint32_t)(md * 16 + (jm & 1) * 8);   // first channel of the block
            const uint32_t addr = vbase + (c0 >> 6) * 16384u + tok * 128u +
                                  ((((c0 & 63u) >> 3) ^ (tok & 7u)) << 4);
            uint32_t a0, a1, a2, a3;
            wmma16::ldsm_x4_trans(addr, a0, a1, a2, a3);
            wmma16::mma_bf16(S.acc[md], a0, a1, a2, a3, pbh[ks][0], pbh[ks][1]);
            wmma16::mma_bf16(S.acc[md], a0, a1, a2, a3, pbl[ks][0], pbl[ks][1]);
        }
    }
    (void)q4;
}

// The split merge of a head whose splits form one thread-block cluster (the
// producer warp calls it too, with tid >= NT, for the cluster barriers): each
// block puts its (O, max, sum) in its own shared memory (`scratch`); after a
// cluster barrier, block r of S merges output channels [r * 128 / S, ...) of
// every query head of the group from all S blocks' shared memory, in split
// order, and writes them; a second barrier keeps every block's shared memory
// alive until the reads are done.  No global partials, no ticket.
template <int G, int NT>
__device__ __forceinline__ void cluster_finish(const DecodeArgs &a, const float (&O)[G], const float (&M)[G],
                                               const float (&L)[G], float *scratch, int b, int kv, int tid)
{
    float *co = scratch;            // [G][128]
    float *cml = scratch + G * kD;  // [G][2]
    if (tid < kD) {
#pragma unroll
        for (int g = 0; g < G; ++g) co[g * kD + tid] = O[g];
        if (tid == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                cml[2 * g] = M[g];
                cml[2 * g + 1] = L[g];
            }
        }
    }
    cluster_sync_all();
    const int S = a.cluster;
    const int per = kD / S;  // S divides 128
    const uint32_t r = cluster_rank();
    for (int i = tid; i < G * per && tid < NT; i += NT) {
        const int g = i / per, c = (int)r * per + i % per;
        float ms[16], ls[16], os[16];  // all loads first, so that their latencies overlap
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) {
            if (s2 < S) {
                ms[s2] = ld_dsmem_f32(cml + 2 * g, (uint32_t)s2);
                ls[s2] = ld_dsmem_f32(cml + 2 * g + 1, (uint32_t)s2);
                os[s2] = ld_dsmem_f32(co + g * kD + c, (uint32_t)s2);
            }
        }
        float Mx = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2)
            if (s2 < S) Mx = fmaxf(Mx, ms[s2]);
        float o = 0.f, l = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) {
            if (s2 < S && ms[s2] != -INFINITY) {  // an empty split holds (0, -inf, 0)
                const float w = exp2_approx(ms[s2] - Mx);
                o = fmaf(os[s2], w, o);
                l = fmaf(ls[s2], w, l);
            }
        }
        const int64_t hq = (int64_t)b * a.Hq + (int64_t)kv * G + g;
        if (THINK_IN_RANGE(hq < (int64_t)gridDim.y / a.Hkv * a.Hq, a.status)) a.out[hq * kD + c] = o / l;
    }
    cluster_sync_all();
}

// Merge the CW consumer warps of the block (through mo/mml in shared
// memory), then the split merge (finish_split, which reuses `scratch`, or
// cluster_finish when the head's splits form a cluster).
template <int G, int CW>
__device__ __forceinline__ void mma_merge_and_finish(const DecodeArgs &a, MmaState &S, float *mo, float *mml,
                                                     float *scratch, unsigned *flag, int head, int split,
                                                     int b, int kv, int tid, size_t scratch_floats)
{
    const int warp = tid >> 5, lane = tid & 31;
    const int q4 = lane & 3, r8 = lane >> 2;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        S.l[h2] += __shfl_xor_sync(0xffffffffu, S.l[h2], 4);
        S.l[h2] += __shfl_xor_sync(0xffffffffu, S.l[h2], 8);
        S.l[h2] += __shfl_xor_sync(0xffffffffu, S.l[h2], 16);
    }
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int g = 2 * q4 + h2;
        if (g < G) {
#pragma unroll
            for (int md = 0; md < 8; ++md) {
                mo[(warp * G + g) * kD + md * 16 + r8] = S.acc[md][h2];
                mo[(warp * G + g) * kD + md * 16 + 8 + r8] = S.acc[md][2 + h2];
            }
            if (r8 == 0) {
                mml[(warp * G + g) * 2] = S.m[h2];
                mml[(warp * G + g) * 2 + 1] = S.l[h2];
            }
        }
    }
    named_barrier(1, CW * 32);
    const int d = tid & (kD - 1);  // one output channel per thread (threads >= 128 repeat it)
    float O[G], M[G], Lsum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        M[g] = -INFINITY;
#pragma unroll
        for (int w = 0; w < CW; ++w) M[g] = fmaxf(M[g], mml[(w * G + g) * 2]);
        O[g] = 0.f;
        Lsum[g] = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
            const float mw = mml[(w * G + g) * 2];
            if (mw == -INFINITY) continue;
            const float sw = exp2_approx(mw - M[g]);
            O[g] = fmaf(mo[(w * G + g) * kD + d], sw, O[g]);
            Lsum[g] = fmaf(mml[(w * G + g) * 2 + 1], sw, Lsum[g]);
        }
    }
    named_barrier(1, CW * 32);  // the split merge below reuses stage memory
    if (a.cluster > 0) {
        cluster_finish<G, CW * 32>(a, O, M, Lsum, scratch, b, kv, tid);
        return;
    }
    finish_split<G, CW * 32>(a, head, split, b, kv, tid, O, M, Lsum, scratch, flag, 1, scratch_floats);
}

__device__ __forceinline__ void mma_state_init(MmaState &S)
{
    S.m[0] = S.m[1] = -INFINITY;
    S.l[0] = S.l[1] = 0.f;
#pragma unroll
    for (int md = 0; md < 8; ++md)
#pragma unroll
        for (int e = 0; e < 4; ++e) S.acc[md][e] = 0.f;
}

template <int G, int CW>
__global__ void __launch_bounds__(CW * 32 + 32)
    pruned_decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a)
{
    static_assert(G >= 1 && G <= 8, "the group's query heads fill at most the 8 MMA columns");
    static_assert(CW == 4 || CW == 8, "32 or 16 tokens of a tile per consumer warp");
    constexpr int TPW = kBN / CW;
    constexpr int NT = CW * 32;
    // Shared memory layout (kernel parameters only) and the ring barriers are
    // set up before the dependency wait: they touch no global memory.
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);
    const int stages = a.stages;
    const MmaLayout L = mma_layout(a.T);
    unsigned char *qsm = smem + (size_t)stages * L.stage;                       // [16][t_pad] bf16
    float *mo = reinterpret_cast<float *>(qsm + 32u * L.t_pad);                 // [CW][G][128]
    float *mml = mo + CW * G * kD;                                              // [CW][G][2]
    uint64_t *bars = reinterpret_cast<uint64_t *>(mml + CW * G * 2);
    unsigned *flag = reinterpret_cast<unsigned *>(bars + 2 * stages);
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + stages);
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, CW);
        }
        fence_barrier_init();
    }
    __syncthreads();  // barriers initialised

    // Launched as a programmatic dependent of the previous kernel in the
    // stream: everything it wrote is visible after this wait; let the next
    // decode be scheduled on SMs as ours free up.  Such a block becomes
    // resident while the previous decode drains (its merge and last tiles), so
    // before the wait the producer lane asks L2 for this block's first tiles.
    // K' and V are inputs that no kernel which lets this one start early
    // writes, and L2 is the point of coherence, so the prefetch cannot hand
    // stale data to the loads made after the wait (the same holds for q and
    // idx, which may well be written by the previous kernel: a prefetch only
    // warms L2); only kernel parameters are read before it (a ragged cache's
    // K' rows come from device data: V only).
    if (threadIdx.x == CW * 32) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (a.early && threadIdx.x == CW * 32) {
        const int kv0 = (int)blockIdx.y % a.Hkv, b0 = (int)blockIdx.y / a.Hkv;
        const int64_t t0 = (int64_t)blockIdx.x * a.tiles_per_split;
        const int64_t n = min((int64_t)min(a.tiles_per_split, a.stages), (a.N + kBN - 1) / kBN - t0);
        for (int64_t it = 0; it < n; ++it) {
            const int x = (int)((t0 + it) * kBN);
            if (a.Th == nullptr) {
                tma_prefetch_l2_4d(&tm_k, x, 0, kv0, b0);
                tma_prefetch_l2_4d(&tm_k, x + 64, 0, kv0, b0);
            }
            tma_prefetch_l2_4d(&tm_v, 0, x, kv0, b0);
            tma_prefetch_l2_4d(&tm_v, 64, x, kv0, b0);
        }
        // and the lines that the q' staging reads first (the group's q rows,
        // the kept channels)
        const char *qrow = reinterpret_cast<const char *>(a.q) + ((int64_t)b0 * a.Hq + (int64_t)kv0 * G) * kD * 2;
        for (int o = 0; o < G * kD * 2; o += 128) prefetch_l2(qrow + o);
        if (a.Th == nullptr) {
            const char *irow = reinterpret_cast<const char *>(a.idx + (int64_t)blockIdx.y * a.T);
            for (int o = 0; o < a.T * 4; o += 128) prefetch_l2(irow + o);
        }
    }
    grid_dependency_wait();
    grid_launch_dependents();

    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    // Ragged thinner cache (a.Th set): this head keeps Th[head] channels, its
    // K' rows start at rowoff[head] and are padded with zero rows to a
    // multiple of 16; the stage layout is that of the widest head (a.T).
    const bool ragged = a.Th != nullptr;
    const int T = ragged ? min(max(a.Th[head], 1), a.T) : a.T;
    // rows of all heads: gridDim.y * roundup16(a.T); an offset outside it is
    // clamped (garbage in, no access outside K' or idx)
    const int64_t row_cap = (int64_t)gridDim.y * ((a.T + 15) & ~15);
    const int64_t row0 = ragged ? min(max((int64_t)a.rowoff[head], (int64_t)0), row_cap - ((T + 15) & ~15)) : 0;
    const uint32_t t_rows = ragged ? (uint32_t)((T + 15) & ~15) : L.t_pad;  // K' rows used
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t tx = ragged ? 2u * t_rows * 128u + 32768u : 2u * 64u * (uint32_t)T * 2u + 32768u;
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
                mbar_arrive_expect_tx(full, tx);
                const int x = (int)((tile0 + it) * kBN);
                const uint32_t st = smem_addr(smem + (size_t)s * L.stage);
                if (ragged) {
                    // 16-row boxes of this head's rows (its zero pad rows included)
                    for (uint32_t j = 0; j < t_rows / 16u; ++j) {
                        tma_load_4d(st + 2048u * j, &tm_k, x, (int)(row0 + 16 * j), 0, 0, full);
                        tma_load_4d(st + L.k_half + 2048u * j, &tm_k, x + 64, (int)(row0 + 16 * j), 0, 0, full);
                    }
                } else {
                    tma_load_4d(st, &tm_k, x, 0, kv, b, full);
                    tma_load_4d(st + L.k_half, &tm_k, x + 64, 0, kv, b, full);
                }
                tma_load_4d(st + L.v_off, &tm_v, 0, x, kv, b, full);
                tma_load_4d(st + L.v_off + 16384u, &tm_v, 64, x, kv, b, full);
                ++issued;
            }
            if (!ok) {
                for (int it = max(0, issued - stages); it < issued; ++it)
                    mbar_wait_bounded(full0 + 8 * (it % stages), (it / stages) & 1, a.status,
                                      THINK_DEVICE_TIMEOUT_FULL);
            }
        }
        __syncwarp();
        if (a.cluster > 0) {  // the cluster barriers count every thread of every block
            const float z[G] = {};
            cluster_finish<G, NT>(a, z, z, z, reinterpret_cast<float *>(smem), b, kv, tid);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    // Operand set-up (while the first tiles load): zero the K' rows T..t_pad-1
    // of every stage (TMA writes rows 0..T-1 only; the matching q' columns are
    // zero, but stale bits could be NaN), and stage q' = q[idx] as [g][t] bf16.
    {
        const uint32_t pad16 = ragged ? 0u : (L.t_pad - (uint32_t)T) * 8u;  // 16-byte words per half
        for (uint32_t i = tid; i < (uint32_t)stages * 2u * pad16; i += NT) {
            const uint32_t hs = i / pad16, o = i % pad16;  // hs = stage * 2 + half
            *reinterpret_cast<uint4 *>(smem + (hs >> 1) * L.stage + (hs & 1u) * L.k_half +
                                       (uint32_t)T * 128u + o * 16u) = make_uint4(0, 0, 0, 0);
        }
        mma_stage_q<G, NT>(a, qsm, L.t_pad, T, a.idx + (ragged ? row0 : (int64_t)head * T), b, kv, tid,
                           reinterpret_cast<unsigned char *>(mo));
    }
    named_barrier(1, NT);  // zeroed rows and q' visible to all consumers

    uint32_t qb[kD / 16][2];
    const int ksteps = (int)(t_rows / 16u);
    mma_load_qb(qsm, L.t_pad, ksteps, lane, qb);
    MmaState S;
    mma_state_init(S);
    const uint32_t sbase = smem_addr(smem);

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (it / stages) & 1, a.status, THINK_DEVICE_TIMEOUT_FULL))
            break;
        const uint32_t st = sbase + (uint32_t)s * L.stage;
        const int64_t tok_base = (tile0 + it) * kBN + warp * TPW;
        mma_tile<TPW>(st, L.k_half, st + L.v_off, qb, ksteps, warp, lane, tok_base, a.N, a.scale_log2, S);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
    mma_merge_and_finish<G, CW>(a, S, mo, mml, reinterpret_cast<float *>(smem), flag, head, split, b, kv, tid,
                                a.staged_merge ? (size_t)stages * L.stage / sizeof(float) : 0);
}

}  // namespace think

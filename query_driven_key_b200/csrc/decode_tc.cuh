// decode_tc.cuh -- decode attention with the thinner key cache on the 5th-
// generation tensor cores (tcgen05, accumulators in tensor memory).
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework, last step): run inference with the pruned cache.
//
// For one KV head with G query heads and a 128-token tile, both contractions
// are small-N dense matrix products with M = 128 on the tensor core:
//   logits   S[tok][g]  = K'[tok][t] * q'[g][t]^T       (M = 128 tokens, K = T)
//   values   O^T[c][g]  = V[tok][c]^T * P[g][tok]^T      (M = 128 channels, K = 128 tokens)
// with N = 16 columns: the G query heads (logits), or the G softmax weights
// split into a bf16 high part and a bf16 low part (values; p = hi + lo keeps
// the weights to about 2^-17 relative).  K' and V tiles arrive by TMA in the
// 128-byte-swizzled MN-major layout, q' and P are written by threads in the
// K-major interleaved (8 x 16-byte core matrix) layout.
//
// K' tiles and V tiles have separate shared-memory rings: a K' slot is
// released as soon as the logits MMA of its tile completes and a V slot as
// soon as the values MMA completes, so K' runs ahead of V and a V tile waits
// in shared memory only for its own MMA, not for the softmax.  The producer
// and the MMA issuer are polling event loops that act on whichever mbarrier
// is ready first.
//
// Warp roles per block (576 threads):
//   warps 0-15  four softmax + accumulate warpgroups; warpgroup w takes the
//              tiles i with i % 4 == w and keeps its own running (max, sum,
//              output); thread t of a warpgroup reads TMEM lane t, i.e. token
//              t of a logits tile and channel t of a value tile;
//   warp 16    TMA producer (one elected thread);
//   warp 17    TMEM allocator and MMA issuer (one elected thread).
// TMEM: four S buffers (columns 0-63) and four O buffers (columns 64-127);
// tile i uses buffer i % 4, so the logits MMA can run up to three tiles
// ahead of the values MMA and each warpgroup always has its next logits tile
// ready; the four warpgroups give each tile's softmax and accumulation four
// tile-times.  The warpgroups' states are merged at the end.
// Every mbarrier wait is bounded; a wait that runs out sets the workspace
// status bit and a block-wide abort flag that turns every later wait into an
// immediate return, so all warps still reach every barrier and the final
// TMEM release.
#pragma once

#include "decode_kernels.cuh"
#include "tc05.cuh"

namespace think {

constexpr int kTcGroups = 4;                        // consumer warpgroups (tile i -> i % 4)
constexpr int kTcConsumerThreads = kTcGroups * 128;
constexpr int kTcProducerWarp = kTcGroups * 4;
constexpr int kTcMmaWarp = kTcProducerWarp + 1;
constexpr int kTcThreads = kTcConsumerThreads + 64;
constexpr uint32_t kTcCols = 128;   // S: 4 x 16 columns, O: 4 x 16 columns
constexpr int kTcBufs = 4;          // S, O and P buffers (tile i uses buffer i % 4)

struct TcLayout {
    uint32_t t_pad;   // T rounded up to 16 (one MMA K step)
    uint32_t k_half;  // bytes of one 64-token half of a K' tile: t_pad rows x 128 B
    uint32_t k_slot;  // bytes of one K' ring slot (two halves)
    uint32_t v_off;   // start of the V ring (slots of 128 tokens x 128 channels bf16)
    uint32_t p_off, q_off, red_off, bar_off, total;
};

constexpr uint32_t kVSlot = 32768u;

__host__ __device__ inline TcLayout tc_layout(int T, int sk, int sv)
{
    TcLayout L;
    L.t_pad = (uint32_t)((T + 15) & ~15);
    L.k_half = L.t_pad * 128u;
    L.k_slot = 2u * L.k_half;
    L.v_off = (uint32_t)sk * L.k_slot;
    L.p_off = L.v_off + (uint32_t)sv * kVSlot;  // 4 x (16 rows x 128 tokens) bf16
    L.q_off = L.p_off + 16384u;                 // 16 rows x t_pad bf16
    L.red_off = L.q_off + 32u * L.t_pad;        // tile maxima, totals, warpgroup merge
    L.bar_off = L.red_off + 8192u;
    L.total = L.bar_off + (uint32_t)(2 * sk + 2 * sv + 4 * kTcBufs) * 8u + 16u;
    return L;
}

// Bounded mbarrier wait that honours (and raises) the block's abort flag.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                        unsigned *status, unsigned code)
{
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t spin = 0; spin < kWaitLimitSpins; ++spin) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    *abort_flag = 1u;
    atomicOr(status, code);
    return false;
}

// Byte offset of element (row, col) in a K-major interleaved operand whose
// rows are N (or M) and whose columns are K: 8 x 8 core matrices of 128 B,
// consecutive along K (128 B apart), row groups of 8 `sbo` bytes apart.
__device__ __forceinline__ uint32_t kmajor_off(uint32_t row, uint32_t col, uint32_t sbo)
{
    return (col >> 3) * 128u + (row >> 3) * sbo + (row & 7u) * 16u + (col & 7u) * 2u;
}

// Fold values tile i (TMEM O buffer i % 4, this thread's channel row) into
// the warpgroup's running output: acc = acc * alpha + (O_hi + O_lo), then
// hand the O buffer back to the MMA thread.
template <int G>
__device__ __forceinline__ void tc_accumulate(int i, const float (&al)[G], float (&acc)[G],
                                              uint32_t ofull0, uint32_t ofree0, uint32_t lane_addr,
                                              int lane, volatile uint32_t *abort_flag, unsigned *status)
{
    const int buf = i & 3;
    float ov[16];
    if (tc_wait(ofull0 + 8 * buf, (i >> 2) & 1, abort_flag, status, THINK_DEVICE_TIMEOUT_FULL)) {
        tc05::fence_after_sync();
        tc05::tmem_ld16(lane_addr + 64u + 16u * buf, ov);
    } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) ov[c] = 0.f;
    }
    tc05::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(ofree0 + 8 * buf);
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = fmaf(acc[g], al[g], ov[g] + ov[G + g]);
}

template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    pruned_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a)
{
    static_assert(2 * G <= 16, "hi/lo weights of the group must fit N = 16");
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);

    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int T = a.T;
    const int sk = a.stages, sv = a.stages_v;
    const TcLayout L = tc_layout(T, sk, sv);
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    const uint32_t fullk0 = smem_addr(bars);
    const uint32_t emptyk0 = fullk0 + 8u * sk;
    const uint32_t fullv0 = emptyk0 + 8u * sk;
    const uint32_t emptyv0 = fullv0 + 8u * sv;
    const uint32_t sfull0 = emptyv0 + 8u * sv;
    const uint32_t pfull0 = sfull0 + 8u * kTcBufs;
    const uint32_t ofull0 = pfull0 + 8u * kTcBufs;
    const uint32_t ofree0 = ofull0 + 8u * kTcBufs;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * sk + 2 * sv + 4 * kTcBufs);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    unsigned *flag = tmem_slot + 2;
    float *red = reinterpret_cast<float *>(smem + L.red_off);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < sk; ++s) {
            mbar_init(fullk0 + 8 * s, 1);
            mbar_init(emptyk0 + 8 * s, 1);
        }
        for (int s = 0; s < sv; ++s) {
            mbar_init(fullv0 + 8 * s, 1);
            mbar_init(emptyv0 + 8 * s, 1);
        }
        for (int i = 0; i < kTcBufs; ++i) {
            mbar_init(sfull0 + 8 * i, 1);
            mbar_init(pfull0 + 8 * i, 4);   // the 4 warps of the warpgroup using buffer i
            mbar_init(ofull0 + 8 * i, 1);
            mbar_init(ofree0 + 8 * i, 4);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == kTcMmaWarp) {
        tc05::tmem_alloc(smem_addr(tmem_slot), kTcCols);
        tc05::tmem_relinquish();
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();

    float O[G], M[G], Lsum[G];  // warpgroup 0 results after the merge (d = tid)

    if (warp == kTcProducerWarp) {
        // ------------------------------------------------------ producer
        // Starts at once; the other warps prepare the operands meanwhile (the
        // rows they zero are never written by TMA).
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            const uint32_t ktx = 2u * 64u * (uint32_t)T * 2u;
            int ik = 0, iv = 0, loaded_k = 0, loaded_v = 0;
            uint64_t t_idle = 0;
            uint32_t polls = 0;
            while (iv < ntiles && !*abort_flag) {
                bool progress = false;
                if (ik < ntiles && (ik < sk || mbar_test_wait(emptyk0 + 8 * (ik % sk), ((ik / sk) - 1) & 1))) {
                    const uint32_t full = fullk0 + 8 * (ik % sk);
                    const uint32_t dst = smem_addr(smem + (size_t)(ik % sk) * L.k_slot);
                    const int x = (int)((tile0 + ik) * kBN);
                    mbar_arrive_expect_tx(full, ktx);
                    tma_load_4d(dst, &tm_k, x, 0, kv, b, full);
                    tma_load_4d(dst + L.k_half, &tm_k, x + 64, 0, kv, b, full);
                    loaded_k = ++ik;
                    progress = true;
                }
                if (iv < ik && (iv < sv || mbar_test_wait(emptyv0 + 8 * (iv % sv), ((iv / sv) - 1) & 1))) {
                    const uint32_t full = fullv0 + 8 * (iv % sv);
                    const uint32_t dst = smem_addr(smem + L.v_off + (size_t)(iv % sv) * kVSlot);
                    const int x = (int)((tile0 + iv) * kBN);
                    mbar_arrive_expect_tx(full, kVSlot);
                    tma_load_4d(dst, &tm_v, 0, x, kv, b, full);
                    tma_load_4d(dst + 16384u, &tm_v, 64, x, kv, b, full);
                    loaded_v = ++iv;
                    progress = true;
                }
                if (progress) {
                    polls = 0;
                    continue;
                }
                if ((++polls & 63u) == 0u) {
                    const uint64_t now = global_ns();
                    if (polls == 64u) t_idle = now;
                    else if (now - t_idle > kWaitLimitNs || polls > kWaitLimitSpins) {
                        *abort_flag = 1u;
                        atomicOr(a.status, THINK_DEVICE_TIMEOUT_EMPTY);
                    }
                }
            }
            if (*abort_flag) {
                // Let the loads already in flight land before the block exits.
                for (int i = max(0, loaded_k - sk); i < loaded_k; ++i) {
                    const uint64_t t0 = global_ns();
                    while (!mbar_try_wait(fullk0 + 8 * (i % sk), (i / sk) & 1) && global_ns() - t0 < kWaitLimitNs) {
                    }
                }
                for (int i = max(0, loaded_v - sv); i < loaded_v; ++i) {
                    const uint64_t t0 = global_ns();
                    while (!mbar_try_wait(fullv0 + 8 * (i % sv), (i / sv) & 1) && global_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- operand set-up (consumers + MMA warp)
        // Zero the P and q' operands (their padding rows stay zero) and the K'
        // rows T .. t_pad-1 of every K' slot (TMA writes only rows 0 .. T-1).
        const int nt = kTcConsumerThreads + 32;  // threads taking part here
        const int ti = tid < kTcConsumerThreads ? tid : tid - 32;  // 0 .. nt-1
        {
            uint4 *z = reinterpret_cast<uint4 *>(smem + L.p_off);
            for (uint32_t i = ti; i < (16384u + 32u * L.t_pad) / 16u; i += nt) z[i] = make_uint4(0, 0, 0, 0);
            const uint32_t pad16 = (L.t_pad - (uint32_t)T) * 8u;  // 16-byte words per half
            for (uint32_t i = ti; i < (uint32_t)sk * 2u * pad16; i += nt) {
                const uint32_t half_idx = i / pad16, o = i % pad16;
                *reinterpret_cast<uint4 *>(smem + half_idx * L.k_half + (uint32_t)T * 128u + o * 16u) =
                    make_uint4(0, 0, 0, 0);
            }
        }
        named_barrier(6, nt);
        // q' = q[idx] (bf16, unscaled) as the B operand of the logits MMA: row g, column t.
        {
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
            const int32_t *ih = a.idx + (int64_t)head * T;
            const uint32_t sbo_q = (L.t_pad / 8u) * 128u;
            for (int i = ti; i < T * G; i += nt) {
                const int t = i / G, g = i % G;
                const int c = ih[t];
                __nv_bfloat16 x = __float2bfloat16(0.f);
                if ((unsigned)c < (unsigned)kD) x = q[((int64_t)b * a.Hq + (int64_t)kv * G + g) * kD + c];
                *reinterpret_cast<__nv_bfloat16 *>(smem + L.q_off + kmajor_off(g, t, sbo_q)) = x;
            }
        }
        tc05::fence_proxy_async_smem();
        named_barrier(6, nt);
    }
    const uint32_t tmem = *tmem_slot;

    if (warp == kTcProducerWarp) {
        // done above
    } else if (warp == kTcMmaWarp) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc05::idesc_bf16_f32<128, 16, true>();
            const uint32_t q_addr = smem_addr(smem + L.q_off);
            const uint32_t p_addr = smem_addr(smem + L.p_off);
            const uint32_t sbo_q = (L.t_pad / 8u) * 128u;
            const int ksteps = (int)(L.t_pad / 16u);
            int last_pv = -1, last_qk = -1;
            auto issue_qk = [&](int i) {
                tc05::fence_after_sync();
                const uint32_t kb = smem_addr(smem + (size_t)(i % sk) * L.k_slot);
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint64_t ad = tc05::smem_desc(kb + 2048u * ks, L.k_half, 1024u,
                                                        tc05::kLayoutSwizzle128B);
                    const uint64_t bd = tc05::smem_desc(q_addr + 256u * ks, 128u, sbo_q,
                                                        tc05::kLayoutInterleave);
                    tc05::mma_bf16(tmem + 16u * (i & 3), ad, bd, idesc, ks > 0);
                }
                tc05::commit(sfull0 + 8 * (i & 3));
                tc05::commit(emptyk0 + 8 * (i % sk));
                last_qk = i;
            };
            auto issue_pv = [&](int i) {
                tc05::fence_after_sync();
                const uint32_t vb = smem_addr(smem + L.v_off + (size_t)(i % sv) * kVSlot);
                const uint32_t pb = p_addr + 4096u * (uint32_t)(i & 3);
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint64_t ad =
                        tc05::smem_desc(vb + 2048u * ks, 16384u, 1024u, tc05::kLayoutSwizzle128B);
                    const uint64_t bd =
                        tc05::smem_desc(pb + 256u * ks, 128u, 2048u, tc05::kLayoutInterleave);
                    tc05::mma_bf16(tmem + 64u + 16u * (i & 3), ad, bd, idesc, ks > 0);
                }
                tc05::commit(ofull0 + 8 * (i & 3));
                tc05::commit(emptyv0 + 8 * (i % sv));
                last_pv = i;
            };
            // Event loop: the logits MMA of tile nq as soon as its K' slot has
            // landed and its S buffer is free (the values MMA of tile nq-4 has
            // been issued, which needed the softmax of tile nq-4); the values MMA
            // of tile nv as soon as its V slot has landed, its weights are written
            // and its O buffer has been read.  Neither waits for the other.
            int nq = 0, nv = 0;
            uint64_t t_idle = 0;
            uint32_t polls = 0;
            while (nv < ntiles && !*abort_flag) {
                bool progress = false;
                if (nq < ntiles && nq < nv + kTcBufs && mbar_test_wait(fullk0 + 8 * (nq % sk), (nq / sk) & 1)) {
                    issue_qk(nq++);
                    progress = true;
                }
                if (nv < nq && mbar_test_wait(pfull0 + 8 * (nv & 3), (nv >> 2) & 1) &&
                    (nv < kTcBufs || mbar_test_wait(ofree0 + 8 * (nv & 3), ((nv - 4) >> 2) & 1)) &&
                    mbar_test_wait(fullv0 + 8 * (nv % sv), (nv / sv) & 1)) {
                    issue_pv(nv++);
                    progress = true;
                }
                if (progress) {
                    polls = 0;
                    continue;
                }
                if ((++polls & 63u) == 0u) {
                    const uint64_t now = global_ns();
                    if (polls == 64u) t_idle = now;
                    else if (now - t_idle > kWaitLimitNs || polls > kWaitLimitSpins) {
                        *abort_flag = 1u;
                        atomicOr(a.status, THINK_DEVICE_TIMEOUT_FULL);
                    }
                }
            }
            // No MMA may still run when the block releases its tensor memory:
            // wait for the commits of the last logits and the last values MMA.
            if (last_qk >= 0) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(sfull0 + 8 * (last_qk & 3), (last_qk >> 2) & 1) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
            if (last_pv >= 0) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(ofull0 + 8 * (last_pv & 3), (last_pv >> 2) & 1) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------- softmax + accumulate
        const int wg = warp >> 2;          // warpgroup: tiles i with i % kTcGroups == wg
        const int wq = warp & 3;           // warp within the warpgroup
        const int t = tid & 127;           // TMEM lane: token t / channel t
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        float m[G], lp[G], acc[G], alpha[G], alpha_prev[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            lp[g] = 0.f;
            acc[g] = 0.f;
            alpha[g] = alpha_prev[g] = 1.f;
        }
        const uint32_t sbo_p = 2048u;
        int j = 0;
        for (int i = wg; i < ntiles; i += kTcGroups, ++j) {
            const int sb = i & 3;          // S / P / O buffer of this tile
            float sv[16];
            if (tc_wait(sfull0 + 8 * sb, (i >> 2) & 1, abort_flag, a.status, THINK_DEVICE_TIMEOUT_FULL)) {
                tc05::fence_after_sync();
                tc05::tmem_ld16(lane_addr + 16u * sb, sv);
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) sv[c] = 0.f;
            }
            const bool valid = (tile0 + i) * kBN + t < a.N;
            // tile maxima: [group][j & 1][4 warps][8]; two slots, so one barrier per tile
            float *gred = red + (wg * 2 + (j & 1)) * 32;
            float x[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                x[g] = valid ? sv[g] * a.scale_log2 : -INFINITY;
                const float wm = warp_max(x[g]);
                if (lane == 0) gred[wq * 8 + g] = wm;
            }
            named_barrier(1 + wg, 128);
            float p[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float tmax = gred[g];
#pragma unroll
                for (int w = 1; w < 4; ++w) tmax = fmaxf(tmax, gred[w * 8 + g]);
                const float mnew = fmaxf(m[g], tmax);
                alpha[g] = (m[g] == mnew) ? 1.f : exp2_approx(m[g] - mnew);
                p[g] = valid ? exp2_approx(x[g] - mnew) : 0.f;
                lp[g] = fmaf(lp[g], alpha[g], p[g]);
                m[g] = mnew;
            }
            // this group's previous values tile: done before P is rewritten,
            // which also proves the values MMA that read this P buffer finished
            if (j >= 1)
                tc_accumulate<G>(i - kTcGroups, alpha_prev, acc, ofull0, ofree0, lane_addr, lane,
                                 abort_flag, a.status);
            unsigned char *pbuf = smem + L.p_off + 4096u * (uint32_t)sb;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(p[g]);
                const __nv_bfloat16 lo = __float2bfloat16_rn(p[g] - __bfloat162float(hi));
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmajor_off(g, t, sbo_p)) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmajor_off(G + g, t, sbo_p)) = lo;
            }
            tc05::fence_proxy_async_smem();
            tc05::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull0 + 8 * sb);
#pragma unroll
            for (int g = 0; g < G; ++g) alpha_prev[g] = alpha[g];
        }
        if (j >= 1)
            tc_accumulate<G>(wg + kTcGroups * (j - 1), alpha_prev, acc, ofull0, ofree0, lane_addr, lane,
                             abort_flag, a.status);
        // group totals: sum of the per-thread weight sums
        float *tot = red + 2 * kTcGroups * 32 + wg * 32;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float ws = warp_sum(lp[g]);
            if (lane == 0) tot[wq * 8 + g] = ws;
        }
        named_barrier(1 + wg, 128);
        float l[G];
#pragma unroll
        for (int g = 0; g < G; ++g) l[g] = (tot[g] + tot[8 + g]) + (tot[16 + g] + tot[24 + g]);
        // merge groups 1.. into group 0 (same channel t).  Once every group has
        // passed its last accumulation, every values MMA has completed and the
        // V ring is free for the exchange.
        named_barrier(5, kTcConsumerThreads);
        float *xo = reinterpret_cast<float *>(smem + L.v_off);   // [group-1][128][G]
        float *xm = xo + (kTcGroups - 1) * 128 * G;             // [group-1][2G]
        if (wg > 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) xo[((wg - 1) * 128 + t) * G + g] = acc[g];
            if (t == 0) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    xm[(wg - 1) * 2 * G + g] = m[g];
                    xm[(wg - 1) * 2 * G + G + g] = l[g];
                }
            }
        }
        named_barrier(5, kTcConsumerThreads);
        if (wg == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float mx = m[g];
#pragma unroll
                for (int w = 1; w < kTcGroups; ++w) mx = fmaxf(mx, xm[(w - 1) * 2 * G + g]);
                float s0 = (m[g] == -INFINITY) ? 0.f : exp2_approx(m[g] - mx);
                float Ls = l[g] * s0, Os = acc[g] * s0;
#pragma unroll
                for (int w = 1; w < kTcGroups; ++w) {
                    const float mw = xm[(w - 1) * 2 * G + g];
                    const float sw = (mw == -INFINITY) ? 0.f : exp2_approx(mw - mx);
                    Ls = fmaf(xm[(w - 1) * 2 * G + G + g], sw, Ls);
                    Os = fmaf(xo[((w - 1) * 128 + t) * G + g], sw, Os);
                }
                M[g] = mx;
                Lsum[g] = Ls;
                O[g] = Os;
            }
        }
    }

    // every tcgen05 operation of the block has completed: release tensor memory
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, kTcCols);
    }
    if (warp < 4 * kTcGroups)   // warpgroup 0 holds the block's partial; all groups merge
        finish_split<G, kTcConsumerThreads>(a, head, split, b, kv, tid, O, M, Lsum,
                                            reinterpret_cast<float *>(smem), flag, 5);
}

}  // namespace think

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
// Warp roles per block (192 threads):
//   warps 0-3  softmax + accumulate: thread t reads TMEM lane t, i.e. token t
//              of the logits tile and channel t of the value tile;
//   warp 4     TMA producer (one elected thread);
//   warp 5     TMEM allocator and MMA issuer (one elected thread).
// TMEM: S double buffer (columns 0-31) and O double buffer (columns 32-63).
// The MMA thread issues the logits of tile i+1 before the values of tile i,
// so the tensor core works on the next tile while the softmax runs.
// Every mbarrier wait is bounded; a wait that runs out sets the workspace
// status bit and a block-wide abort flag that turns every later wait into an
// immediate return, so all warps still reach every barrier and the final
// TMEM release.
#pragma once

#include "decode_kernels.cuh"
#include "tc05.cuh"

namespace think {

constexpr int kTcThreads = 192;
constexpr uint32_t kTcCols = 64;

struct TcLayout {
    uint32_t t_pad;   // T rounded up to 16 (one MMA K step)
    uint32_t k_half;  // bytes of one 64-token half of the K' tile: t_pad rows x 128 B
    uint32_t stage;   // bytes per ring stage: K' (2 halves) + V (2 halves of 128 x 128 B)
    uint32_t p_off, q_off, red_off, bar_off, total;
};

__host__ __device__ inline TcLayout tc_layout(int T, int stages)
{
    TcLayout L;
    L.t_pad = (uint32_t)((T + 15) & ~15);
    L.k_half = L.t_pad * 128u;
    L.stage = 2u * L.k_half + 32768u;
    L.p_off = (uint32_t)stages * L.stage;       // 2 x (16 rows x 128 tokens) bf16
    L.q_off = L.p_off + 8192u;                  // 16 rows x t_pad bf16
    L.red_off = L.q_off + 32u * L.t_pad;        // [3][4 warps][8] floats
    L.bar_off = L.red_off + 512u;
    L.total = L.bar_off + (uint32_t)(2 * stages + 8) * 8u + 16u;
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

// Fold the values tile i (TMEM O buffer i % 2, this thread's channel row)
// into the running output: acc = acc * alpha_i + (O_hi + O_lo), then hand
// the O buffer back to the MMA thread.
template <int G>
__device__ __forceinline__ void tc_accumulate(int i, const float (&al)[G], float (&acc)[G],
                                              uint32_t ofull0, uint32_t ofree0, uint32_t lane_addr,
                                              int lane, volatile uint32_t *abort_flag, unsigned *status)
{
    float ov[16];
    if (tc_wait(ofull0 + 8 * (i & 1), (i >> 1) & 1, abort_flag, status, THINK_DEVICE_TIMEOUT_FULL)) {
        tc05::fence_after_sync();
        tc05::tmem_ld16(lane_addr + 32u + 16u * (i & 1), ov);
    } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) ov[c] = 0.f;
    }
    tc05::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(ofree0 + 8 * (i & 1));
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = fmaf(acc[g], al[g], ov[g] + ov[G + g]);
}

template <int G>
__global__ void __launch_bounds__(kTcThreads)
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
    const int stages = a.stages;
    const TcLayout L = tc_layout(T, stages);
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = full0 + 8u * stages;
    const uint32_t sfull0 = empty0 + 8u * stages;
    const uint32_t pfull0 = sfull0 + 16u;
    const uint32_t ofull0 = pfull0 + 16u;
    const uint32_t ofree0 = ofull0 + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * stages + 8);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    unsigned *flag = tmem_slot + 2;
    float *red = reinterpret_cast<float *>(smem + L.red_off);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(sfull0 + 8 * i, 1);
            mbar_init(pfull0 + 8 * i, kConsumerWarps);
            mbar_init(ofull0 + 8 * i, 1);
            mbar_init(ofree0 + 8 * i, kConsumerWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 5) {
        tc05::tmem_alloc(smem_addr(tmem_slot), kTcCols);
        tc05::tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    // Zero the P and q' operands (their padding rows stay zero) and the K'
    // rows T .. t_pad-1 of every stage (TMA writes only rows 0 .. T-1).
    {
        uint4 *z = reinterpret_cast<uint4 *>(smem + L.p_off);
        for (uint32_t i = tid; i < (8192u + 32u * L.t_pad) / 16u; i += kTcThreads)
            z[i] = make_uint4(0, 0, 0, 0);
        const uint32_t pad_bytes = (L.t_pad - (uint32_t)T) * 128u;
        const uint32_t per_stage = 2u * pad_bytes / 16u;
        for (uint32_t i = tid; i < (uint32_t)stages * per_stage; i += kTcThreads) {
            const uint32_t s = i / per_stage, r = i % per_stage;
            const uint32_t half = r / (pad_bytes / 16u), o = r % (pad_bytes / 16u);
            *reinterpret_cast<uint4 *>(smem + s * L.stage + half * L.k_half + (uint32_t)T * 128u + o * 16u) =
                make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    // q' = q[idx] (bf16, unscaled) as the B operand of the logits MMA: row g, column t.
    {
        const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
        const int32_t *ih = a.idx + (int64_t)head * T;
        const uint32_t sbo_q = (L.t_pad / 8u) * 128u;
        for (int i = tid; i < T * G; i += kTcThreads) {
            const int t = i / G, g = i % G;
            const int c = ih[t];
            __nv_bfloat16 x = __float2bfloat16(0.f);
            if ((unsigned)c < (unsigned)kD) x = q[((int64_t)b * a.Hq + (int64_t)kv * G + g) * kD + c];
            *reinterpret_cast<__nv_bfloat16 *>(smem + L.q_off + kmajor_off(g, t, sbo_q)) = x;
        }
    }
    tc05::fence_proxy_async_smem();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    float O[G], M[G], Lsum[G];  // consumer results (d = tid)

    if (warp == 4) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t tx = 2u * 64u * (uint32_t)T * 2u + 2u * 64u * 128u * 2u;
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % stages, f = it / stages;
                if (f > 0 && !tc_wait(empty0 + 8 * s, (f - 1) & 1, abort_flag, a.status,
                                      THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                const uint32_t full = full0 + 8 * s;
                mbar_arrive_expect_tx(full, tx);
                const int x = (int)((tile0 + it) * kBN);
                const uint32_t st = smem_addr(smem + (size_t)s * L.stage);
                tma_load_4d(st, &tm_k, x, 0, kv, b, full);
                tma_load_4d(st + L.k_half, &tm_k, x + 64, 0, kv, b, full);
                tma_load_4d(st + 2u * L.k_half, &tm_v, 0, x, kv, b, full);
                tma_load_4d(st + 2u * L.k_half + 16384u, &tm_v, 64, x, kv, b, full);
                ++issued;
            }
            if (*abort_flag) {
                // Let the loads already in flight land before the block exits.
                for (int it = max(0, issued - stages); it < issued; ++it) {
                    const uint64_t t0 = global_ns();
                    while (!mbar_try_wait(full0 + 8 * (it % stages), (it / stages) & 1) &&
                           global_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc05::idesc_bf16_f32<128, 16, true>();
            const uint32_t q_addr = smem_addr(smem + L.q_off);
            const uint32_t p_addr = smem_addr(smem + L.p_off);
            const uint32_t sbo_q = (L.t_pad / 8u) * 128u;
            const int ksteps = (int)(L.t_pad / 16u);
            int last_pv = -1, last_qk = -1;
            auto issue_qk = [&](int i) -> bool {
                const int s = i % stages;
                if (!tc_wait(full0 + 8 * s, (i / stages) & 1, abort_flag, a.status,
                             THINK_DEVICE_TIMEOUT_FULL))
                    return false;
                tc05::fence_after_sync();
                const uint32_t kb = smem_addr(smem + (size_t)s * L.stage);
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint64_t ad = tc05::smem_desc(kb + 2048u * ks, L.k_half, 1024u,
                                                        tc05::kLayoutSwizzle128B);
                    const uint64_t bd = tc05::smem_desc(q_addr + 256u * ks, 128u, sbo_q,
                                                        tc05::kLayoutInterleave);
                    tc05::mma_bf16(tmem + 16u * (i & 1), ad, bd, idesc, ks > 0);
                }
                tc05::commit(sfull0 + 8 * (i & 1));
                last_qk = i;
                return true;
            };
            bool ok = ntiles > 0 && issue_qk(0);
            for (int i = 0; ok && i < ntiles; ++i) {
                if (i + 1 < ntiles && !issue_qk(i + 1)) break;
                if (!tc_wait(pfull0 + 8 * (i & 1), (i >> 1) & 1, abort_flag, a.status,
                             THINK_DEVICE_TIMEOUT_FULL))
                    break;
                if (i >= 2 && !tc_wait(ofree0 + 8 * (i & 1), ((i - 2) >> 1) & 1, abort_flag, a.status,
                                       THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                tc05::fence_after_sync();
                const int s = i % stages;
                const uint32_t vb = smem_addr(smem + (size_t)s * L.stage + 2u * L.k_half);
                const uint32_t pb = p_addr + 4096u * (i & 1);
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint64_t ad =
                        tc05::smem_desc(vb + 2048u * ks, 16384u, 1024u, tc05::kLayoutSwizzle128B);
                    const uint64_t bd =
                        tc05::smem_desc(pb + 256u * ks, 128u, 2048u, tc05::kLayoutInterleave);
                    tc05::mma_bf16(tmem + 32u + 16u * (i & 1), ad, bd, idesc, ks > 0);
                }
                tc05::commit(ofull0 + 8 * (i & 1));
                tc05::commit(empty0 + 8 * s);
                last_pv = i;
            }
            // No MMA may still run when the block releases its tensor memory:
            // wait for the commits of the last logits and the last values MMA.
            if (last_qk >= 0) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(sfull0 + 8 * (last_qk & 1), (last_qk >> 1) & 1) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
            if (last_pv >= 0) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(ofull0 + 8 * (last_pv & 1), (last_pv >> 1) & 1) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------- softmax + accumulate
        const int t = tid;  // TMEM lane: token t of a logits tile, channel t of a value tile
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float m[G], lp[G], acc[G], alpha[G], alpha_prev[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            lp[g] = 0.f;
            acc[g] = 0.f;
            alpha[g] = alpha_prev[g] = 1.f;
        }
        const uint32_t sbo_p = 2048u;
        for (int i = 0; i < ntiles; ++i) {
            const int bi = i & 1;
            float sv[16];
            if (tc_wait(sfull0 + 8 * bi, (i >> 1) & 1, abort_flag, a.status, THINK_DEVICE_TIMEOUT_FULL)) {
                tc05::fence_after_sync();
                tc05::tmem_ld16(lane_addr + 16u * bi, sv);
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) sv[c] = 0.f;
            }
            const bool valid = (tile0 + i) * kBN + t < a.N;
            float x[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                x[g] = valid ? sv[g] * a.scale_log2 : -INFINITY;
                const float wm = warp_max(x[g]);
                if (lane == 0) red[(bi * 4 + warp) * 8 + g] = wm;
            }
            named_barrier(1, kConsumerThreads);
            unsigned char *pbuf = smem + L.p_off + 4096u * bi;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float tmax = red[(bi * 4 + 0) * 8 + g];
#pragma unroll
                for (int w = 1; w < kConsumerWarps; ++w) tmax = fmaxf(tmax, red[(bi * 4 + w) * 8 + g]);
                const float mnew = fmaxf(m[g], tmax);
                alpha[g] = (m[g] == mnew) ? 1.f : exp2_approx(m[g] - mnew);
                const float p = valid ? exp2_approx(x[g] - mnew) : 0.f;
                lp[g] = fmaf(lp[g], alpha[g], p);
                m[g] = mnew;
                const __nv_bfloat16 hi = __float2bfloat16_rn(p);
                const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmajor_off(g, t, sbo_p)) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmajor_off(G + g, t, sbo_p)) = lo;
            }
            tc05::fence_proxy_async_smem();
            tc05::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull0 + 8 * bi);
            if (i >= 1)
                tc_accumulate<G>(i - 1, alpha_prev, acc, ofull0, ofree0, lane_addr, lane, abort_flag,
                                 a.status);
#pragma unroll
            for (int g = 0; g < G; ++g) alpha_prev[g] = alpha[g];
        }
        if (ntiles >= 1)
            tc_accumulate<G>(ntiles - 1, alpha_prev, acc, ofull0, ofree0, lane_addr, lane, abort_flag,
                             a.status);
        // block totals: sum of the per-thread weight sums (third slot of `red`,
        // untouched by the per-tile maxima)
        float *tot = red + 64;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float ws = warp_sum(lp[g]);
            if (lane == 0) tot[warp * 8 + g] = ws;
        }
        named_barrier(1, kConsumerThreads);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            Lsum[g] = (tot[0 * 8 + g] + tot[1 * 8 + g]) + (tot[2 * 8 + g] + tot[3 * 8 + g]);
            M[g] = m[g];
            O[g] = acc[g];
        }
    }

    // every tcgen05 operation of the block has completed: release tensor memory
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, kTcCols);
    }
    if (warp < kConsumerWarps)
        finish_split<G>(a, head, split, b, kv, tid, O, M, Lsum, reinterpret_cast<float *>(smem), flag);
}

}  // namespace think

// mass_tc.cuh -- the window attention mass of every token (token eviction
// composed with channel pruning) on the 5th-generation tensor cores.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", abstract: the pruned
// cache combines with KV-cache eviction; the Keyformer page keeps the tokens
// that receive the most attention.  Per KV head, with the R = G * S_obs
// window rows of the group,
//     mass[n] = sum_r softmax_n(scale * Qwin[r] . K[n])
// (the same quantity as token_mass_kernel, evict.cuh).
//
// Per 128-token tile the logits of the window rows are a dense product,
//     D_m[row][tok] = Q_m[row][:] . K[tok][:]    M = 128 rows, N = 128 tokens, K = 128 channels,
// for MB = ceil(R / 128) blocks m of 128 rows.  One thread issues it as
// tcgen05.mma with both operands K-major in shared memory: Q staged once per
// block with the 128-byte swizzle (rows >= R zero), each K tile by TMA with
// the same swizzle (two 64-channel halves), accumulators in tensor memory in
// two buffers of MB x 128 fp32 columns, so the MMA of tile i + 1 runs while
// the softmax warps work on tile i.  Pass 1: two softmax warpgroups per row
// block m read its TMEM lanes: thread t of warpgroup 2 m + hh holds row
// 128 m + t and the tile's tokens 64 hh .. 64 hh + 63 (the column half).
//   pass 1: per row, the maximum z and the sum of 2^(z - max) over the block's
//           tokens (the sum rescaled only when the maximum grows), the two
//           halves of a row merged at the end, then the head's last block
//           merges the splits into (max, 1 / sum);
//   pass 2: the product transposed, D[token][row] (M = 128 tokens, N = 128 MB
//           rows), with one extra K step that adds -off_r / sl to every row
//           (off_r = max_r + log2(sum_r), its bf16 parts against channels of
//           ones), so that a token's weights 2^(sl D) lie in one TMEM lane:
//           each thread sums 64 rows of its token, then the four (MB = 1: two)
//           row groups are added in order.
// Warps: 8 MB softmax warps, one TMA producer warp, one MMA warp (which also
// owns the tensor memory).  Every wait is bounded; a wait that runs out sets
// the status bit and a block abort flag, and every warp still reaches the
// final barrier, after which the tensor memory is released.
#pragma once

#include "decode_tc.cuh"
#include "evict.cuh"
#include "tc05.cuh"

namespace think {

template <int MB>
struct MassTc {
    static constexpr int kSoftWarps = 8 * MB;      // per row block: 4 lane quarters x 2 column halves
    static constexpr int kSoftThreads = 32 * kSoftWarps;
    static constexpr int kProdWarp = kSoftWarps;
    static constexpr int kMmaWarp = kSoftWarps + 1;
    static constexpr int kThreads = kSoftThreads + 64;
    static constexpr uint32_t kCols = 2u * MB * 128u;  // two accumulator buffers
};

// shared memory: K ring (stages x 32 KB), Q (MB x 32 KB), pass 2's extra K
// step operands (4 KB + MB x 4 KB), per-warp token sums [softmax warps][64]
// fp32, the upper column halves' pass-1 row partials [MB * 128] float2,
// mbarriers (K full/empty per stage, accumulator full/empty per buffer), the
// TMEM address, an abort flag, a flag, alignment slack
template <int MB>
__host__ __device__ inline size_t mass_tc_smem_bytes(int stages)
{
    return (size_t)stages * 32768u + (size_t)MB * 32768u + 4096u + (size_t)MB * 4096u +
           (size_t)MassTc<MB>::kSoftWarps * 64u * 4u + (size_t)MB * 128u * 8u + (size_t)(2 * stages + 4) * 8u +
           16u + 1024u;
}

template <int PASS, int MB>
__global__ void __launch_bounds__(MassTc<MB>::kThreads, 1)
    token_mass_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const MassArgs a)
{
    using C = MassTc<MB>;
    constexpr int NT = C::kSoftThreads;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);
    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int stages = a.stages;
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)max((int64_t)0, min((int64_t)a.tiles_per_split, tiles_all - tile0));

    unsigned char *qs = smem + (size_t)stages * 32768u;                         // [2 halves][MB * 128 rows][128 B]
    unsigned char *xa = qs + (size_t)MB * 32768u;                               // pass 2: [128 tokens][16] bf16
    unsigned char *xb = xa + 4096u;                                             // pass 2: [MB * 128 rows][16] bf16
    float *tsum = reinterpret_cast<float *>(xb + (size_t)MB * 4096u);           // [softmax warps][64]
    float2 *rhalf = reinterpret_cast<float2 *>(tsum + C::kSoftWarps * 64);      // [MB * 128] pass 1, upper half
    uint64_t *bars = reinterpret_cast<uint64_t *>(rhalf + MB * 128);
    const uint32_t kfull0 = smem_addr(bars);
    const uint32_t kempty0 = kfull0 + 8u * (uint32_t)stages;
    const uint32_t dfull0 = kempty0 + 8u * (uint32_t)stages;
    const uint32_t dempty0 = dfull0 + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * stages + 4);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    unsigned *flag = tmem_slot + 2;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(kfull0 + 8 * s, 1);
            mbar_init(kempty0 + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(dfull0 + 8 * i, 1);
            mbar_init(dempty0 + 8 * i, C::kSoftWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == C::kMmaWarp) {
        tc05::tmem_alloc(smem_addr(tmem_slot), C::kCols);
        tc05::tmem_relinquish();
    }
    // the window rows r = g * S + s of the group (rows >= R zero), K-major with
    // the 128-byte swizzle: channel half h at qs + h * MB * 16 KB, row r at
    // + 128 r (rows of both row blocks contiguous, 8-row atoms 1 KB apart)
    for (int i = tid; i < MB * 128 * 16; i += C::kThreads) {
        const int r = i >> 4, c16 = i & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < a.R) {
            const int g = r / a.S, s = r % a.S;
            v = *reinterpret_cast<const uint4 *>(
                a.qwin + (((int64_t)b * a.Hq + (int64_t)kv * a.G + g) * a.S + s) * kD + 8 * c16);
        }
        *reinterpret_cast<uint4 *>(qs + (size_t)(c16 >> 3) * (MB * 16384u) + (uint32_t)r * 128u +
                                   ((((uint32_t)c16 & 7u) ^ ((uint32_t)r & 7u)) << 4)) = v;
    }
    if (PASS == 2) {
        // The extra K step of pass 2's product: token t's 16 extra channels
        // are (1, 1, 1, 0, ...), row r's are the bf16 parts of -off_r / sl,
        // off_r = max_r + log2(sum_r), so that the accumulator holds
        // z - off_r / sl and the weight is 2^(sl * that).  Rows >= R get a
        // large finite negative value (weight 0).  K-major, no swizzle (core
        // matrices of 8 rows x 8 channels, 128 B; the two along K 128 B apart,
        // row groups 256 B apart).
        const float sl = a.scale_log2;
        for (int i = tid; i < 128 * 16; i += C::kThreads) {
            const int t = i >> 4, c = i & 15;
            *reinterpret_cast<__nv_bfloat16 *>(xa + kmajor_off((uint32_t)t, (uint32_t)c, 256u)) =
                __float2bfloat16_rn(c < 3 ? 1.f : 0.f);
        }
        for (int r = tid; r < MB * 128; r += C::kThreads) {
            float x = -1.0e30f;
            if (r < a.R) {
                const float2 st = __ldcg(a.stats + (int64_t)head * a.R + r);  // (max, 1 / sum)
                x = -(st.x - log2f(st.y)) / sl;
            }
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const float r1 = x - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<__nv_bfloat16 *>(xb + kmajor_off((uint32_t)r, (uint32_t)c, 256u)) =
                    c == 0 ? hi : c == 1 ? mid : c == 2 ? lo : z;
        }
    }
    tc05::fence_proxy_async_smem();  // Q written by threads -> read by the tensor core
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    float row_m = -INFINITY, row_l = 0.f;  // pass 1: this thread's row
    if (warp == C::kProdWarp) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % stages;
                if (it >= stages &&
                    !tc_wait(kempty0 + 8 * s, ((it / stages) - 1) & 1, abort_flag, a.status, THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                const uint32_t full = kfull0 + 8 * s;
                const uint32_t dst = smem_addr(smem + (size_t)s * 32768u);
                const int x = (int)((tile0 + it) * kBN);
                mbar_arrive_expect_tx(full, 32768u);
                tma_load_4d(dst, &tm_k, 0, x, kv, b, full);
                tma_load_4d(dst + 16384u, &tm_k, 64, x, kv, b, full);
                ++issued;
            }
            if (*abort_flag)  // the loads in flight land before the block ends
                for (int it = max(0, issued - stages); it < issued; ++it)
                    mbar_wait_bounded(kfull0 + 8 * (it % stages), (it / stages) & 1, a.status,
                                      THINK_DEVICE_TIMEOUT_FULL);
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // pass 1: D[row][token], one MMA per row block (M = 128 rows, N = 128 tokens);
            // pass 2: D[token][row] (M = 128 tokens, N = MB * 128 rows) plus the extra K step
            constexpr uint32_t idesc = PASS == 1 ? tc05::idesc_bf16_f32<128, 128, false>()
                                                 : tc05::idesc_bf16_f32<128, 128 * MB, false>();
            const uint32_t q_addr = smem_addr(qs);
            int last = -1;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % stages, buf = it & 1;
                if (!tc_wait(kfull0 + 8 * s, (it / stages) & 1, abort_flag, a.status, THINK_DEVICE_TIMEOUT_FULL))
                    break;
                if (it >= 2 && !tc_wait(dempty0 + 8 * buf, ((it >> 1) - 1) & 1, abort_flag, a.status,
                                        THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                tc05::fence_after_sync();
                const uint32_t kb = smem_addr(smem + (size_t)s * 32768u);
                if constexpr (PASS == 1) {
#pragma unroll
                    for (int m = 0; m < MB; ++m) {
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            // 16 channels: half ks / 4, 32 bytes into each 128-byte row
                            const uint32_t ko = (uint32_t)(ks & 3) * 32u;
                            const uint64_t ad = tc05::smem_desc(q_addr + (uint32_t)(ks >> 2) * (MB * 16384u) +
                                                                    (uint32_t)m * 16384u + ko,
                                                                16u, 1024u, tc05::kLayoutSwizzle128B);
                            const uint64_t bd = tc05::smem_desc(kb + (uint32_t)(ks >> 2) * 16384u + ko, 16u, 1024u,
                                                                tc05::kLayoutSwizzle128B);
                            tc05::mma_bf16(tmem + (uint32_t)(buf * MB + m) * 128u, ad, bd, idesc, ks > 0);
                        }
                    }
                } else {
                    const uint32_t d = tmem + (uint32_t)buf * (MB * 128u);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t ko = (uint32_t)(ks & 3) * 32u;
                        const uint64_t ad = tc05::smem_desc(kb + (uint32_t)(ks >> 2) * 16384u + ko, 16u, 1024u,
                                                            tc05::kLayoutSwizzle128B);
                        const uint64_t bd = tc05::smem_desc(q_addr + (uint32_t)(ks >> 2) * (MB * 16384u) + ko, 16u,
                                                            1024u, tc05::kLayoutSwizzle128B);
                        tc05::mma_bf16(d, ad, bd, idesc, ks > 0);
                    }
                    tc05::mma_bf16(d, tc05::smem_desc(smem_addr(xa), 128u, 256u, tc05::kLayoutInterleave),
                                   tc05::smem_desc(smem_addr(xb), 128u, 256u, tc05::kLayoutInterleave), idesc, true);
                }
                tc05::commit(dfull0 + 8 * buf);
                tc05::commit(kempty0 + 8 * s);
                last = it;
            }
            // no MMA may still run when the tensor memory is released
            if (last >= 0) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(dfull0 + 8 * (last & 1), (last >> 1) & 1) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- softmax warps
        // Every softmax warp runs every tile's iteration, so that the named
        // barriers of pass 2 always match; after an abort (tc_wait then
        // returns false at once) the iterations only pass the barriers.
        // pass 1: warp w = 8 m + 4 hh + wq holds rows 128 m + 32 wq + lane and
        //         the tile's tokens 64 hh .. 64 hh + 63;
        // pass 2: warp w = 4 cg + wq holds token 32 wq + lane of the tile and
        //         the rows 64 cg .. 64 cg + 63.
        const int wq = warp & 3, hi = warp >> 2;  // hi: 2 m + hh (pass 1), cg (pass 2)
        const int m = hi >> 1, hh = hi & 1;
        const int row = 128 * m + 32 * wq + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        const float sl = a.scale_log2;
        for (int it = 0; it < ntiles; ++it) {
            const int buf = it & 1;
            float v[64];
            const bool ok = __all_sync(0xffffffffu, tc_wait(dfull0 + 8 * buf, (it >> 1) & 1, abort_flag, a.status,
                                                            THINK_DEVICE_TIMEOUT_FULL));
            if (ok) {
                tc05::fence_after_sync();
                uint32_t r[4][16];
                const uint32_t col = PASS == 1 ? lane_addr + (uint32_t)(buf * MB + m) * 128u + 64u * (uint32_t)hh
                                               : lane_addr + (uint32_t)buf * (MB * 128u) + 64u * (uint32_t)hi;
#pragma unroll
                for (int j = 0; j < 4; ++j) tc05::tmem_ld16_issue(col + 16u * j, r[j]);
#pragma unroll
                for (int j = 0; j < 4; ++j) tc05::tmem_ld_wait(r[j]);
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int q = 0; q < 16; ++q) v[16 * j + q] = __uint_as_float(r[j][q]);
                tc05::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty0 + 8 * buf);  // the accumulator buffer may be rewritten
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) v[c] = 0.f;
            }
            const int64_t tok0 = (tile0 + it) * kBN;
            if constexpr (PASS == 1) {
                // valid columns of this thread's half
                const int nvalid = ok ? (int)max((int64_t)0, min((int64_t)64, a.N - tok0 - 64 * hh)) : 0;
                float tmax = -INFINITY, l = 0.f;
                if (nvalid == 64) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) tmax = fmaxf(tmax, v[c] * sl);
                } else {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < nvalid) tmax = fmaxf(tmax, v[c] * sl);
                }
                if (tmax > row_m) {
                    row_l *= exp2_approx(row_m - tmax);  // 0 while the row has no tokens yet
                    row_m = tmax;
                }
                if (nvalid == 64) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) l += exp2_approx(v[c] * sl - row_m);
                } else {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < nvalid) l += exp2_approx(v[c] * sl - row_m);
                }
                row_l += l;
            } else {
                // the token's weights over these 64 rows (the accumulator
                // holds z - off / sl; rows >= R give 0), summed in row order
                const int tok = 32 * wq + lane;
                float x = 0.f;
                if (ok && tok0 + tok < a.N) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) x += exp2_approx(v[c] * sl);
                }
                tsum[hi * kBN + tok] = x;
                named_barrier(1, NT);
                // token t: its row groups' sums in order
                if (tid < kBN && tok0 + tid < a.N && !*abort_flag) {
                    float y = 0.f;
#pragma unroll
                    for (int g2 = 0; g2 < 2 * MB; ++g2) y += tsum[g2 * kBN + tid];
                    a.mass[(int64_t)head * a.N + tok0 + tid] = y;
                }
                named_barrier(1, NT);  // tsum is read before the next tile rewrites it
            }
        }
        if (PASS == 1 && hh == 1) rhalf[row] = make_float2(row_m, row_l);  // to the thread of the lower half
    }

    // every tcgen05 operation of the block has completed: release tensor memory
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == C::kMmaWarp) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tmem, C::kCols);
    }
    if constexpr (PASS == 1) {
        if (tid < NT) {
            // the two column halves of a row (threads of the lower half merge),
            // then the block's row partials and the split merge
            const int w = tid >> 5, m = w >> 3, hh = (w >> 2) & 1, wq = w & 3;
            const int row = 128 * m + 32 * wq + (tid & 31);
            if (hh == 0 && row < a.R) {
                const float2 o = rhalf[row];
                const float mx = fmaxf(row_m, o.x);
                const float mref = mx == -INFINITY ? 0.f : mx;
                const float l = row_l * exp2_approx(row_m - mref) + o.y * exp2_approx(o.x - mref);
                a.part[((int64_t)head * a.splits + split) * a.R + row] = make_float2(mx, l);
            }
            mass_merge_splits<NT>(a, head, tid, flag);
        }
    }
}

}  // namespace think

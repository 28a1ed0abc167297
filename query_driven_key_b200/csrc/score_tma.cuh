// score_tma.cuh -- the channel-energy pass of the prune for bf16 keys, with
// the key tiles staged in shared memory by TMA.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): every key channel is rated against the query window,
// s[c] = ||Q_win[:, c]|| * ||K[:, c]||; this pass reads K once for the
// ||K[:, c]||^2 of every channel.
//
// The pass only streams K (N * 128 * 2 bytes per head) and adds squares, so it
// is bound by HBM.  score_kernel keeps its loads in registers (about 8 loads
// of 16 bytes per thread in flight); here one producer thread per block keeps
// a ring of 16 KB tiles in flight by TMA (the two 64-channel halves of a
// 64-token tile, 128-byte swizzle), so the bytes in flight per SM are set by
// the ring, not by registers.  The arithmetic is that of score_kernel bit for
// bit: the same split plan and blocks (split, head), the same thread -> (row
// group, channel chunk) map (rows rg, rg + 16, rg + 32, rg + 48 of each tile,
// channels 8cc .. 8cc + 7), add_squares4_bf16 in tile order, the same block
// partial and the same last-block merge (score_block_end).  Rows past N come
// from TMA's zero fill and add nothing, as the zero words of score_kernel do.
//
// Every wait is bounded: on expiry the kernel sets a bit in the status word,
// stops its loop, and the producer waits (bounded) for its loads in flight
// before the ring is reused or the block ends.
#pragma once

#include "prune_kernels.cuh"
#include "think.h"

namespace think {

constexpr int kStConsumerWarps = 8;
constexpr int kStThreads = 32 * kStConsumerWarps + 32;   // + one producer warp
constexpr int kStTileRows = 64;
constexpr uint32_t kStHalfBytes = 64u * 64u * 2u;        // 64 tokens x 64 channels x bf16
constexpr uint32_t kStTileBytes = 2u * kStHalfBytes;
constexpr int kStMaxStages = 8;

// Dynamic shared memory: the ring (stages x 16 KB, 1024-byte aligned for the
// swizzle; after the loop its first 16 KB hold the [16][128] fp64 partials),
// then full[stages] and empty[stages] mbarriers, plus alignment slack.
inline size_t score_tma_smem_bytes(int stages)
{
    return (size_t)stages * kStTileBytes + 2u * (size_t)stages * 8u + 1024u;
}

__global__ void __launch_bounds__(kStThreads, 3)
    score_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a)
{
    extern __shared__ unsigned char st_smem_dyn[];
    unsigned char *smem = st_smem_dyn + ((1024u - (smem_addr(st_smem_dyn) & 1023u)) & 1023u);
    const int stages = a.stages;
    const uint32_t ring = smem_addr(smem);
    const uint32_t full0 = ring + (uint32_t)stages * kStTileBytes;
    const uint32_t empty0 = full0 + 8u * (uint32_t)stages;

    const int head = blockIdx.y;
    const int split = blockIdx.x;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int tid = threadIdx.x;
    const int64_t n0 = (int64_t)split * a.rows_per_split;
    const int64_t n1 = min(a.N, n0 + a.rows_per_split);
    const int tile0 = (int)(n0 / kStTileRows);
    const int ntiles = (int)((n1 - n0 + kStTileRows - 1) / kStTileRows);

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kStConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    // the compaction that follows in think_prune may start its loads of K
    // on the SMs that this grid leaves idle at its end
    grid_launch_dependents();

    // consumer thread -> row group and 16-byte channel chunk, as in score_kernel
    const int cc = tid & 15, rg = tid >> 4;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;

    if (tid >= 32 * kStConsumerWarps) {
        if (tid == 32 * kStConsumerWarps) {
            prefetch_tensormap(&tm_k);
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % stages, f = i / stages;
                if (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)((f - 1) & 1), a.status,
                                                THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                const uint32_t full = full0 + 8 * s;
                const uint32_t dst = ring + (uint32_t)s * kStTileBytes;
                const int row = (tile0 + i) * kStTileRows;
                mbar_arrive_expect_tx(full, kStTileBytes);
                tma_load_4d(dst, &tm_k, 0, row, kv, b, full);
                tma_load_4d(dst + kStHalfBytes, &tm_k, 64, row, kv, b, full);
                ++issued;
            }
            // every load issued has landed before the ring is reused below
            for (int i = max(0, issued - stages); i < issued; ++i)
                mbar_wait_bounded(full0 + 8 * (i % stages), (uint32_t)((i / stages) & 1), a.status,
                                  THINK_DEVICE_TIMEOUT_FULL);
        }
        __syncwarp();
    } else {
        score_window_energies<__nv_bfloat16>(a, head, split);
        const int lane = tid & 31;
        const uint32_t half = (uint32_t)(cc >> 3) * kStHalfBytes;
        const uint32_t chunk = (uint32_t)(cc & 7);
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % stages;
            if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((i / stages) & 1), a.status,
                                   THINK_DEVICE_TIMEOUT_FULL))
                break;
            const uint32_t st = ring + (uint32_t)s * kStTileBytes + half;
            uint4 w[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const uint32_t row = (uint32_t)(rg + 16 * k4);
                const uint32_t addr = st + row * 128u + ((chunk ^ (row & 7u)) << 4);
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[k4].x), "=r"(w[k4].y), "=r"(w[k4].z), "=r"(w[k4].w)
                             : "r"(addr)
                             : "memory");
            }
            // the loads have returned (the fence orders them before the
            // producer's next TMA write into this stage), then release it
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
            add_squares4_bf16(w, acc);
        }
    }
    __syncthreads();  // every tile has been read: the ring is free

    double *red = reinterpret_cast<double *>(smem);  // [16][128]
    if (tid < 32 * kStConsumerWarps) {
#pragma unroll
        for (int e = 0; e < 8; ++e) red[rg * kD + cc * 8 + e] = acc[e];
    }
    __syncthreads();
    score_block_end<16>(a, head, split, red);
}

}  // namespace think

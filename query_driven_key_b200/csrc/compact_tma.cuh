// compact_tma.cuh -- the key compaction of the prune for bf16 keys, with the
// key tiles staged in shared memory by TMA.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): once the channels are chosen, the cache keeps only
// the kept channels of K, K'[n, t] = K[n, idx[t]], stored channel-major (row
// h*T + t of K' holds channel idx[t] of every token).
//
// The pass reads K once (N * 128 * 2 bytes per head) and writes K' (N * T * 2),
// so it is bound by HBM.  compact_kernel loads one 64-token tile per block in
// a single phase (16 KB in flight per block, about five tiles per SM at any
// time); here each block streams a run of tiles through a ring that one
// producer thread keeps full by TMA (two 64-channel SW128 boxes per tile), so
// about 12 tiles per SM stay in flight.  The eight consumer warps transpose
// each tile with ldmatrix.trans and a word transpose inside groups of four
// lanes (compact_tile_load / compact_tile_store), so that each lane stores 8
// consecutive tokens of one kept channel as one 16-byte write.  A block keeps
// one head, so each warp finds the K' rows of its channels once.  K' is a pure
// copy: the output is that of compact_kernel bit for bit, in the uniform and
// in the ragged layout (kept width per head, zero pad rows).
//
// Launched with programmatic stream serialisation after the score kernel: the
// producer streams K (not written by the score pass) while the score grid
// drains; the consumers wait for the score grid before they read the
// selection or write K'.
//
// Every wait is bounded: on expiry the kernel sets a bit in the status word,
// the consumers stop, and the producer waits (bounded) for its loads in flight
// before the block ends.
#pragma once

#include "prune_kernels.cuh"
#include "think.h"

namespace think {

constexpr int kCtConsumerWarps = 8;  // the warp layout of compact_tile_load
constexpr int kCtThreads = 32 * kCtConsumerWarps + 32;
constexpr int kCtTileRows = 64;
constexpr uint32_t kCtHalfBytes = 64u * 64u * 2u;
constexpr uint32_t kCtTileBytes = 2u * kCtHalfBytes;
constexpr int kCtMaxStages = 8;

struct CompactTmaArgs {
    int Hkv, T;
    int run_tiles;           // tiles per block (block x: tiles [x * run_tiles, ...) of head y)
    int stages;
    int64_t N, tiles, ldk;   // tiles = ceil(N / 64)
    const int32_t *idx;      // [heads][T] kept channels, ascending (ragged: at rowoff[head])
    __nv_bfloat16 *kp;       // K' [heads][T][ldk] (ragged: rows rowoff[head] ..)
    unsigned *status;        // device status word
    const int32_t *Th;       // ragged layout: kept width per head, or null (T for every head)
    const int32_t *rowoff;   // ragged layout: first K' row (and idx entry) of each head
    int64_t row_cap;         // ragged layout: rows of K' (heads * roundup16(T))
};

inline size_t compact_tma_smem_bytes(int stages)
{
    return (size_t)stages * kCtTileBytes + 2u * (size_t)stages * 8u + 1024u;
}

__global__ void __launch_bounds__(kCtThreads, 3)
    compact_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const CompactTmaArgs a)
{
    extern __shared__ unsigned char ct_smem_dyn[];
    unsigned char *smem = ct_smem_dyn + ((1024u - (smem_addr(ct_smem_dyn) & 1023u)) & 1023u);
    const int stages = a.stages;
    const uint32_t ring = smem_addr(smem);
    const uint32_t full0 = ring + (uint32_t)stages * kCtTileBytes;
    const uint32_t empty0 = full0 + 8u * (uint32_t)stages;

    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int tid = threadIdx.x;
    const int64_t tile0 = (int64_t)blockIdx.x * a.run_tiles;
    const int ntiles = (int)min((int64_t)a.run_tiles, a.tiles - tile0);
    // Ragged layout (a.Th set): this head keeps Tk = Th[head] channels at rows
    // r0 = rowoff[head] .., then zero rows up to Tw = roundup16(Tk).  Those are
    // device data written by the selection, so the whole block waits first; a
    // head whose rows fall outside K' is skipped (garbage in, no access out).
    int Tk = a.T, Tw = a.T;
    int64_t r0 = (int64_t)head * a.T;
    if (a.Th != nullptr) {
        grid_dependency_wait();
        Tk = min(max(a.Th[head], 0), a.T);
        Tw = (Tk + 15) & ~15;
        r0 = a.rowoff[head];
        if (r0 < 0 || r0 + Tw > a.row_cap) return;
    }

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kCtConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (tid >= 32 * kCtConsumerWarps) {
        if (tid == 32 * kCtConsumerWarps) {
            prefetch_tensormap(&tm_k);
            const uint64_t pol = l2_policy_evict_first();  // the last read of K in the prune
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % stages, f = i / stages;
                if (f > 0 && !mbar_wait_bounded(empty0 + 8 * s, (uint32_t)((f - 1) & 1), a.status,
                                                THINK_DEVICE_TIMEOUT_EMPTY))
                    break;
                const uint32_t full = full0 + 8 * s;
                const uint32_t dst = ring + (uint32_t)s * kCtTileBytes;
                const int row = (int)((tile0 + i) * kCtTileRows);
                mbar_arrive_expect_tx(full, kCtTileBytes);
                tma_load_4d_hint(dst, &tm_k, 0, row, kv, b, full, pol);
                tma_load_4d_hint(dst + kCtHalfBytes, &tm_k, 64, row, kv, b, full, pol);
                ++issued;
            }
            // the loads in flight land before the block ends
            for (int i = max(0, issued - stages); i < issued; ++i)
                mbar_wait_bounded(full0 + 8 * (i % stages), (uint32_t)((i / stages) & 1), a.status,
                                  THINK_DEVICE_TIMEOUT_FULL);
        }
        __syncwarp();
        return;
    }

    const int warp = tid >> 5, lane = tid & 31;
    const int tb0 = 4 * (warp & 1), cw = warp >> 1;
    const uint32_t c_row = (uint32_t)(8 * (tb0 + (lane >> 3)) + (lane & 7));
    int64_t crow[4];
    grid_dependency_wait();  // the selection (idx) is complete; K' may be written
    kept_rows_of_warp(a.idx + r0, Tk, r0, cw, lane, crow);
    // ragged: thread tid zeroes 8 tokens (run tid % 8) of pad row Tk + tid / 8
    const int pad_row = Tk + (tid >> 3);
    const uint32_t zero[4] = {0u, 0u, 0u, 0u};
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((i / stages) & 1), a.status, THINK_DEVICE_TIMEOUT_FULL))
            break;
        uint32_t v[4][4];
        compact_tile_load(ring + (uint32_t)s * kCtTileBytes, c_row, cw, v);
        // the loads have returned (the fence orders them before the producer's
        // next TMA write into this stage), then release it
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        compact_tile_transpose(v, lane);
        const int64_t x0 = (tile0 + i) * kCtTileRows;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (crow[k] >= 0 && THINK_IN_RANGE(crow[k] < (a.Th ? a.row_cap : (int64_t)gridDim.y * a.T), a.status))
                store_run8(a.kp + crow[k] * a.ldk, x0 + 8 * (tb0 + (lane & 3)), a.N, v[k]);
        if (pad_row < Tw && THINK_IN_RANGE(r0 + pad_row < a.row_cap, a.status))
            store_run8(a.kp + (r0 + pad_row) * a.ldk, x0 + 8 * (tid & 7), a.N, zero);
    }
}

}  // namespace think

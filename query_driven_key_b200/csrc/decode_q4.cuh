// decode_q4.cuh -- the thinner key cache at 4 bits per element: quantisation
// and decode attention over it.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", abstract and method
// section (technical framework): the pruned cache combines with KV-cache
// quantisation such as KIVI; the MiniKV page (quantisation) quantises keys per
// (sub-)channel.  The reading used here, for every kept channel t of a head
// and every group of 128 tokens (one decode tile):
//     mn = min, scale = (max - mn) / 15                       (fp32)
//     code = 0 if scale == 0 else clamp(rint((x - mn) / scale), 0, 15)
//     dequantised key = bf16(fma(code, scale, mn))            (fp32, then RNE)
// Layouts:
//     codes   [B][Hkv][T][ldq] bytes, token n of row t in byte n/2 (even token
//             in the low nibble); ldq = 64 * (capacity in 128-token groups)
//     groups  [B][Hkv][ldq/64][T2][2] fp32 (scale, mn), T2 = T rounded up to 2
// Decode reads 0.5 byte per kept key element plus 8 bytes per 128 tokens and
// channel instead of 2 bytes: the warp-level tensor-core decode with a
// dequantisation step in front of each tile.
#pragma once

#include "decode_mma.cuh"

namespace think {

constexpr int kQ4Group = 128;  // tokens per quantisation group (= kBN)

// ---------------------------------------------------------------------------
// Quantise: block (group, head), four warps over the channel rows, each lane
// four tokens of the group.  Every operation is the fp32 one written above
// (IEEE subtraction and division, round-half-even), so the codes and the
// group parameters match a plain C implementation bit for bit.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    quantize_q4_kernel(const __nv_bfloat16 *__restrict__ kp, int64_t ldk, int T, int64_t N,
                       uint8_t *__restrict__ codes, int64_t ldq, float2 *__restrict__ groups)
{
    const int g = blockIdx.x, head = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T2 = (T + 1) & ~1;
    const int64_t ng = ldq / 64;
    const int64_t n0 = (int64_t)g * kQ4Group + 4 * lane;
    for (int t = warp; t < T2; t += 4) {
        float x[4];
        float mn = INFINITY, mx = -INFINITY;
        const __nv_bfloat16 *row = kp + ((int64_t)head * T + min(t, T - 1)) * ldk;
        if (t < T && n0 + 4 <= N) {
            const uint2 w = *reinterpret_cast<const uint2 *>(row + n0);
            x[0] = bf16lo(w.x);
            x[1] = bf16hi(w.x);
            x[2] = bf16lo(w.y);
            x[3] = bf16hi(w.y);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mn = fminf(mn, x[j]);
                mx = fmaxf(mx, x[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool valid = t < T && n0 + j < N;
                x[j] = valid ? Elem<__nv_bfloat16>::to_float(row[n0 + j]) : 0.f;
                if (valid) {
                    mn = fminf(mn, x[j]);
                    mx = fmaxf(mx, x[j]);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (t >= T) {  // the pad row of an odd T
            if (lane == 0) groups[((int64_t)head * ng + g) * T2 + t] = make_float2(0.f, 0.f);
            continue;
        }
        const float scale = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        uint32_t packed = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float c = 0.f;
            if (scale != 0.f && n0 + j < N)
                c = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x[j], mn), scale)), 0.f), 15.f);
            packed |= (uint32_t)c << (4 * j);
        }
        *reinterpret_cast<uint16_t *>(codes + ((int64_t)head * T + t) * ldq + (int64_t)g * 64 + 2 * lane) =
            (uint16_t)packed;
        if (lane == 0) groups[((int64_t)head * ng + g) * T2 + t] = make_float2(scale, mn);
    }
}

// ---------------------------------------------------------------------------
// Decode over the 4-bit thinner cache.  Same structure as
// pruned_decode_mma_kernel (producer warp + four consumer warps, split-N, last
// block merges); a stage holds the codes tile (T rows x 64 B), the group
// parameters (T2 x 8 B) and the V tile.  Each consumer warp dequantises the
// codes of its own 32 tokens into its own columns of one bf16 K' tile
// (128-byte swizzle, the layout mma_tile reads), so no block barrier is
// needed; then it runs the same tensor-core tile as the bf16 kernel.
// ---------------------------------------------------------------------------
struct Q4Layout {
    uint32_t t_pad;    // T rounded up to 16
    uint32_t k_half;   // one 64-token half of the bf16 tile: t_pad rows x 128 B
    uint32_t meta_off; // group parameters inside a stage
    uint32_t v_off;    // V tile inside a stage (1024-aligned)
    uint32_t stage;    // bytes per stage
    uint32_t tx;       // bytes a stage receives
};

__host__ __device__ inline Q4Layout q4_layout(int T)
{
    Q4Layout L;
    const uint32_t T2 = (uint32_t)((T + 1) & ~1);
    L.t_pad = (uint32_t)((T + 15) & ~15);
    L.k_half = L.t_pad * 128u;
    L.meta_off = ((uint32_t)T * 64u + 127u) & ~127u;  // TMA destinations 128-byte aligned
    L.v_off = (L.meta_off + T2 * 8u + 1023u) & ~1023u;
    L.stage = L.v_off + 32768u;
    L.tx = (uint32_t)T * 64u + T2 * 8u + 32768u;
    return L;
}

// stages, then the bf16 tile (two halves), q' [16][t_pad] bf16, the warp merge
// area [CW][G][128] + [CW][G][2] floats, barriers, a flag
__host__ __device__ inline size_t q4_smem_bytes(int T, int G, int stages, int CW)
{
    const Q4Layout L = q4_layout(T);
    return (size_t)stages * L.stage + 2u * L.k_half + 32u * L.t_pad + (size_t)CW * G * 130 * 4 +
           (size_t)2 * stages * 8 + 16 + 1024;
}

template <int G, int CW>
__global__ void __launch_bounds__(CW * 32 + 32)
    pruned_decode_q4_kernel(const __grid_constant__ CUtensorMap tm_codes,
                            const __grid_constant__ CUtensorMap tm_groups,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a)
{
    static_assert(G >= 1 && G <= 8, "the group's query heads fill at most the 8 MMA columns");
    static_assert(CW == 4 || CW == 8, "32 or 16 tokens of a tile per consumer warp");
    constexpr int TPW = kBN / CW;        // tokens per consumer warp
    constexpr int NT = CW * 32;
    constexpr int PARTS = TPW / 8;       // 8-token chunks per warp and channel row
    constexpr int RPP = 32 / PARTS;      // channel rows per pass of a warp
    // Launched as a programmatic dependent of the previous kernel in the
    // stream: everything it wrote is visible after this wait; let the next
    // decode be scheduled on SMs as ours free up.  Before the wait the
    // producer lane asks L2 for this block's first tiles and the q and idx
    // lines (as in pruned_decode_mma_kernel: the kernels that let a decode
    // start early write none of codes, groups or V, and L2 is coherent).
    if (a.early && threadIdx.x == CW * 32) {
        const int kv0 = (int)blockIdx.y % a.Hkv, b0 = (int)blockIdx.y / a.Hkv;
        const int64_t t0 = (int64_t)blockIdx.x * a.tiles_per_split;
        const int64_t n = min((int64_t)min(a.tiles_per_split, a.stages), (a.N + kBN - 1) / kBN - t0);
        for (int64_t it = 0; it < n; ++it) {
            const int tile = (int)(t0 + it);
            tma_prefetch_l2_4d(&tm_codes, tile * 64, 0, kv0, b0);
            tma_prefetch_l2_4d(&tm_groups, 0, tile, kv0, b0);
            tma_prefetch_l2_4d(&tm_v, 0, tile * kBN, kv0, b0);
            tma_prefetch_l2_4d(&tm_v, 64, tile * kBN, kv0, b0);
        }
        const char *qrow = reinterpret_cast<const char *>(a.q) + ((int64_t)b0 * a.Hq + (int64_t)kv0 * G) * kD * 2;
        for (int o = 0; o < G * kD * 2; o += 128) prefetch_l2(qrow + o);
        const char *irow = reinterpret_cast<const char *>(a.idx + (int64_t)blockIdx.y * a.T);
        for (int o = 0; o < a.T * 4; o += 128) prefetch_l2(irow + o);
    }
    grid_dependency_wait();
    grid_launch_dependents();
    extern __shared__ unsigned char smem_dyn[];
    unsigned char *smem = smem_dyn + ((1024u - (smem_addr(smem_dyn) & 1023u)) & 1023u);

    const int split = blockIdx.x;
    const int head = blockIdx.y;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int T = a.T;
    const int stages = a.stages;
    const Q4Layout L = q4_layout(T);
    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tiles_all = (a.N + kBN - 1) / kBN;
    const int ntiles = (int)min((int64_t)a.tiles_per_split, tiles_all - tile0);

    unsigned char *kbf = smem + (size_t)stages * L.stage;                        // bf16 K' tile
    unsigned char *qsm = kbf + 2u * L.k_half;                                    // [16][t_pad] bf16
    float *mo = reinterpret_cast<float *>(qsm + 32u * L.t_pad);                  // [CW][G][128]
    float *mml = mo + CW * G * kD;                                               // [CW][G][2]
    uint64_t *bars = reinterpret_cast<uint64_t *>(mml + CW * G * 2);
    unsigned *flag = reinterpret_cast<unsigned *>(bars + 2 * stages);
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + stages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, CW);
        }
        fence_barrier_init();
    }
    __syncthreads();  // barriers initialised

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tm_codes);
            prefetch_tensormap(&tm_groups);
            prefetch_tensormap(&tm_v);
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
                mbar_arrive_expect_tx(full, L.tx);
                const int tile = (int)(tile0 + it);
                const int x = tile * kBN;
                const uint32_t st = smem_addr(smem + (size_t)s * L.stage);
                tma_load_4d(st, &tm_codes, tile * 64, 0, kv, b, full);
                tma_load_4d(st + L.meta_off, &tm_groups, 0, tile, kv, b, full);
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
        return;
    }

    // ---------------------------------------------------------- consumers
    // zero the bf16 tile's rows T..t_pad-1 once (dequantisation writes rows
    // 0..T-1 only), stage q'
    {
        const uint32_t pad16 = (L.t_pad - (uint32_t)T) * 8u;  // 16-byte words per half
        for (uint32_t i = tid; i < 2u * pad16; i += NT)
            *reinterpret_cast<uint4 *>(kbf + (i / pad16) * L.k_half + (uint32_t)T * 128u + (i % pad16) * 16u) =
                make_uint4(0, 0, 0, 0);
        mma_stage_q<G, NT>(a, qsm, L.t_pad, T, a.idx + (int64_t)head * T, b, kv, tid,
                           reinterpret_cast<unsigned char *>(mo));
    }
    named_barrier(1, NT);

    uint32_t qb[kD / 16][2];
    const int ksteps = (int)(L.t_pad / 16u);
    mma_load_qb(qsm, L.t_pad, ksteps, lane, qb);
    MmaState S;
    mma_state_init(S);
    const uint32_t sbase = smem_addr(smem);
    const uint32_t kbase = smem_addr(kbf);
    // dequantisation: lane = PARTS * rr + p handles rows t = RPP i + rr, tokens
    // TPW * warp + 8 p .. +7 (one 16-byte chunk of the bf16 tile)
    const int rr = lane / PARTS, p = lane % PARTS;
    const uint32_t dq_dst = kbase + (uint32_t)((TPW * warp) >> 6) * L.k_half;
    const uint32_t dq_chunk = (uint32_t)(((TPW * warp) & 63) / 8 + p);
    const uint32_t dq_src = (uint32_t)(TPW / 2 * warp + 4 * p);   // byte of the codes row

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % stages;
        if (!mbar_wait_bounded(full0 + 8 * s, (it / stages) & 1, a.status, THINK_DEVICE_TIMEOUT_FULL))
            break;
        const uint32_t st = sbase + (uint32_t)s * L.stage;
        for (int t = rr; t < T; t += RPP) {
            uint32_t w;
            float2 sm;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(st + (uint32_t)t * 64u + dq_src));
            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                         : "=f"(sm.x), "=f"(sm.y)
                         : "r"(st + L.meta_off + (uint32_t)t * 8u));
            // even and odd tokens' codes, one per byte; a byte permute builds the
            // float 2^23 + code, from which an exact subtraction gives the code;
            // then fma(code, scale, mn) per element (packed pairs) and bf16 RNE
            const uint32_t ev = w & 0x0F0F0F0Fu, od = (w >> 4) & 0x0F0F0F0Fu;
            const float2 sc2 = make_float2(sm.x, sm.x), mn2 = make_float2(sm.y, sm.y);
            const float2 bias = make_float2(-8388608.f, -8388608.f);
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t sel = 0x7440u | (uint32_t)j;
                const float2 c = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, sel)),
                                                        __uint_as_float(__byte_perm(od, 0x4B000000u, sel))),
                                            bias);
                const float2 y = __ffma2_rn(c, sc2, mn2);
                o[j] = wmma16::pack_bf16x2(y.x, y.y);
            }
            const uint32_t dst = dq_dst + (uint32_t)t * 128u + ((dq_chunk ^ ((uint32_t)t & 7u)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                         "r"(o[3])
                         : "memory");
        }
        __syncwarp();
        const int64_t tok_base = (tile0 + it) * kBN + warp * TPW;
        mma_tile<TPW>(kbase, L.k_half, st + L.v_off, qb, ksteps, warp, lane, tok_base, a.N, a.scale_log2, S);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
    mma_merge_and_finish<G, CW>(a, S, mo, mml, reinterpret_cast<float *>(smem), flag, head, split, b, kv, tid,
                                a.staged_merge ? (size_t)stages * L.stage / sizeof(float) : 0);
}

}  // namespace think

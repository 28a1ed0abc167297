// decode_f64.cuh -- pruned-K decode attention for fp32 caches, with every
// step after the loads carried out in fp64.
//
// "ThinK: Thinner Key Cache by Query-Driven Pruning", method section
// (technical framework): decoding attends with the thinner key cache; the
// query is gathered at the kept channels,
//     z_n = (q[idx] . K'[n, :T]) * scale,   p = softmax_n(z),   out = sum_n p_n V[n, :].
//
// fp32 inputs are exact in fp64, so the only rounding that reaches the output
// at fp32 size is the final conversion (relative 2^-24); the logits, the
// exponentials (the library's double exp), the running sums and the split
// merge add errors of order 1e-15 relative.  The path is latency-bound on the
// shapes it serves (fp32 caches are the small parity case), so it keeps the
// plain structure: grid (splits, B*Hkv) like the other decodes, 128-token
// tiles read straight from global memory (coalesced along the token axis for
// K'^T and along the channel axis for V), one online softmax per split,
// partials (O, max, sum) in fp64 in the workspace and a merge by the last
// block of each head (ticket counter), in split order.
#pragma once

#include "decode_kernels.cuh"

namespace think {

struct DecodeF64Args {
    const float *q;          // [B][Hq][128]
    const float *kp;         // K'^T [B][Hkv][T][ldk]
    const float *v;          // [B][Hkv][N][128] with element strides
    int64_t sb, sh, sn;      // V strides (batch, head, token)
    const int32_t *idx;      // [B][Hkv][T]
    float *out;              // [B][Hq][128]
    double *part_o;          // [heads][splits][G][128]
    double *part_ml;         // [heads][splits][G][2]  (max, sum) in natural-log units
    unsigned *tickets;       // [heads], zero between calls
    int Hq, Hkv, T, splits, tiles_per_split;
    int64_t N, ldk;
    double scale;
};

template <int G>
__global__ void __launch_bounds__(256) pruned_decode_f64_kernel(const DecodeF64Args a)
{
    __shared__ double qs[G][kD];      // q at the kept channels, t < T
    __shared__ double zp[G][kBN];     // the tile's logits, then its weights
    __shared__ double m_s[G], l_s[G], alpha_s[G];
    __shared__ double o_half[G][kD];  // the odd tokens' share of O, added at the end
    __shared__ unsigned last;

    const int tid = threadIdx.x;
    const int head = blockIdx.y, split = blockIdx.x;
    const int b = head / a.Hkv, kv = head % a.Hkv;
    const int T = a.T;
    const int32_t *idx = a.idx + (int64_t)head * T;
    for (int i = tid; i < G * T; i += 256) {
        const int g = i / T, t = i % T;
        const int64_t hq = (int64_t)b * a.Hq + (int64_t)kv * G + g;
        const int c = idx[t];
        qs[g][t] = ((unsigned)c < (unsigned)kD) ? (double)a.q[hq * kD + c] : 0.0;
    }
    if (tid < G) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.0;
    }
    __syncthreads();

    const float *kh = a.kp + (int64_t)head * T * a.ldk;
    const float *vh = a.v + (int64_t)b * a.sb + (int64_t)kv * a.sh;
    const int d = tid & (kD - 1), half = tid >> 7;  // V: channel d, tokens of parity `half`
    double o[G];
#pragma unroll
    for (int g = 0; g < G; ++g) o[g] = 0.0;

    const int64_t tile0 = (int64_t)split * a.tiles_per_split;
    const int64_t tile1 = min(tile0 + a.tiles_per_split, (a.N + kBN - 1) / kBN);
    for (int64_t tile = tile0; tile < tile1; ++tile) {
        const int64_t n0 = tile * kBN;
        // logits of the tile's tokens (threads 0..127, one token each)
        if (tid < kBN) {
            const int64_t n = n0 + tid;
            double z[G];
#pragma unroll
            for (int g = 0; g < G; ++g) z[g] = 0.0;
            if (n < a.N) {
                for (int t = 0; t < T; ++t) {
                    const double kx = (double)kh[(int64_t)t * a.ldk + n];
#pragma unroll
                    for (int g = 0; g < G; ++g) z[g] = fma(qs[g][t], kx, z[g]);
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) zp[g][tid] = (n < a.N) ? z[g] * a.scale : -INFINITY;
        }
        __syncthreads();
        // running max, rescale factor (thread g)
        if (tid < G) {
            double mx = m_s[tid];
            for (int j = 0; j < kBN; ++j) mx = fmax(mx, zp[tid][j]);
            alpha_s[tid] = (m_s[tid] == -INFINITY) ? 0.0 : exp(m_s[tid] - mx);
            m_s[tid] = mx;
        }
        __syncthreads();
        for (int i = tid; i < G * kBN; i += 256) {
            const int g = i / kBN, j = i % kBN;
            const double zz = zp[g][j];
            zp[g][j] = (zz == -INFINITY) ? 0.0 : exp(zz - m_s[g]);
        }
        __syncthreads();
        if (tid < G) {
            double s = 0.0;
            for (int j = 0; j < kBN; ++j) s += zp[tid][j];
            l_s[tid] = fma(l_s[tid], alpha_s[tid], s);
        }
        // values: this thread's channel over the tile's tokens of its parity
        double acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.0;
        for (int j = half; j < kBN; j += 2) {
            const int64_t n = n0 + j;
            if (n >= a.N) break;
            const double vx = (double)vh[n * a.sn + d];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = fma(zp[g][j], vx, acc[g]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) o[g] = fma(o[g], alpha_s[g], acc[g]);
        __syncthreads();  // zp, alpha_s are rewritten by the next tile
    }

    // split partial: O = even-token share + odd-token share, then (max, sum)
    if (half == 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) o_half[g][d] = o[g];
    }
    __syncthreads();
    const int64_t slot0 = ((int64_t)head * a.splits + split) * G;
    if (half == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) a.part_o[(slot0 + g) * kD + d] = o[g] + o_half[g][d];
    }
    if (tid < G) {
        a.part_ml[(slot0 + tid) * 2] = m_s[tid];
        a.part_ml[(slot0 + tid) * 2 + 1] = l_s[tid];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last = (atomicAdd(a.tickets + head, 1u) == (unsigned)(a.splits - 1)) ? 1u : 0u;
    __syncthreads();
    if (!last) return;

    // the last block of the head: merge the splits in split order
    __threadfence();
    const int64_t base = (int64_t)head * a.splits * G;
    for (int i = tid; i < G * kD; i += 256) {
        const int g = i / kD, c = i % kD;
        double M = -INFINITY;
        for (int s = 0; s < a.splits; ++s) M = fmax(M, __ldcg(a.part_ml + (base + (int64_t)s * G + g) * 2));
        double O = 0.0, L = 0.0;
        for (int s = 0; s < a.splits; ++s) {
            const int64_t sl = base + (int64_t)s * G + g;
            const double ms = __ldcg(a.part_ml + sl * 2);
            if (ms == -INFINITY) continue;
            const double w = exp(ms - M);
            O = fma(__ldcg(a.part_o + sl * kD + c), w, O);
            L = fma(__ldcg(a.part_ml + sl * 2 + 1), w, L);
        }
        const int64_t hq = (int64_t)b * a.Hq + (int64_t)kv * G + g;
        a.out[hq * kD + c] = (float)(O / L);
    }
    if (tid == 0) a.tickets[head] = 0u;  // ready for the next call
}

}  // namespace think

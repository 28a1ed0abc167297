/*
 * think_oracle.c -- plain, slow fp64 CPU oracle of the ThinK decode-time path.
 *
 * TEST INFRASTRUCTURE. Only the tests, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library. The CUDA product path never
 * links, imports or calls it, and it shares no code with that path.
 *
 * Source: "ThinK: Thinner Key Cache by Query-Driven Pruning" (Xu et al.,
 * ICLR 2025).  Its method section ("方法详解", technical framework) gives the
 * flow implemented here: rate every key channel by its relevance to the query,
 * sort the channels, drop the least relevant ones, then run inference with the
 * pruned cache.  Its abstract states the goal of the ranking: keep the
 * attention weights QK^T as close as possible while removing the least
 * significant channels of the key cache.  The page gives no formula, so the
 * readings below are the plainest ones consistent with that text:
 *
 *   score   s[c] = sum over the query heads g of the KV group of
 *                  || Qwin_g[:,c] K[:,c]^T ||_F  =  ||Qwin_g[:,c]||_2 ||K[:,c]||_2
 *           (the Frobenius norm of channel c's rank-one share of Qwin K^T)
 *   select  keep the T channels with the largest s[c]; equal scores go to the
 *           lower channel index; the kept list is returned in ascending order
 *   compact K'[n,t] = K[n, idx[t]]   (V is not touched)
 *   decode  q'[t] = q[idx[t]];  z[n] = (q' . K'[n,:]) / sqrt(d) with the full
 *           head width d;  p = softmax(z);  out = sum_n p[n] V[n,:]
 *
 * Query head h belongs to KV head h / G (G = Hq / Hkv: consecutive query heads
 * share one KV head).  Everything is fp64 with sums in ascending index order.
 * No blocking, fusion or reordering beyond that.
 *
 * Layouts (all C-contiguous, last index fastest):
 *   qwin [B][Hq][S][d], k [B][Hkv][N][d], v [B][Hkv][N][d], q [B][Hq][d],
 *   scores [B][Hkv][d], idx [B][Hkv][T] (int32), kp [B][Hkv][N][T],
 *   out [B][Hq][d].
 *
 * Every function returns 0 on success and a negative value on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Per-channel relevance of the key cache to the observation-window queries
 * (ThinK, method section: "compute each channel's relevance to the query").
 * kn2[c] = sum_n K[n,c]^2 and qn2[g,c] = sum_s Qwin_g[s,c]^2, both summed in
 * ascending order; s[c] = sum_g sqrt(qn2[g,c]) * sqrt(kn2[c]). */
int oracle_score(const double *qwin, const double *k, int B, int Hq, int Hkv,
                 int S, int N, int d, double *scores)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || S < 0 || N < 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -2;
    const int G = Hq / Hkv;
    const long long heads = (long long)B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bh = 0; bh < heads; ++bh) {
        const long long b = bh / Hkv, kv = bh % Hkv;
        double *kn2 = (double *)calloc((size_t)d, sizeof(double));
        const double *kh = k + (size_t)bh * (size_t)N * (size_t)d;
        for (long long n = 0; n < N; ++n)
            for (int c = 0; c < d; ++c) {
                const double x = kh[(size_t)n * d + c];
                kn2[c] += x * x;
            }
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int g = 0; g < G; ++g) {
                const long long h = kv * G + g;
                const double *qh = qwin + ((size_t)b * Hq + (size_t)h) * (size_t)S * (size_t)d;
                double qn2 = 0.0;
                for (int t = 0; t < S; ++t) {
                    const double x = qh[(size_t)t * d + c];
                    qn2 += x * x;
                }
                s += sqrt(qn2) * sqrt(kn2[c]);
            }
            scores[(size_t)bh * d + c] = s;
        }
        free(kn2);
    }
    return 0;
}

/* The definition the factorised score stands for: the Frobenius norm of the
 * explicit S x N matrix Qwin_g[:,c] K[:,c]^T, summed over the group.  Slow
 * (S*N products per channel); used only to pin oracle_score on small inputs. */
int oracle_score_explicit(const double *qwin, const double *k, int B, int Hq,
                          int Hkv, int S, int N, int d, double *scores)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || S < 0 || N < 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -2;
    const int G = Hq / Hkv;
    for (long long b = 0; b < B; ++b)
        for (long long kv = 0; kv < Hkv; ++kv)
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int g = 0; g < G; ++g) {
                    const long long h = kv * G + g;
                    const double *qh = qwin + ((size_t)b * Hq + (size_t)h) * (size_t)S * (size_t)d;
                    const double *kh = k + ((size_t)b * Hkv + (size_t)kv) * (size_t)N * (size_t)d;
                    double fro2 = 0.0;
                    for (int t = 0; t < S; ++t)
                        for (long long n = 0; n < N; ++n) {
                            const double m = qh[(size_t)t * d + c] * kh[(size_t)n * d + c];
                            fro2 += m * m;
                        }
                    s += sqrt(fro2);
                }
                scores[((size_t)b * Hkv + (size_t)kv) * d + c] = s;
            }
    return 0;
}

/* Ordering of the channels of one head: larger score first, equal scores by
 * lower channel index (ThinK, method section: sort the channels by relevance,
 * prune the low ones).  A NaN score is ordered after every number. */
static const double *g_sort_scores; /* only read inside qsort below */

static int by_score_desc(const void *pa, const void *pb)
{
    const int a = *(const int *)pa, b = *(const int *)pb;
    const double sa = g_sort_scores[a], sb = g_sort_scores[b];
    const int na = isnan(sa), nb = isnan(sb);
    if (na != nb) return na ? 1 : -1;
    if (!na) {
        if (sa > sb) return -1;
        if (sa < sb) return 1;
    }
    return (a > b) - (a < b);
}

static int ascending_int(const void *pa, const void *pb)
{
    const int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

int oracle_select(const double *scores, int B, int Hkv, int d, int T, int32_t *idx)
{
    if (B < 0 || Hkv < 0 || d <= 0 || T < 1 || T > d) return -1;
    int *order = (int *)malloc((size_t)d * sizeof(int));
    for (long long bh = 0; bh < (long long)B * Hkv; ++bh) {
        for (int c = 0; c < d; ++c) order[c] = c;
        g_sort_scores = scores + (size_t)bh * d;
        qsort(order, (size_t)d, sizeof(int), by_score_desc);
        qsort(order, (size_t)T, sizeof(int), ascending_int);
        for (int t = 0; t < T; ++t) idx[(size_t)bh * T + t] = order[t];
    }
    free(order);
    g_sort_scores = NULL;
    return 0;
}

/* Thinner key cache: K'[n,t] = K[n, idx[t]] (ThinK title and method section:
 * the key cache keeps only the selected channels; V is left as it is). */
int oracle_compact(const double *k, const int32_t *idx, int B, int Hkv, int N,
                   int d, int T, double *kp)
{
    if (B < 0 || Hkv < 0 || N < 0 || d <= 0 || T < 1 || T > d) return -1;
    for (long long bh = 0; bh < (long long)B * Hkv; ++bh) {
        const int32_t *ih = idx + (size_t)bh * T;
        for (int t = 0; t < T; ++t)
            if (ih[t] < 0 || ih[t] >= d) return -3;
        for (long long n = 0; n < N; ++n)
            for (int t = 0; t < T; ++t)
                kp[((size_t)bh * N + (size_t)n) * T + t] =
                    k[((size_t)bh * N + (size_t)n) * d + ih[t]];
    }
    return 0;
}

/* One query head's attention over N keys of width W (shared by the pruned and
 * the dense decode below; plain softmax with the maximum subtracted). */
static void attend_one(const double *qv, const double *keys, int W,
                       const double *v, int N, int d, double scale,
                       double *z, double *out)
{
    double m = -INFINITY;
    for (long long n = 0; n < N; ++n) {
        double dot = 0.0;
        for (int t = 0; t < W; ++t) dot += qv[t] * keys[(size_t)n * W + t];
        z[n] = dot * scale;
        if (z[n] > m) m = z[n];
    }
    double l = 0.0;
    for (long long n = 0; n < N; ++n) {
        z[n] = exp(z[n] - m);
        l += z[n];
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (long long n = 0; n < N; ++n) {
        const double p = z[n] / l;
        for (int c = 0; c < d; ++c) out[c] += p * v[(size_t)n * d + c];
    }
}

/* Decode attention with the thinner key cache (ThinK, method section: run
 * inference with the pruned cache).  Scale is passed in; the readings use
 * 1/sqrt(d) of the full head width. */
int oracle_decode(const double *q, const double *kp, const double *v,
                  const int32_t *idx, int B, int Hq, int Hkv, int N, int d,
                  int T, double scale, double *out)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || N <= 0 || d <= 0 || T < 1 || T > d) return -1;
    if (Hq % Hkv != 0) return -2;
    const int G = Hq / Hkv;
    const long long heads = (long long)B * Hq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long long bhq = 0; bhq < heads; ++bhq) {
        const long long b = bhq / Hq, h = bhq % Hq, kv = h / G;
        const size_t kvh = (size_t)b * Hkv + (size_t)kv;
        const int32_t *ih = idx + kvh * T;
        double *qp = (double *)malloc((size_t)T * sizeof(double));
        double *z = (double *)malloc((size_t)N * sizeof(double));
        for (int t = 0; t < T; ++t) {
            if (ih[t] < 0 || ih[t] >= d) { bad = 1; qp[t] = 0.0; continue; }
            qp[t] = q[(size_t)bhq * d + ih[t]];
        }
        attend_one(qp, kp + kvh * (size_t)N * T, T, v + kvh * (size_t)N * d, N, d,
                   scale, z, out + (size_t)bhq * d);
        free(qp);
        free(z);
    }
    return bad ? -3 : 0;
}

/* Dense decode attention over the full key cache (the lambda = 0 case). */
int oracle_dense_decode(const double *q, const double *k, const double *v, int B,
                        int Hq, int Hkv, int N, int d, double scale, double *out)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || N <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -2;
    const int G = Hq / Hkv;
    const long long heads = (long long)B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bhq = 0; bhq < heads; ++bhq) {
        const long long b = bhq / Hq, h = bhq % Hq, kv = h / G;
        const size_t kvh = (size_t)b * Hkv + (size_t)kv;
        double *z = (double *)malloc((size_t)N * sizeof(double));
        attend_one(q + (size_t)bhq * d, k + kvh * (size_t)N * d, d,
                   v + kvh * (size_t)N * d, N, d, scale, z, out + (size_t)bhq * d);
        free(z);
    }
    return 0;
}

/*
 * 4-bit thinner key cache (ThinK composed with per-channel key quantisation,
 * as in the ThinK + KIVI combination of the experiments section; KIVI
 * quantises keys per channel over groups of tokens).  Reading used here, for
 * each (b, h_kv), kept channel t and group of `group` consecutive tokens:
 *
 *   mn    = min of the group's K'[n,t]      mx = max            (fp32, exact)
 *   scale = (mx - mn) / 15                                      (fp32 division)
 *   code  = 0 if scale == 0, else clamp(rint((K'[n,t] - mn) / scale), 0, 15)
 *           (fp32 subtraction and division, rint = round half to even)
 *   K^[n,t] = bf16(fma(code, scale, mn))    (fp32 fused multiply-add, then
 *                                            round to nearest-even bf16)
 *
 * The inputs are bf16 values (carried as doubles); every step is the fp32
 * operation written, so the codes, the group parameters and the dequantised
 * keys are defined exactly.
 *
 *   kp    [B][Hkv][N][T]     values of the thinner key cache (bf16-exact)
 *   codes [B][Hkv][N][T]     uint8, 0..15
 *   gs    [B][Hkv][ng][T][2] fp32 (scale, mn), ng = ceil(N / group)
 */
static float bf16_round(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;   /* finite inputs only */
    float y;
    memcpy(&y, &u, 4);
    return y;
}

int oracle_quantize_q4(const double *kp, int B, int Hkv, int N, int T, int group, uint8_t *codes,
                       float *gs)
{
    if (B < 0 || Hkv < 0 || N < 0 || T < 1 || group < 1) return -1;
    const int ng = (N + group - 1) / group;
    for (int bh = 0; bh < B * Hkv; ++bh)
        for (int g = 0; g < ng; ++g) {
            const int n0 = g * group, n1 = (n0 + group < N) ? n0 + group : N;
            for (int t = 0; t < T; ++t) {
                float mn = (float)kp[((size_t)bh * N + n0) * T + t], mx = mn;
                for (int n = n0 + 1; n < n1; ++n) {
                    const float x = (float)kp[((size_t)bh * N + n) * T + t];
                    if (x < mn) mn = x;
                    if (x > mx) mx = x;
                }
                const float scale = (mx - mn) / 15.0f;
                gs[(((size_t)bh * ng + g) * T + t) * 2 + 0] = scale;
                gs[(((size_t)bh * ng + g) * T + t) * 2 + 1] = mn;
                for (int n = n0; n < n1; ++n) {
                    const float x = (float)kp[((size_t)bh * N + n) * T + t];
                    float c = 0.0f;
                    if (scale != 0.0f) {
                        c = rintf((x - mn) / scale);
                        if (c < 0.0f) c = 0.0f;
                        if (c > 15.0f) c = 15.0f;
                    }
                    codes[((size_t)bh * N + n) * T + t] = (uint8_t)c;
                }
            }
        }
    return 0;
}

int oracle_dequantize_q4(const uint8_t *codes, const float *gs, int B, int Hkv, int N, int T,
                         int group, double *khat)
{
    if (B < 0 || Hkv < 0 || N < 0 || T < 1 || group < 1) return -1;
    const int ng = (N + group - 1) / group;
    for (int bh = 0; bh < B * Hkv; ++bh)
        for (int n = 0; n < N; ++n)
            for (int t = 0; t < T; ++t) {
                const size_t gi = (((size_t)bh * ng + n / group) * T + t) * 2;
                const float c = (float)codes[((size_t)bh * N + n) * T + t];
                khat[((size_t)bh * N + n) * T + t] = (double)bf16_round(fmaf(c, gs[gi], gs[gi + 1]));
            }
    return 0;
}

/*
 * Adaptive kept width per head (ThinK method section, key design 3: the
 * pruning ratio adapts to the query and the cache; key design 2: the pruning
 * keeps the attention-weight loss small).  Reading used here: rank the
 * channels as oracle_select does (score descending, index ascending); with
 * E = the sum of the squared scores taken in rank order and cum_k the sum of
 * the first k squared scores in rank order (fp64, sequential),
 *     T_h = the smallest k in [T_min, T_max] with cum_k >= tau * E,
 *           T_max if there is none, T_min if E == 0;
 * the kept channels are the first T_h in rank order, written ascending at
 * idx[off_h .. off_h + T_h), off_h = T_0 + ... + T_{h-1} over the heads in
 * (b, h_kv) order.  For one query head and orthogonal window queries the
 * squared score of a channel is exactly its share of the squared attention
 * loss, so T_h is then the fewest channels whose dropped loss^2 stays within
 * (1 - tau) E.
 *   scores [B][Hkv][d]; Th [B*Hkv] int32; off [B*Hkv + 1] int32 (off[B*Hkv] =
 *   total rows); idx [total rows] int32.  Returns the total number of rows.
 */
int oracle_select_adaptive(const double *scores, int B, int Hkv, int d, double tau, int T_min, int T_max,
                           int32_t *Th, int32_t *off, int32_t *idx, int idx_cap)
{
    if (B < 0 || Hkv < 0 || d < 1 || T_min < 1 || T_max < T_min || T_max > d) return -1;
    if (!(tau >= 0.0 && tau <= 1.0)) return -1;
    int *order = (int *)malloc(sizeof(int) * (size_t)d);
    if (!order) return -2;
    int32_t rows = 0;
    for (int bh = 0; bh < B * Hkv; ++bh) {
        const double *s = scores + (size_t)bh * d;
        g_sort_scores = s;
        for (int c = 0; c < d; ++c) order[c] = c;
        qsort(order, (size_t)d, sizeof(int), by_score_desc);
        double E = 0.0;
        for (int i = 0; i < d; ++i) E += s[order[i]] * s[order[i]];
        int T = T_max;
        if (E == 0.0) {
            T = T_min;
        } else {
            double cum = 0.0;
            for (int k = 1; k <= T_max; ++k) {
                cum += s[order[k - 1]] * s[order[k - 1]];
                if (k >= T_min && cum >= tau * E) {
                    T = k;
                    break;
                }
            }
        }
        Th[bh] = T;
        off[bh] = rows;
        if (rows + T > idx_cap) {
            free(order);
            return -3;
        }
        qsort(order, (size_t)T, sizeof(int), ascending_int);
        for (int t = 0; t < T; ++t) idx[rows + t] = order[t];
        rows += T;
    }
    off[B * Hkv] = rows;
    free(order);
    return rows;
}

/*
 * Token eviction composed with channel pruning (ThinK abstract and
 * experiments: compared with and combined with KV-cache eviction; Keyformer
 * page: keep the "key tokens" that receive the most attention).  Reading used
 * here (the observation-window attention mass): for each (b, h_kv) and cached
 * token n,
 *     mass[n] = sum over the group's query heads g and window rows s of
 *               softmax_n( scale * Qwin[b,g,s,:] . K[b,h_kv,n,:] )
 * (fp64; for each row the max, then the sum of exp(z - max) over n ascending,
 * then the rows added in (g, s) order); keep the M tokens with the largest
 * mass (ties to the lower index), in ascending order; the channel pruning then
 * runs on the kept tokens' keys.
 *   qwin [B][Hq][S][d], k [B][Hkv][N][d] -> mass [B][Hkv][N];
 *   kept [B][Hkv][M] int32.
 */
int oracle_token_mass(const double *qwin, const double *k, int B, int Hq, int Hkv, int S, int N, int d,
                      double scale, double *mass)
{
    if (B < 0 || Hq < 0 || Hkv < 1 || S < 0 || N < 1 || d < 1 || Hq % Hkv) return -1;
    const int G = Hq / Hkv;
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    if (!z) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const double *kh = k + ((size_t)b * Hkv + h) * (size_t)N * d;
            double *mh = mass + ((size_t)b * Hkv + h) * (size_t)N;
            for (int n = 0; n < N; ++n) mh[n] = 0.0;
            for (int g = 0; g < G; ++g)
                for (int s = 0; s < S; ++s) {
                    const double *qv = qwin + (((size_t)b * Hq + (size_t)h * G + g) * S + s) * d;
                    double m = -INFINITY;
                    for (int n = 0; n < N; ++n) {
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c) dot += qv[c] * kh[(size_t)n * d + c];
                        z[n] = dot * scale;
                        if (z[n] > m) m = z[n];
                    }
                    double l = 0.0;
                    for (int n = 0; n < N; ++n) {
                        z[n] = exp(z[n] - m);
                        l += z[n];
                    }
                    for (int n = 0; n < N; ++n) mh[n] += z[n] / l;
                }
        }
    free(z);
    return 0;
}

int oracle_select_tokens(const double *mass, int B, int Hkv, int N, int M, int32_t *kept)
{
    if (B < 0 || Hkv < 0 || N < 1 || M < 1 || M > N) return -1;
    int *order = (int *)malloc((size_t)N * sizeof(int));
    if (!order) return -2;
    for (long long bh = 0; bh < (long long)B * Hkv; ++bh) {
        for (int n = 0; n < N; ++n) order[n] = n;
        g_sort_scores = mass + (size_t)bh * N;
        qsort(order, (size_t)N, sizeof(int), by_score_desc);
        qsort(order, (size_t)M, sizeof(int), ascending_int);
        for (int t = 0; t < M; ++t) kept[(size_t)bh * M + t] = order[t];
    }
    free(order);
    g_sort_scores = NULL;
    return 0;
}

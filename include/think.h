/*
 * think.h -- C ABI of the ThinK decode-time hot path on NVIDIA B200 (sm_100a).
 *
 * Method: "ThinK: Thinner Key Cache by Query-Driven Pruning" (Xu et al., ICLR
 * 2025).  Its method section gives the flow (technical framework): compute
 * every key channel's relevance to the query, sort the channels, prune the
 * least relevant ones, then run inference with the pruned ("thinner") key
 * cache; its abstract states the aim of the ranking (lose as little of the
 * attention weights as possible).  The library implements that flow as four
 * calls, each one hand-written CUDA kernel:
 *
 *   think_score_channels      s[c] = sum_g ||Qwin_g[:,c]||_2 * ||K[:,c]||_2
 *   think_select_channels     keep the T largest s[c] (ties: lower index)
 *   think_compact_keys        K'[n,t] = K[n, idx[t]]   (V is not touched)
 *   think_pruned_decode_attn  out = softmax((q[idx] . K'^T) / sqrt(d)) V
 *
 * plus think_prune, the first three in two launches; think_append_keys,
 * which appends new tokens' keys to the thinner cache; a 4-bit thinner
 * cache (think_quantize_keys_q4, think_pruned_decode_attn_q4); a kept
 * width per head (think_select_adaptive, think_prune_adaptive and the _ragged
 * calls); and token
 * eviction to compose with it (think_token_mass, think_select_tokens,
 * think_gather_tokens).
 *
 * Conventions shared by every call
 *   - Shapes: B batch, Hq query heads, Hkv KV heads (G = Hq/Hkv query heads
 *     share one KV head; query head h reads KV head h / G), N cached tokens,
 *     d head width (only d = 128 is built), S_obs window queries, T kept
 *     channels (1 <= T <= d).
 *   - dtype: THINK_BF16 (bfloat16) or THINK_F32 (float32) for every input
 *     tensor of a call; accumulation is fp32 (decode) and fp64 (scores).
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned.  Strides are
 *     in ELEMENTS and must be multiples of 16 bytes / element size; the last
 *     dimension (channels) is always contiguous.
 *   - Ownership: the caller owns every buffer, including workspaces.  No call
 *     allocates, frees or synchronises.  Every call validates its arguments
 *     on the host before any CUDA call, then enqueues its kernels on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream) and
 *     returns.  Kernel faults surface at the caller's next synchronisation.
 *   - Errors: a call that returns anything but THINK_OK launched nothing
 *     (except THINK_ERR_CUDA, returned when a launch itself failed).
 *   - Empty batches (B == 0 or Hkv == 0) return THINK_OK and launch nothing.
 *   - Inputs must be finite; selection on NaN/Inf keys is unspecified.
 *   - Calls on different streams with disjoint buffers may run concurrently;
 *     calls that share a workspace must be stream-ordered.
 *   - Workspaces hold arrival counters that every call leaves at zero; where
 *     they sit depends on the call's shape (and, in a score workspace, on the
 *     split plan).  One workspace may serve calls of any shape it is large
 *     enough for: the library remembers, per workspace address, where the
 *     counters of the last call on it were, and when a call's counters sit
 *     elsewhere it zeroes them first (a memset on the call's stream).  The
 *     first call on an address relies on think_workspace_init.
 */
#ifndef THINK_H_
#define THINK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    THINK_OK = 0,
    THINK_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, T out of range, ... */
    THINK_ERR_UNSUPPORTED = 2,   /* d != 128, group size not in {1,2,4,8}, ... */
    THINK_ERR_WORKSPACE = 3,     /* workspace missing or too small */
    THINK_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    THINK_ERR_ALIGNMENT = 5      /* pointer or stride not 16-byte aligned */
} think_status_t;

typedef enum { THINK_F32 = 0, THINK_BF16 = 1 } think_dtype_t;

/* Device-side status bits written into the first 4 bytes of a decode or
 * score workspace when a bounded wait (2 s) inside a kernel gives up (the
 * kernel then returns early and its outputs are invalid).  Read them with
 * think_read_device_status; clear them with think_workspace_init. */
#define THINK_DEVICE_TIMEOUT_FULL    0x1u   /* a tile load never arrived */
#define THINK_DEVICE_TIMEOUT_EMPTY   0x2u   /* a stage was never released */
#define THINK_DEVICE_TIMEOUT_READY   0x4u   /* a head's channel selection never became ready */
#define THINK_DEVICE_TIMEOUT_BARRIER 0x8u   /* a block-internal barrier was not reached */
#define THINK_DEVICE_OOB             0x10u  /* debug builds only: an index check failed (store skipped) */

/* Human-readable name of a status code (static string, never NULL). */
const char *think_status_string(think_status_t status);

/* Kept channels for pruning ratio lambda (ThinK abstract: prune the least
 * significant channels): T = floor((1 - lambda) * d + 0.5), clamped to
 * [1, d].  Returns 0 if d < 1 or lambda is not finite. */
int think_t_from_lambda(int d, double lambda);

/* Smallest valid token pitch of the thinner key cache for N tokens and the
 * given dtype: N rounded up to a multiple of 16 bytes.  Returns -1 if N < 0. */
int64_t think_pruned_ld(int64_t N, think_dtype_t dtype);

/* ---------------------------------------------------------------- score --
 * Channel relevance of the key cache to the observation window (ThinK,
 * method section: "compute each channel's relevance to the query"; abstract:
 * keep the attention weights Qwin K^T).  For each batch item b and KV head
 * h_kv, with the group's query heads g = h_kv*G .. h_kv*G+G-1:
 *     kn2[c]  = sum_n K[b,h_kv,n,c]^2
 *     s[c]    = sum_g sqrt(sum_s Qwin[b,g,s,c]^2) * sqrt(kn2[c])
 * which is the Frobenius norm of channel c's rank-one share Qwin_g[:,c]K[:,c]^T
 * of the window's attention logits, summed over the group.  Arithmetic:
 * fp32 keys are squared and summed in fp64; bf16 keys are squared exactly,
 * summed four tokens at a time in fp32, then in fp64 (kn2 within 1.8e-7
 * relative for keys of magnitude in [2^-63, 2^64)); window energies and the
 * score in fp64.
 *
 *   q_win     [B][Hq][S_obs][d] contiguous, dtype.  May be NULL if S_obs == 0.
 *   k         key cache; element (b,h,n,c) at k[b*k_strides[0] + h*k_strides[1]
 *             + n*k_strides[2] + c].
 *   scores    [B][Hkv][d] fp64 output, contiguous.
 *   workspace device scratch of at least think_score_workspace_size() bytes,
 *             16-byte aligned, zeroed once by think_workspace_init before its
 *             first use (it holds arrival counters that every call leaves at
 *             zero, see the workspace rule above; the rest is scratch).
 * One kernel launch.  Bit-for-bit deterministic for a given shape (fixed
 * summation order).  N == 0 or S_obs == 0 gives all-zero scores. */
size_t think_score_workspace_size(int B, int Hq, int Hkv, int64_t N, int d);
think_status_t think_score_channels(const void *q_win, const void *k, const int64_t k_strides[3],
                                    int B, int Hq, int Hkv, int64_t N, int S_obs, int d,
                                    think_dtype_t dtype, double *scores,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------- select --
 * Top-T channels per (b, h_kv) (ThinK, method section: sort the channels by
 * relevance and prune the low ones).  Order: larger score first, equal
 * scores by lower channel index.  The kept channels are written in ascending
 * channel order, so T = d gives idx = 0..d-1.
 *   scores  [B][Hkv][d] fp64 (as written by think_score_channels; >= 0).
 *   idx     [B][Hkv][T] int32 output, contiguous, 4-byte aligned. */
think_status_t think_select_channels(const double *scores, int B, int Hkv, int d, int T,
                                     int32_t *idx, void *stream);

/* -------------------------------------------------------------- compact --
 * Thinner key cache (ThinK title and method section: the key cache keeps only
 * the selected channels; V is left as it is).  K'[n,t] = K[n, idx[t]], a pure
 * copy (bit-exact).  K' is stored channel-major so that decode reads each kept
 * channel as one contiguous run of tokens:
 *     element (b, h, t, n) of K' at k_pruned[((b*Hkv + h)*T + t)*ldk + n]
 * with ldk >= N and ldk*sizeof(dtype) a multiple of 16 (see think_pruned_ld).
 * Columns n in [N, ldk) are not written.
 *   k, k_strides as for think_score_channels; idx [B][Hkv][T] int32, each in
 *   [0, d) (checked on the device: an out-of-range index copies zeros). */
think_status_t think_compact_keys(const void *k, const int64_t k_strides[3], int B, int Hkv,
                                  int64_t N, int d, think_dtype_t dtype, const int32_t *idx,
                                  int T, void *k_pruned, int64_t ldk, void *stream);

/* --------------------------------------------------------------- append --
 * Growing cache (after the prune; the ThinK pages only say that inference
 * runs with the pruned cache, and this library reads new tokens' keys the
 * same way as the cached ones): the keys of n_new new tokens are compacted
 * with each head's kept channels, fixed at prune time, and written to token
 * columns [n_at, n_at + n_new) of K':
 *     K'[b,h,t, n_at + n] = k_new[b,h,n, idx[b,h,t]]      (a pure copy)
 *   k_new, k_strides  [B][Hkv][n_new][d] keys of the new tokens (layout as K
 *                     in think_score_channels).
 *   idx, T, k_pruned, ldk  as for think_compact_keys.
 *   n_at              first column to write, usually the current cache
 *                     length; n_at + n_new <= ldk (the capacity of a K' row),
 *                     else THINK_ERR_INVALID_ARG.  Other columns are not
 *                     touched; V is the caller's (append its rows as usual).
 * Decode the grown cache with think_pruned_decode_attn and N = n_at + n_new
 * (its workspace must be sized for that N).  n_new == 0 launches nothing.
 * One launch (the compaction kernel with a column offset). */
think_status_t think_append_keys(const void *k_new, const int64_t k_strides[3], int B, int Hkv,
                                 int64_t n_new, int d, think_dtype_t dtype, const int32_t *idx,
                                 int T, void *k_pruned, int64_t ldk, int64_t n_at, void *stream);

/* ---------------------------------------------------------------- prune --
 * The whole prune step of one layer in two launches: scores and the top-T
 * selection in one kernel (the last block of each head selects), then the
 * compaction.  Same results, bit for bit, as think_score_channels,
 * think_select_channels and think_compact_keys called in a row; arguments as
 * documented there.  With THINK_PRUNE_FUSED=1 in the environment a bf16 prune
 * runs as one persistent kernel instead (same results; its bounded waits
 * report through the workspace's status word, see think_read_device_status).
 * workspace: think_score_workspace_size() bytes, zeroed once before first use. */
think_status_t think_prune(const void *q_win, const void *k, const int64_t k_strides[3], int B,
                           int Hq, int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype,
                           int T, double *scores, int32_t *idx, void *k_pruned, int64_t ldk,
                           void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------- decode --
 * Decode attention with the thinner key cache (ThinK, method section: run
 * inference with the pruned cache).  For every query head h (KV head
 * h_kv = h / G):
 *     z[n]   = scale * sum_t q[b,h,idx[b,h_kv,t]] * K'[b,h_kv,t,n]
 *     out    = sum_n softmax(z)[n] * V[b,h_kv,n,:]
 * Pass scale = 1/sqrt(d) (the full head width, not T) for the unpruned
 * model's temperature.  Split-N flash decoding in one kernel launch: tiles of
 * K' and V are staged in shared memory by TMA, each block forms a partial
 * (max, sum, weighted V) for its split, and the partials of a KV head are
 * merged into `out`: through the workspace by the head's last block to
 * finish, or, for bf16 heads short enough that their splits form one
 * thread-block cluster, through the blocks' shared memory (the workspace's
 * partials are then not used).  fp32 caches are decoded with fp64 arithmetic
 * after the loads (one rounding to fp32 at the end).
 *   q         [B][Hq][d] contiguous, dtype.
 *   k_pruned  thinner key cache with pitch ldk, as written by think_compact_keys.
 *   v         element (b,h,n,c) at v[b*v_strides[0] + h*v_strides[1] + n*v_strides[2] + c].
 *   idx       [B][Hkv][T] int32 kept channels, each in [0, d).
 *   out       [B][Hq][d] fp32 output, contiguous.
 *   workspace at least think_decode_workspace_size() bytes, 16-byte aligned,
 *             zeroed once by think_workspace_init before its first use.  Its
 *             first 4 bytes hold the device status bits, then come per-head
 *             arrival counters that every completed call leaves at zero; the
 *             rest is scratch.
 * Requires N >= 1 and G in {1, 2, 4, 8}. */
size_t think_decode_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, think_dtype_t dtype);
think_status_t think_pruned_decode_attn(const void *q, const void *k_pruned, int64_t ldk,
                                        const void *v, const int64_t v_strides[3],
                                        const int32_t *idx, int B, int Hq, int Hkv, int64_t N,
                                        int d, int T, think_dtype_t dtype, float scale,
                                        float *out, void *workspace, size_t workspace_bytes,
                                        void *stream);

/* ---------------------------------------------- decode without allocation --
 * No counterpart in the paper: an implementation convenience.  Some callers
 * may not allocate device memory at all, e.g. a library running inside a
 * host framework that owns the whole device-memory budget, or a
 * latency-critical path where an allocation (which can synchronise the
 * device) is not allowed.  This entry point is think_pruned_decode_attn with
 * its workspace replaced by a scratch array that the library holds in device
 * memory (think_noalloc_scratch_bytes() bytes, 4 MiB, on every GPU that loads
 * the library, until the process exits).  Arguments and results are those of
 * think_pruned_decode_attn.
 *   - It calls no cudaMalloc or cudaFree.  The first call on a device looks
 *     up the array's device address (cudaGetSymbolAddress) with that device
 *     current; make that first call before any stream capture.
 *   - Every call clears the array's counters (a stream-ordered memset) and
 *     then uses the array; all calls share it, so calls that overlap on the
 *     GPU (different streams, or different host threads without ordering)
 *     race and give wrong results.  Order them on one stream.
 *   - A problem whose workspace (think_decode_workspace_size) exceeds the
 *     array returns THINK_ERR_WORKSPACE and launches nothing.
 *   - The kernels' device status word (THINK_DEVICE_TIMEOUT_* bits) lives in
 *     the array's first 4 bytes; each call clears it.  Read it after a call
 *     with think_noalloc_read_device_status (a non-zero value means that
 *     call's outputs are invalid).
 *   - The array's device address is looked up once per device and kept for
 *     the life of the process; after cudaDeviceReset the library must be
 *     reloaded before this entry point is used again on that device. */
size_t think_noalloc_scratch_bytes(void);
think_status_t think_pruned_decode_attn_noalloc(const void *q, const void *k_pruned, int64_t ldk,
                                                const void *v, const int64_t v_strides[3],
                                                const int32_t *idx, int B, int Hq, int Hkv,
                                                int64_t N, int d, int T, think_dtype_t dtype,
                                                float scale, float *out, void *stream);
/* The device status word of the no-allocation decode on the current device
 * (that of the last call ordered before this one on `stream`): copies it to
 * *status and synchronises `stream`, like think_read_device_status.  No
 * counterpart on the pages; it allocates nothing.  THINK_ERR_INVALID_ARG for a
 * null status, THINK_ERR_CUDA if a CUDA call fails. */
think_status_t think_noalloc_read_device_status(uint32_t *status, void *stream);

/* ---------------------------------------------------------- 4-bit K' --
 * The thinner key cache at 4 bits per element (ThinK abstract and method
 * section, technical framework: the pruned cache combines with KV-cache
 * quantisation such as KIVI; MiniKV page, quantisation: keys quantised per
 * (sub-)channel).  Reading used here: for each (b, h_kv), kept channel t and
 * group of 128 consecutive tokens,
 *     mn = min, scale = (max - mn) / 15                          (fp32)
 *     code = 0 if scale == 0, else clamp(rint((K'[n,t] - mn) / scale), 0, 15)
 *     dequantised key = bf16(fma(code, scale, mn))               (fp32, RNE)
 * each step the IEEE fp32 operation written (rint rounds half to even).
 *   codes   [B][Hkv][T][ldq] bytes: token n of row t in byte n/2, the even
 *           token in the low nibble; ldq >= think_q4_ld(N), a multiple of 64.
 *   groups  [B][Hkv][ldq/64][T2][2] fp32 (scale, mn) per 128-token group,
 *           T2 = T rounded up to even (the pad row is zero);
 *           think_q4_groups_bytes(B, Hkv, ldq*2, T) bytes.
 * bf16 only.  Token columns past N in the last group get code 0. */
int64_t think_q4_ld(int64_t N);   /* bytes per codes row: 64 per 128 tokens; -1 if N < 0 */
size_t think_q4_groups_bytes(int B, int Hkv, int64_t N, int T);
/* Quantise the bf16 thinner cache k_pruned (layout of think_compact_keys,
 * pitch ldk) into codes and group parameters.  One launch. */
think_status_t think_quantize_keys_q4(const void *k_pruned, int64_t ldk, int B, int Hkv, int64_t N, int T,
                                      uint8_t *codes, int64_t ldq, float *groups, void *stream);
/* think_pruned_decode_attn over the 4-bit thinner cache: the keys are the
 * dequantised values above; q, v bf16; everything else (layouts, scale,
 * workspace of think_decode_workspace_size(..., THINK_BF16), status bits) as
 * there.  One launch. */
think_status_t think_pruned_decode_attn_q4(const void *q, const uint8_t *codes, int64_t ldq,
                                           const float *groups, const void *v, const int64_t v_strides[3],
                                           const int32_t *idx, int B, int Hq, int Hkv, int64_t N, int d, int T,
                                           float scale, float *out, void *workspace, size_t workspace_bytes,
                                           void *stream);

/* ------------------------------------------------- adaptive kept width --
 * A kept width per head (ThinK method section, key design 3: the pruning
 * ratio adapts to the query and the cache; key design 2: keep the
 * attention-weight loss small).  Reading used here: rank a head's channels as
 * think_select_channels does; with E the sum of the squared scores in rank
 * order and cum_k the sum of the first k of them (fp64, sequential),
 *     T_h = the smallest k in [T_min, T_max] with cum_k >= tau * E
 *           (T_max if none, T_min if E == 0).
 * Ragged layout: head h = b*Hkv + h_kv owns rows rowoff[h] .. rowoff[h] +
 * P_h - 1 of K' and of idx, P_h = T_h rounded up to a multiple of 16;
 * rowoff[h] = P_0 + ... + P_{h-1}, rowoff[B*Hkv] = the rows in use.  Rows
 * T_h .. P_h - 1 of K' are zero (their idx entries are unspecified).  K' rows
 * have pitch ldk as in think_compact_keys; allocate think_ragged_rows() rows
 * for K' and idx.
 *   Th      [B*Hkv] int32 output;  rowoff [B*Hkv + 1] int32 output;
 *   idx     [rows] int32 output, each head's kept channels ascending. */
int64_t think_ragged_rows(int B, int Hkv, int T_max);   /* B*Hkv*roundup16(T_max); -1 on bad input */
/* One launch (one block for every head).  scores as written by
 * think_score_channels; 0 <= tau <= 1, 1 <= T_min <= T_max <= d. */
think_status_t think_select_adaptive(const double *scores, int B, int Hkv, int d, double tau, int T_min,
                                     int T_max, int32_t *Th, int32_t *rowoff, int32_t *idx, void *stream);
/* think_compact_keys for the ragged layout (writes the zero pad rows too).
 * One launch. */
think_status_t think_compact_keys_ragged(const void *k, const int64_t k_strides[3], int B, int Hkv, int64_t N,
                                         int d, think_dtype_t dtype, const int32_t *idx, const int32_t *Th,
                                         const int32_t *rowoff, int T_max, void *k_pruned, int64_t ldk,
                                         void *stream);
/* The whole prune with a kept width per head, as think_prune is for one T:
 * scores (think_score_channels), the adaptive selection
 * (think_select_adaptive) and the ragged compaction (think_compact_keys_ragged)
 * in three launches on `stream`, with the same outputs as those three calls.
 * Arguments as for those calls; workspace is the score workspace (its first
 * 4 bytes are the device status word, which the compaction's bounded waits
 * also use). */
think_status_t think_prune_adaptive(const void *q_win, const void *k, const int64_t k_strides[3], int B, int Hq,
                                    int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype, double tau,
                                    int T_min, int T_max, double *scores, int32_t *Th, int32_t *rowoff,
                                    int32_t *idx, void *k_pruned, int64_t ldk, void *workspace,
                                    size_t workspace_bytes, void *stream);
/* think_pruned_decode_attn for the ragged layout: query heads of KV head h
 * use its T_h kept channels; bf16 only; workspace as for
 * think_pruned_decode_attn.  One launch. */
think_status_t think_pruned_decode_attn_ragged(const void *q, const void *k_pruned, int64_t ldk, const void *v,
                                               const int64_t v_strides[3], const int32_t *idx,
                                               const int32_t *Th, const int32_t *rowoff, int T_max, int B, int Hq,
                                               int Hkv, int64_t N, int d, float scale, float *out,
                                               void *workspace, size_t workspace_bytes, void *stream);

/* ----------------------------------------------------- token eviction --
 * Token eviction composed with the channel pruning (ThinK abstract and
 * experiments: compared with and combined with KV-cache eviction; Keyformer
 * page: keep the tokens that receive the most attention).  Reading used here:
 *     mass[n] = sum over the group's query heads g and window rows s of
 *               softmax_n(scale * Qwin[b,g,s,:] . K[b,h_kv,n,:])
 * (the observation-window attention mass); each head keeps the M tokens of
 * largest mass, ties to the lower index, ascending.  The pipeline is
 * think_token_mass -> think_select_tokens -> think_gather_tokens (K and V)
 * -> think_prune on the gathered keys -> decode with N = M.
 *
 * think_token_mass: two launches (row statistics, then the masses) on the
 *   tensor cores; bf16 only; G * S_obs <= 512.  q_win [B][Hq][S_obs][d]
 *   contiguous; k, k_strides as for think_score_channels; mass [B][Hkv][N]
 *   fp32 output; workspace of think_token_mass_workspace_size() bytes, zeroed
 *   once before first use (per-head counters that every call leaves at zero;
 *   its first 4 bytes are the device status word). */
size_t think_token_mass_workspace_size(int B, int Hq, int Hkv, int64_t N, int S_obs);
think_status_t think_token_mass(const void *q_win, const void *k, const int64_t k_strides[3], int B, int Hq,
                                int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype, float scale, float *mass,
                                void *workspace, size_t workspace_bytes, void *stream);
/* kept [B][Hkv][M] int32 output: the M tokens of largest mass per head (ties
 * to the lower index), ascending; 1 <= M <= N <= INT32_MAX.  mass
 * [B][Hkv][N] fp32, contiguous, non-negative (as think_token_mass writes it).
 * Six launches, each over the whole GPU (a block per chunk of keys and head):
 * four 8-bit radix passes on the masses' bits for the M-th largest value,
 * a count per chunk, then the ordered write.  workspace: device scratch of
 * think_select_tokens_workspace_size() bytes, 16-byte aligned, zeroed once
 * (think_workspace_init) before its first use; every call leaves its radix
 * histograms at zero.  THINK_ERR_WORKSPACE if it is too small. */
size_t think_select_tokens_workspace_size(int B, int Hkv, int64_t N);
think_status_t think_select_tokens(const float *mass, int B, int Hkv, int64_t N, int M, int32_t *kept,
                                   void *workspace, size_t workspace_bytes, void *stream);
/* out[b,h,j,:] = x[b,h,kept[b,h,j],:], out contiguous [B][Hkv][M][d] (a copy;
 * an out-of-range index gives a zero row).  One launch. */
think_status_t think_gather_tokens(const void *x, const int64_t x_strides[3], int B, int Hkv, int64_t N, int d,
                                   think_dtype_t dtype, const int32_t *kept, int M, void *out, void *stream);

/* Zero a score or decode workspace (stream-ordered memset); the library
 * forgets the counter place it remembered for this address. */
think_status_t think_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Copy the device status bits of a decode or score workspace (its first 4
 * bytes) to *status after the stream's queued work has finished
 * (synchronises `stream`). */
think_status_t think_read_device_status(const void *workspace, uint32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* THINK_H_ */

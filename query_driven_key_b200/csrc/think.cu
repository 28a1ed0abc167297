// think.cu -- host side of the C ABI declared in include/think.h: argument
// validation, launch planning, TMA descriptors and kernel launches.
//
// Method: "ThinK: Thinner Key Cache by Query-Driven Pruning" (method section:
// score channels against the query, sort, prune, infer with the pruned cache).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <utility>

#include "decode_kernels.cuh"
#include "decode_f64.cuh"
#include "decode_mma.cuh"
#include "decode_q4.cuh"
#include "evict.cuh"
#include "mass_tc.cuh"
#include "decode_tc.cuh"
#include "prune_fused.cuh"
#include "prune_kernels.cuh"
#include "score_tma.cuh"
#include "compact_tma.cuh"
#include "think.h"

namespace think {
namespace {

constexpr int kTargetSMs = 148;             // B200
constexpr int kScoreResidentPerSM = 3;      // score blocks resident per SM (both score kernels)
constexpr int kScoreMaxWaves = 4;
constexpr int kPlanBlocks = 2 * kTargetSMs; // runs per round of the score plan
constexpr int64_t kRoundTilesMax = 2560;    // tiles per round (40 MB of bf16 keys; L2 holds two)
constexpr int kRunTilesMax = 64;            // tiles per run at most
constexpr int kCompactWaves = 4;            // waves of compact_tma_kernel blocks the plan aims for
constexpr int kDecodeBlocksPerSM = 2;       // decode blocks the plan aims to keep per SM
constexpr int kDecodePrefetchTiles = 0;     // tiles a decode block prefetches into L2 ahead of TMA
constexpr int kTcBlocksPerSM = 1;           // tcgen05 decode: blocks per SM the plan aims for
constexpr size_t kDecodeHeader = 256;       // status word + reserved, start of the workspace
constexpr size_t kSmemPerSM = 233472;       // 228 KB
constexpr size_t kSmemPerBlockMax = 232448; // 227 KB opt-in
constexpr size_t kSmemReservedPerBlock = 1024;

inline bool env_flag(const char *name)
{
    const char *v = std::getenv(name);
    return v && v[0] == '1';
}

inline int env_int(const char *name, int dflt, int lo, int hi)
{
    const char *v = std::getenv(name);
    if (!v || !*v) return dflt;
    const int x = std::atoi(v);
    return x < lo ? lo : (x > hi ? hi : x);
}

inline size_t esize(think_dtype_t t) { return t == THINK_BF16 ? 2 : 4; }
inline bool dtype_ok(int t) { return t == THINK_F32 || t == THINK_BF16; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline think_status_t launch_status()
{
    return cudaGetLastError() == cudaSuccess ? THINK_OK : THINK_ERR_CUDA;
}

// Arrival counters.  Several kernels count arrivals (blocks of a head, runs of
// a group) in counters that live in the caller's workspace and that every
// call leaves at zero.  Where they sit depends on the call's shape (B x Hkv,
// N) and, in a score workspace, on its split plan; a workspace reused for a
// call whose counters sit elsewhere may hold the earlier call's scratch
// values there.  So the library remembers, per workspace address, the byte
// range of the counters of the last call made on it, and zeroes the new range
// first (a memset in stream order) when it differs.  The first call on an
// address relies on think_workspace_init, which also forgets the address.
std::mutex g_counters_mu;
std::unordered_map<const void *, std::pair<size_t, size_t>> g_counters;

think_status_t ready_counters(void *ws, size_t begin, size_t end, cudaStream_t st)
{
    if (end <= begin) return THINK_OK;
    {
        std::lock_guard<std::mutex> lock(g_counters_mu);
        auto it = g_counters.find(ws);
        if (it == g_counters.end()) {
            if (g_counters.size() >= 65536) g_counters.clear();
            g_counters.emplace(ws, std::make_pair(begin, end));
            return THINK_OK;
        }
        if (it->second == std::make_pair(begin, end)) return THINK_OK;
        it->second = std::make_pair(begin, end);
    }
    return cudaMemsetAsync(static_cast<unsigned char *>(ws) + begin, 0, end - begin, st) == cudaSuccess
               ? THINK_OK
               : THINK_ERR_CUDA;
}

void forget_counters(const void *ws)
{
    std::lock_guard<std::mutex> lock(g_counters_mu);
    g_counters.erase(ws);
}

// Launch with programmatic stream serialisation (the kernel may start while
// the previous kernel of the stream drains; it waits in griddepcontrol.wait
// before its first global access).  THINK_PDL=0 launches plainly.
// With cluster > 0, blocks (x, y) .. (x + cluster - 1, y), x a multiple of
// cluster, form one thread-block cluster.
template <typename... KArgs, typename... Args>
think_status_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  int cluster, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (env_int("THINK_PDL", 1, 0, 1)) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? THINK_OK : THINK_ERR_CUDA;
}

template <typename... KArgs, typename... Args>
think_status_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args &&...args)
{
    return launch_pdl_cluster(kern, grid, block, smem, st, 0, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- plans --

// Split of each head's tokens for scoring, shared by the score kernels and
// the one-kernel prune (so that all add the squares in the same order): runs
// of s_tiles 64-token tiles, one score block per run.  The heads are also
// grouped in rounds of hpr heads for the one-kernel prune: a round holds about
// kPlanBlocks runs and at most kRoundTilesMax tiles, so that the prune can
// compact a round from L2 while it scores the next one.  The plan depends only
// on the shape.
struct ScorePlan {
    int splits;              // runs per head
    int s_tiles;             // 64-token tiles per run
    int64_t rows_per_split;  // = 64 * s_tiles
    int64_t tiles_per_head;
    int hpr, rounds;         // heads per round, rounds
    int groups;              // groups of kMergeGroup runs per head (the merge order)
};

// The one-kernel prune's plan: the run length L (tiles) that minimises
// rounds x runs-per-block x (L + 2); the 2 tiles stand for a run's fixed cost
// (partial sums, tickets).
ScorePlan plan_score_rounds(int64_t heads, int64_t N)
{
    const int64_t tph = std::max<int64_t>(1, ceil_div(N, kPfTile));
    heads = std::max<int64_t>(heads, 1);
    ScorePlan best{};
    int64_t best_cost = -1;
    for (int64_t L = 1; L <= std::min<int64_t>(kRunTilesMax, tph); ++L) {
        const int64_t R = ceil_div(tph, L);
        int64_t hpr = std::min<int64_t>(std::max<int64_t>(kPlanBlocks / R, 1), heads);
        if (hpr > 1 && hpr * tph > kRoundTilesMax) hpr = std::max<int64_t>(1, kRoundTilesMax / tph);
        const int64_t passes = ceil_div(hpr * R, kPlanBlocks);
        const int64_t rounds = ceil_div(heads, hpr);
        const int64_t cost = rounds * passes * (L + 2);
        if (best_cost < 0 || cost <= best_cost) {  // ties: the longer runs
            best_cost = cost;
            best.s_tiles = (int)L;
            best.splits = (int)R;
            best.hpr = (int)hpr;
            best.rounds = (int)rounds;
        }
    }
    best.tiles_per_head = tph;
    best.rows_per_split = (int64_t)best.s_tiles * kPfTile;
    best.groups = (int)ceil_div(best.splits, kMergeGroup);
    return best;
}

ScorePlan score_plan_from_tiles(int64_t tph, int64_t st)
{
    ScorePlan p{};
    p.tiles_per_head = tph;
    st = std::min<int64_t>(std::max<int64_t>(st, 1), tph);
    p.s_tiles = (int)st;
    p.rows_per_split = st * kPfTile;
    p.splits = (int)ceil_div(tph, st);
    p.groups = (int)ceil_div(p.splits, kMergeGroup);
    p.hpr = p.rounds = 0;  // not a round plan
    return p;
}

// The two-launch prune's plan (one score block per run): the shortest runs
// whose count fits W waves of the resident score blocks (148 SMs x
// kScoreResidentPerSM), for the fewest W (up to kScoreMaxWaves) whose runs
// fill at least 90% of their slots, else the best filled.  Whole waves leave
// no partly filled last wave, whose blocks would stream with the rest of the
// GPU idle.
ScorePlan plan_score_waves(int64_t heads, int64_t N, int waves)
{
    const int64_t tph = std::max<int64_t>(1, ceil_div(N, kPfTile));
    const int64_t slots = (int64_t)kTargetSMs * kScoreResidentPerSM * waves;
    const int64_t runs_per_head = std::max<int64_t>(1, slots / std::max<int64_t>(heads, 1));
    return score_plan_from_tiles(tph, ceil_div(tph, runs_per_head));
}

ScorePlan plan_score_two_launch(int64_t heads, int64_t N)
{
    ScorePlan best = plan_score_waves(heads, N, 1);
    double best_fill = 0.0;
    for (int w = 1; w <= kScoreMaxWaves; ++w) {
        const ScorePlan p = plan_score_waves(heads, N, w);
        const double fill = (double)(heads * p.splits) / ((double)kTargetSMs * kScoreResidentPerSM * w);
        if (fill >= 0.9) return p;
        if (fill > best_fill) {
            best_fill = fill;
            best = p;
        }
    }
    return best;
}

// The plan of a score pass.  The bits of the scores depend only on the plan
// (runs, then groups of runs, in a fixed order), so every score kernel gives
// the same bits for the same plan.  The one-kernel prune needs the round plan;
// the two-launch passes use the wave plan unless THINK_SCORE_PLAN_ROUNDS=1
// (for comparisons with the one-kernel prune).
ScorePlan plan_score(int64_t heads, int64_t N, bool fused = false)
{
    if (fused || env_int("THINK_SCORE_PLAN_ROUNDS", 0, 0, 1)) return plan_score_rounds(heads, N);
    return plan_score_two_launch(heads, N);
}

// The most runs per head of the plans above (workspace size).
int score_max_splits(int64_t heads, int64_t N)
{
    int m = plan_score_rounds(heads, N).splits;
    for (int w = 1; w <= kScoreMaxWaves; ++w) m = std::max(m, plan_score_waves(heads, N, w).splits);
    return m;
}

struct DecodeSplit {
    int splits;
    int tiles_per_split;
};

// Split the token axis so that heads*splits fills kDecodeBlocksPerSM blocks on
// every SM in one wave; each split is a whole number of 128-token tiles.
DecodeSplit plan_decode_split(int64_t heads, int64_t N, int blocks_per_sm = kDecodeBlocksPerSM)
{
    const int64_t tiles = ceil_div(N, kBN);
    const int64_t target = (int64_t)kTargetSMs * blocks_per_sm;
    int64_t s = std::max<int64_t>(1, target / std::max<int64_t>(heads, 1));
    s = std::min(s, tiles);
    const int64_t tps = ceil_div(tiles, s);
    DecodeSplit d;
    d.tiles_per_split = (int)tps;
    d.splits = (int)ceil_div(tiles, tps);
    return d;
}

double decode_fill(int64_t heads, int64_t N, int blocks_per_sm)
{
    const DecodeSplit d = plan_decode_split(heads, N, blocks_per_sm);
    const int64_t blocks = heads * d.splits;
    const int64_t slots = (int64_t)kTargetSMs * blocks_per_sm;
    const int64_t waves = ceil_div(blocks, slots);
    return (double)blocks / (double)(waves * slots);
}

struct DecodeSmem {
    uint32_t stage_bytes, v_off, tx_bytes;
    int stages;
    size_t bytes;
};

DecodeSmem plan_decode_smem(int T, int G, size_t es)
{
    DecodeSmem s;
    const size_t kt = (size_t)T * kBN * es;
    const size_t vb = (size_t)kBN * kD * es;
    s.v_off = (uint32_t)align_up(kt, 1024);
    s.stage_bytes = (uint32_t)align_up(s.v_off + vb, 1024);
    s.tx_bytes = (uint32_t)(kt + vb);
    const size_t extra = align_up((size_t)T * G, 4) * 4          /* q' */ +
                         (size_t)kConsumerWarps * 32 * G * 8          /* softmax weights (p, p) */ +
                         2 * 8 * 8 + 16 /* up to 8 stages of full+empty barriers, a flag */ +
                         1024 /* alignment slack */;
    const size_t per_block_2 = kSmemPerSM / kDecodeBlocksPerSM - kSmemReservedPerBlock;
    int st = (int)((per_block_2 - extra) / s.stage_bytes);
    if (st >= 2) {
        s.stages = std::min(st, 4);
    } else {
        st = (int)((kSmemPerBlockMax - extra) / s.stage_bytes);
        s.stages = std::min(std::max(st, 1), 4);
    }
    s.bytes = (size_t)s.stages * s.stage_bytes + extra;
    // The block merge ([warps][G][D] + [warps][G][2] floats) and the split merge
    // (2 x splits x G floats, splits <= 2 x 148) reuse the stage memory.
    return s;
}

// ------------------------------------------------------------ TMA maps --

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Encoded maps are kept in a small per-thread cache keyed by every input of
// the encoding (a decode step re-encodes the same two maps otherwise).
struct MapKey {
    const void *base;
    uint64_t dims[4], strides[3];
    uint32_t box[2];
    int dtype, swizzle;
};

bool map_cache_find(const MapKey &k, CUtensorMap *m);
void map_cache_put(const MapKey &k, const CUtensorMap &m);

// 4-D map over (x, y, z, w) with element strides sy, sz, sw for y, z, w; box (bx, by, 1, 1).
bool make_map_4d(CUtensorMap *m, think_dtype_t dt, const void *base, uint64_t dx, uint64_t dy,
                 uint64_t dz, uint64_t dw, int64_t sy, int64_t sz, int64_t sw, uint32_t bx,
                 uint32_t by, bool swizzle128 = false)
{
    MapKey key;
    memset(&key, 0, sizeof(key));
    key.base = base;
    key.dims[0] = dx, key.dims[1] = dy, key.dims[2] = dz, key.dims[3] = dw;
    key.strides[0] = (uint64_t)sy, key.strides[1] = (uint64_t)sz, key.strides[2] = (uint64_t)sw;
    key.box[0] = bx, key.box[1] = by;
    key.dtype = (int)dt;
    key.swizzle = swizzle128 ? 1 : 0;
    if (map_cache_find(key, m)) return true;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const size_t es = esize(dt);
    cuuint64_t dims[4] = {dx, dy, dz, dw};
    cuuint64_t strides[3] = {(cuuint64_t)sy * es, (cuuint64_t)sz * es, (cuuint64_t)sw * es};
    cuuint32_t box[4] = {bx, by, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, dt == THINK_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    map_cache_put(key, *m);
    return true;
}

constexpr int kMapCacheSize = 16;
struct MapCacheEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};
thread_local MapCacheEntry g_map_cache[kMapCacheSize];
thread_local int g_map_next = 0;

bool map_cache_find(const MapKey &k, CUtensorMap *m)
{
    for (int i = 0; i < kMapCacheSize; ++i)
        if (g_map_cache[i].used && memcmp(&g_map_cache[i].key, &k, sizeof(MapKey)) == 0) {
            *m = g_map_cache[i].map;
            return true;
        }
    return false;
}

void map_cache_put(const MapKey &k, const CUtensorMap &m)
{
    MapCacheEntry &e = g_map_cache[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCacheSize;
    e.key = k;
    e.map = m;
    e.used = true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel, device
// and size (per thread; the attribute itself is per device).
bool ensure_smem(const void *kern, size_t bytes)
{
    struct Entry {
        const void *kern;
        int dev;
        size_t bytes;
    };
    thread_local Entry seen[64];
    thread_local int nseen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    for (int i = 0; i < nseen; ++i)
        if (seen[i].kern == kern && seen[i].dev == dev && seen[i].bytes >= bytes) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    Entry &e = seen[nseen < 64 ? nseen++ : (int)(reinterpret_cast<uintptr_t>(kern) >> 4) % 64];
    e.kern = kern;
    e.dev = dev;
    e.bytes = bytes;
    return true;
}

// 4-D map of any element type with byte strides; box (bx, by, 1, 1), no swizzle.
bool make_map_raw_4d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t dx, uint64_t dy,
                     uint64_t dz, uint64_t dw, uint64_t sy_bytes, uint64_t sz_bytes, uint64_t sw_bytes,
                     uint32_t bx, uint32_t by)
{
    MapKey key;
    memset(&key, 0, sizeof(key));
    key.base = base;
    key.dims[0] = dx, key.dims[1] = dy, key.dims[2] = dz, key.dims[3] = dw;
    key.strides[0] = sy_bytes, key.strides[1] = sz_bytes, key.strides[2] = sw_bytes;
    key.box[0] = bx, key.box[1] = by;
    key.dtype = 100 + (int)dt;
    if (map_cache_find(key, m)) return true;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {dx, dy, dz, dw};
    cuuint64_t strides[3] = {sy_bytes, sz_bytes, sw_bytes};
    cuuint32_t box[4] = {bx, by, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    map_cache_put(key, *m);
    return true;
}

// ---------------------------------------------------------- validation --

bool strides_ok(const int64_t s[3], size_t es)
{
    const int64_t q = (int64_t)(16 / es);
    for (int i = 0; i < 3; ++i)
        if (s[i] < 0 || s[i] % q != 0) return false;
    return true;
}

template <typename TIn, int G>
think_status_t launch_decode_g(const CUtensorMap &mk, const CUtensorMap &mv, const DecodeArgs &a,
                               const DecodeSmem &sm, int heads, cudaStream_t st)
{
    auto kern = pruned_decode_kernel<TIn, G>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), sm.bytes))
        return THINK_ERR_CUDA;
    dim3 grid(a.splits, heads);
    kern<<<grid, kDecodeThreads, sm.bytes, st>>>(mk, mv, a);
    return launch_status();
}

template <typename TIn>
think_status_t launch_decode(int G, const CUtensorMap &mk, const CUtensorMap &mv,
                             const DecodeArgs &a, const DecodeSmem &sm, int heads, cudaStream_t st)
{
    switch (G) {
    case 1: return launch_decode_g<TIn, 1>(mk, mv, a, sm, heads, st);
    case 2: return launch_decode_g<TIn, 2>(mk, mv, a, sm, heads, st);
    case 4: return launch_decode_g<TIn, 4>(mk, mv, a, sm, heads, st);
    case 8: return launch_decode_g<TIn, 8>(mk, mv, a, sm, heads, st);
    default: return THINK_ERR_UNSUPPORTED;
    }
}


// ---------------------------------------------------------------- score --

// Score workspace: a 256-byte header (status word at 0; the one-kernel
// prune's block-exit counter at 8), per-head ready flags (one-kernel prune),
// per-head tickets, per-(head, group) tickets, window-query energies, per-run
// channel energies, per-group sums.
struct ScoreWs {
    size_t status, exits, ready, tickets, gtickets, qn2, part, gpart, total;  // byte offsets, size
};

ScoreWs score_ws_layout(int64_t heads, int G, const ScorePlan &p)
{
    ScoreWs w;
    w.status = 0;
    w.exits = 8;
    w.ready = 256;
    w.tickets = w.ready + align_up((size_t)heads * sizeof(unsigned), 256);
    w.gtickets = w.tickets + align_up((size_t)heads * sizeof(unsigned), 256);
    w.qn2 = w.gtickets + align_up((size_t)heads * p.groups * sizeof(unsigned), 256);
    w.part = w.qn2 + align_up((size_t)heads * G * kD * sizeof(double), 256);
    w.gpart = w.part + align_up((size_t)heads * p.splits * kD * sizeof(double), 256);
    w.total = w.gpart + (size_t)heads * p.groups * kD * sizeof(double);
    return w;
}

ScoreWs score_ws_layout_max(int64_t heads, int G, int64_t N)
{
    ScorePlan p = plan_score_rounds(heads, N);
    p.splits = score_max_splits(heads, N);
    p.groups = (int)ceil_div(p.splits, kMergeGroup);
    return score_ws_layout(heads, G, p);
}

// The score fields of ScoreArgs that live in the workspace.
void set_score_ws(ScoreArgs &a, unsigned char *ws, const ScoreWs &w, const ScorePlan &p)
{
    a.rows_per_split = p.rows_per_split;
    a.splits = p.splits;
    a.groups = p.groups;
    a.tickets = reinterpret_cast<unsigned *>(ws + w.tickets);
    a.gtickets = reinterpret_cast<unsigned *>(ws + w.gtickets);
    a.qn2 = reinterpret_cast<double *>(ws + w.qn2);
    a.part = reinterpret_cast<double *>(ws + w.part);
    a.gpart = reinterpret_cast<double *>(ws + w.gpart);
    a.status = reinterpret_cast<unsigned *>(ws + w.status);
}

think_status_t validate_score(const void *q_win, const void *k, const int64_t k_strides[3], int B,
                              int Hq, int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype,
                              const double *scores, const void *workspace, size_t workspace_bytes)
{
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0 || S_obs < 0) return THINK_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (Hq < Hkv || Hq % Hkv != 0) return THINK_ERR_INVALID_ARG;
    if (!k || !k_strides || !scores || !workspace || (S_obs > 0 && !q_win))
        return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535) return THINK_ERR_UNSUPPORTED;
    const size_t es = esize(dtype);
    if (!aligned16(k) || !aligned16(workspace) || (q_win && !aligned16(q_win)) ||
        !strides_ok(k_strides, es) || (reinterpret_cast<uintptr_t>(scores) & 7u))
        return THINK_ERR_ALIGNMENT;
    if (workspace_bytes < score_ws_layout_max(heads, Hq / Hkv, N).total)
        return THINK_ERR_WORKSPACE;
    return THINK_OK;
}

think_status_t launch_score(const void *q_win, const void *k, const int64_t k_strides[3], int B,
                            int Hq, int Hkv, int64_t N, int S_obs, think_dtype_t dtype, int T,
                            double *scores, int32_t *idx, void *workspace, cudaStream_t st)
{
    const int64_t heads = (int64_t)B * Hkv;
    const ScorePlan p = plan_score(heads, N);
    const ScoreWs w = score_ws_layout(heads, Hq / Hkv, p);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    ScoreArgs a;
    a.k = k;
    a.sb = k_strides[0];
    a.sh = k_strides[1];
    a.sn = k_strides[2];
    a.qwin = q_win;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.S = S_obs;
    a.N = N;
    set_score_ws(a, ws, w, p);
    if (ready_counters(ws, w.ready, w.qn2, st) != THINK_OK) return THINK_ERR_CUDA;
    a.scores = scores;
    a.T = T;
    a.idx = idx;
    a.stages = env_int("THINK_SCORE_STAGES", 4, 2, kStMaxStages);
    dim3 grid(p.splits, (unsigned)heads);
    // bf16: key tiles staged by TMA when a tensor map can describe K
    // (THINK_SCORE_TMA=0 selects the register-pipelined kernel, for comparison)
    CUtensorMap mk;
    if (dtype == THINK_BF16 && N > 0 && N <= (int64_t)INT32_MAX - kStTileRows &&
        env_int("THINK_SCORE_TMA", 1, 0, 1) == 1 &&
        make_map_4d(&mk, THINK_BF16, k, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, k_strides[2],
                    k_strides[1], k_strides[0], 64, kStTileRows, true)) {
        const size_t bytes = score_tma_smem_bytes(a.stages);
        if (!ensure_smem(reinterpret_cast<const void *>(score_tma_kernel), bytes)) return THINK_ERR_CUDA;
        score_tma_kernel<<<grid, kStThreads, bytes, st>>>(mk, a);
        return launch_status();
    }
    if (dtype == THINK_BF16)
        score_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
    else
        score_kernel<float><<<grid, 256, 0, st>>>(a);
    return launch_status();
}

think_status_t validate_compact(const void *k, const int64_t k_strides[3], int B, int Hkv, int64_t N,
                                int d, think_dtype_t dtype, const int32_t *idx, int T,
                                const void *k_pruned, int64_t ldk)
{
    if (B < 0 || Hkv < 0 || N < 0) return THINK_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (T < 1 || T > d) return THINK_ERR_INVALID_ARG;
    if (ldk < N) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0 || N == 0) return THINK_OK;
    if (!k || !k_strides || !idx || !k_pruned) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535) return THINK_ERR_UNSUPPORTED;
    const size_t es = esize(dtype);
    if (!aligned16(k) || !aligned16(k_pruned) || !strides_ok(k_strides, es) ||
        (ldk * (int64_t)es) % 16 != 0 || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return THINK_ERR_ALIGNMENT;
    if (ceil_div(N, 64) > INT32_MAX) return THINK_ERR_UNSUPPORTED;
    return THINK_OK;
}

think_status_t launch_compact(const void *k, const int64_t k_strides[3], int B, int Hkv, int64_t N,
                              think_dtype_t dtype, const int32_t *idx, int T, void *k_pruned,
                              int64_t ldk, cudaStream_t st, int64_t col0 = 0, const int32_t *Th = nullptr,
                              const int32_t *rowoff = nullptr)
{
    const int64_t heads = (int64_t)B * Hkv;
    const int bnc = dtype == THINK_BF16 ? CompactTokens<__nv_bfloat16>::value : CompactTokens<float>::value;
    dim3 grid((unsigned)ceil_div(N, bnc), (unsigned)heads);
    if (dtype == THINK_BF16)
        compact_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(k), k_strides[0], k_strides[1], k_strides[2], Hkv, N,
            idx, T, static_cast<__nv_bfloat16 *>(k_pruned), ldk, col0, Th, rowoff);
    else
        compact_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(k), k_strides[0],
                                                    k_strides[1], k_strides[2], Hkv, N, idx, T,
                                                    static_cast<float *>(k_pruned), ldk, col0, Th, rowoff);
    return launch_status();
}


// Tiles per block of compact_tma_kernel: runs that give about
// kCompactWaves waves of the resident block slots, at least 4 tiles
// (THINK_COMPACT_TILES overrides, for tuning).
int plan_compact_tma(int64_t heads, int64_t tiles)
{
    const int64_t slots = (int64_t)kTargetSMs * kScoreResidentPerSM * kCompactWaves;
    const int64_t rph = std::max<int64_t>(1, slots / std::max<int64_t>(heads, 1));
    int64_t rt = std::max<int64_t>(4, ceil_div(tiles, rph));
    rt = env_int("THINK_COMPACT_TILES", (int)std::min<int64_t>(rt, 1 << 20), 1, 1 << 20);
    return (int)std::min<int64_t>(rt, tiles);
}

// The TMA compaction for bf16 keys within think_prune (its workspace holds
// the status word).  Returns THINK_ERR_UNSUPPORTED, having launched nothing,
// when the keys cannot be described by a tensor map, or with
// THINK_COMPACT_TMA=0.
think_status_t launch_compact_tma(const void *k, const int64_t k_strides[3], int B, int Hkv, int64_t N,
                                  const int32_t *idx, int T, void *k_pruned, int64_t ldk, void *workspace,
                                  cudaStream_t st, const int32_t *Th = nullptr, const int32_t *rowoff = nullptr)
{
    if (env_int("THINK_COMPACT_TMA", 1, 0, 1) == 0 || N > (int64_t)INT32_MAX - kCtTileRows)
        return THINK_ERR_UNSUPPORTED;
    const int64_t heads = (int64_t)B * Hkv;
    CUtensorMap mk;
    if (!make_map_4d(&mk, THINK_BF16, k, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, k_strides[2],
                     k_strides[1], k_strides[0], 64, kCtTileRows, true))
        return THINK_ERR_UNSUPPORTED;
    CompactTmaArgs a;
    a.Hkv = Hkv;
    a.T = T;
    a.tiles = ceil_div(N, kCtTileRows);
    a.run_tiles = plan_compact_tma(heads, a.tiles);
    a.stages = env_int("THINK_COMPACT_STAGES", 4, 2, kCtMaxStages);
    a.N = N;
    a.ldk = ldk;
    a.idx = idx;
    a.kp = static_cast<__nv_bfloat16 *>(k_pruned);
    a.status = reinterpret_cast<unsigned *>(static_cast<unsigned char *>(workspace));  // score workspace word 0
    a.Th = Th;
    a.rowoff = rowoff;
    a.row_cap = heads * ((T + 15) & ~15);
    const size_t bytes = compact_tma_smem_bytes(a.stages);
    if (!ensure_smem(reinterpret_cast<const void *>(compact_tma_kernel), bytes)) return THINK_ERR_CUDA;
    dim3 grid((unsigned)ceil_div(a.tiles, a.run_tiles), (unsigned)heads);
    return launch_pdl(compact_tma_kernel, grid, dim3(kCtThreads), bytes, st, mk, a);
}

// ---------------------------------------------------------- fused prune --

int device_sm_count()
{
    thread_local int cached_dev = -1, cached_sms = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev != cached_dev) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached_dev = dev;
        cached_sms = sms;
    }
    return cached_sms;
}

// Whether the one-kernel prune serves this shape: bf16, N > 0, groups of at
// most 8 query heads, a round of the plan (two of which must fit in L2) no
// larger than kRoundTilesMax tiles.
bool prune_fused_applies(think_dtype_t dtype, int64_t heads, int G, int64_t N)
{
    if (dtype != THINK_BF16 || N <= 0 || N > (int64_t)INT32_MAX - kPfTile || G > 8) return false;
    if (env_int("THINK_PRUNE_FUSED", 0, 0, 1) == 0) return false;
    const ScorePlan p = plan_score(heads, N, true);
    return (int64_t)p.hpr * p.tiles_per_head <= kRoundTilesMax;
}

// The one-kernel prune (bf16, N > 0).  Returns THINK_ERR_UNSUPPORTED, having
// launched nothing, when a tensor map cannot be built for these strides.
// THINK_PRUNE_STAGES and THINK_PRUNE_CSTAGES set the depths of the score and
// compaction rings (default 7 and 4 tiles), THINK_PRUNE_LAG how many rounds
// the scoring may run ahead of the compaction; THINK_PRUNE_HINTS the L2 policies
// (bits: 1 score loads evict-last, 2 compact loads evict-first, 4 K' stores
// evict-first).  None of them changes the results.
think_status_t launch_prune_fused(const void *q_win, const void *k, const int64_t k_strides[3], int B,
                                  int Hq, int Hkv, int64_t N, int S_obs, int T, double *scores,
                                  int32_t *idx, void *k_pruned, int64_t ldk, void *workspace,
                                  cudaStream_t st)
{
    const int64_t heads = (int64_t)B * Hkv;
    const ScorePlan p = plan_score(heads, N, true);
    const ScoreWs w = score_ws_layout(heads, Hq / Hkv, p);
    CUtensorMap mk;
    if (!make_map_4d(&mk, THINK_BF16, k, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, k_strides[2],
                     k_strides[1], k_strides[0], 64, kPfTile, true))
        return THINK_ERR_UNSUPPORTED;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    PruneFusedArgs a;
    memset(&a, 0, sizeof(a));
    a.sc.k = k;
    a.sc.qwin = q_win;
    a.sc.Hq = Hq;
    a.sc.Hkv = Hkv;
    a.sc.S = S_obs;
    a.sc.N = N;
    set_score_ws(a.sc, ws, w, p);
    if (ready_counters(ws, w.ready, w.qn2, st) != THINK_OK) return THINK_ERR_CUDA;
    a.sc.scores = scores;
    a.sc.T = T;
    a.sc.idx = idx;
    a.G = Hq / Hkv;
    a.T = T;
    a.heads = (int)heads;
    a.tiles_per_head = (int)p.tiles_per_head;
    a.s_tiles = p.s_tiles;
    a.hpr = p.hpr;
    a.rounds = p.rounds;
    a.s_stages = env_int("THINK_PRUNE_STAGES", 7, 2, kPfMaxStages - 2);
    a.c_stages = env_int("THINK_PRUNE_CSTAGES", 4, 2, kPfMaxStages - a.s_stages);
    a.hints = env_int("THINK_PRUNE_HINTS", kPfHintScoreKeep | kPfHintCompactDrop, 0, 7);
    a.lag = env_int("THINK_PRUNE_LAG", 2, 1, 1 << 20);
    a.prefetch = env_int("THINK_PRUNE_PREFETCH", 0, 0, 64);
    a.ready = reinterpret_cast<unsigned *>(ws + w.ready);
    a.exits = reinterpret_cast<unsigned *>(ws + w.exits);
    a.kp = static_cast<__nv_bfloat16 *>(k_pruned);
    a.ldk = ldk;
    a.N = N;
    const size_t bytes = prune_fused_smem_bytes(a.s_stages, a.c_stages);
    const void *kern = reinterpret_cast<const void *>(prune_fused_kernel);
    if (!ensure_smem(kern, bytes)) return THINK_ERR_CUDA;
    // every block must be resident at once (blocks wait for other blocks' flags)
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kPfThreads, bytes) != cudaSuccess || occ < 1)
        return THINK_ERR_CUDA;
    const int64_t sms = device_sm_count();
    if (sms < 1) return THINK_ERR_CUDA;
    const int64_t runs_per_round = (int64_t)p.hpr * p.splits;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sms * occ, runs_per_round));
    // A cooperative launch: the runtime starts the grid only when every block
    // can be resident at once (else the launch fails), so that no block waits
    // on a flag of a block that has not been scheduled.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prune_fused_kernel, mk, a) == cudaSuccess ? THINK_OK : THINK_ERR_CUDA;
}


// ---------------------------------------------------- warp-MMA decode --

struct MmaPlan {
    int stages, blocks_per_sm, warps;  // warps: consumer warps per block (4 or 8)
    size_t bytes;
};

inline int consumer_warps(int dflt) { return env_int("THINK_DECODE_WARPS", dflt, 4, 8) >= 6 ? 8 : 4; }

// One block per SM with up to 4 stages (the deeper ring streams faster) when
// that keeps at least 95% of the SMs busy, else two blocks per SM.
// THINK_DECODE_BLOCKS_PER_SM (1, 2) and THINK_DECODE_STAGES (2..4) cap the
// choice (tuning only).
MmaPlan plan_decode_mma(int T, int G, int64_t heads, int64_t N)
{
    MmaPlan p;
    const size_t per_block_2 = kSmemPerSM / 2 - kSmemReservedPerBlock;
    const int pref_bps = decode_fill(heads, N, 1) >= 0.95 ? 1 : 2;
    const int max_bps = env_int("THINK_DECODE_BLOCKS_PER_SM", pref_bps, 1, 2);
    const int max_st = env_int("THINK_DECODE_STAGES", 4, 2, 4);
    p.warps = consumer_warps(4);
    for (int bps = max_bps; bps >= 1; --bps)
        for (int st = max_st; st >= 2; --st) {
            const size_t bytes = mma_smem_bytes(T, G, st, p.warps);
            if (bytes <= (bps == 2 ? per_block_2 : kSmemPerBlockMax)) {
                p.stages = st;
                p.blocks_per_sm = bps;
                p.bytes = bytes;
                return p;
            }
        }
    p.stages = 0;
    p.blocks_per_sm = 1;
    p.bytes = 0;
    return p;
}

// Clusters of `cluster` blocks of `kern` (threads, bytes of shared memory)
// that can be resident at once on this device; 0 if the launch cannot form
// them.  Cached per kernel, device, cluster size and shared-memory size.
int max_active_clusters(const void *kern, int cluster, int threads, size_t bytes)
{
    struct Entry {
        const void *kern;
        int dev, cluster;
        size_t bytes;
        int n;
    };
    thread_local Entry seen[32];
    thread_local int nseen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    for (int i = 0; i < nseen; ++i)
        if (seen[i].kern == kern && seen[i].dev == dev && seen[i].cluster == cluster && seen[i].bytes == bytes)
            return seen[i].n;
    int n = 0;
    bool refused = false;
    if (cluster > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        refused = true;
    if (!refused) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)cluster, 1, 1);
        cfg.blockDim = dim3((unsigned)threads, 1, 1);
        cfg.dynamicSmemBytes = bytes;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = (unsigned)cluster;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            n = 0;
            refused = true;
        }
    }
    // a refused size is an answer (0), not an error for the caller's next
    // check: clear the error state that the refusing call left, and only then
    if (refused) (void)cudaGetLastError();
    Entry &e = seen[nseen < 32 ? nseen++ : (cluster * 7 + (int)bytes) % 32];
    e.kern = kern;
    e.dev = dev;
    e.cluster = cluster;
    e.bytes = bytes;
    e.n = n;
    return n;
}

// The split merge through a thread-block cluster serves short heads: each
// head becomes one cluster of S blocks (S a power of two, 2..16) that merges
// its split partials in distributed shared memory (no global partials, no
// ticket), when
//   - a split reads at most kClusterTilesMax tiles (longer heads keep the
//     global merge, whose cost is small beside their stream),
//   - all heads' clusters are resident at once, and
//   - the busiest SM streams no more tiles than under the global merge's
//     split (tiles per block x blocks per SM, blocks spread evenly), so that
//     the coarser split costs no bandwidth.
// The largest such S below twice the head's tiles is taken (a split may be
// empty).  THINK_DECODE_CLUSTER caps S (0: never; tuning and tests).
constexpr int kClusterTilesMax = 8;

int plan_decode_cluster(const void *kern, int threads, size_t bytes, int64_t heads, int64_t N,
                        int global_splits, int global_tps)
{
    const int cap = env_int("THINK_DECODE_CLUSTER", 16, 0, 16);
    const int64_t tiles = ceil_div(N, kBN);
    const int64_t sms = device_sm_count();
    if (sms < 1) return 0;
    const int64_t global_load = (int64_t)global_tps * ceil_div(heads * global_splits, sms);
    for (int S = 16; S >= 2; S /= 2) {
        if (S > cap || S >= 2 * tiles) continue;  // no cluster of one tile; S < 2 x tiles
        const int64_t tps = ceil_div(tiles, S);
        if (tps > kClusterTilesMax || tps * ceil_div(heads * S, sms) > global_load) continue;
        if ((int64_t)max_active_clusters(kern, S, threads, bytes) >= heads) return S;
    }
    return 0;
}

template <int G, int CW>
think_status_t launch_decode_mma_gw(const CUtensorMap &mk, const CUtensorMap &mv, DecodeArgs a,
                                    size_t bytes, int heads, cudaStream_t st)
{
    auto kern = pruned_decode_mma_kernel<G, CW>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), bytes))
        return THINK_ERR_CUDA;
    const int S = plan_decode_cluster(reinterpret_cast<const void *>(kern), CW * 32 + 32, bytes, heads, a.N,
                                      a.splits, a.tiles_per_split);
    if (S > 0) {  // one cluster of S splits per head (a split may be empty)
        a.cluster = S;
        a.splits = S;
        a.tiles_per_split = (int)ceil_div(ceil_div(a.N, kBN), S);
    }
    dim3 grid(a.splits, heads);
    return launch_pdl_cluster(kern, grid, dim3(CW * 32 + 32), bytes, st, S, mk, mv, a);
}

template <int G>
think_status_t launch_decode_mma_g(int cw, const CUtensorMap &mk, const CUtensorMap &mv, const DecodeArgs &a,
                                   size_t bytes, int heads, cudaStream_t st)
{
    return cw == 8 ? launch_decode_mma_gw<G, 8>(mk, mv, a, bytes, heads, st)
                   : launch_decode_mma_gw<G, 4>(mk, mv, a, bytes, heads, st);
}

think_status_t launch_decode_mma(int G, int cw, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const DecodeArgs &a, size_t bytes, int heads, cudaStream_t st)
{
    switch (G) {
    case 1: return launch_decode_mma_g<1>(cw, mk, mv, a, bytes, heads, st);
    case 2: return launch_decode_mma_g<2>(cw, mk, mv, a, bytes, heads, st);
    case 4: return launch_decode_mma_g<4>(cw, mk, mv, a, bytes, heads, st);
    case 8: return launch_decode_mma_g<8>(cw, mk, mv, a, bytes, heads, st);
    default: return THINK_ERR_UNSUPPORTED;
    }
}

// ------------------------------------------------------- token eviction --

struct MassPlan {
    int ntw, r_pad, stages, blocks_per_sm;
    size_t bytes;
    DecodeSplit sp;
};

MassPlan plan_mass(int R, int64_t heads, int64_t N)
{
    MassPlan p;
    p.ntw = R <= 64 ? 1 : R <= 128 ? 2 : R <= 256 ? 4 : 8;
    p.r_pad = 8 * kMassWarps * p.ntw;
    const size_t per_block_2 = kSmemPerSM / 2 - kSmemReservedPerBlock;
    p.blocks_per_sm = mass_smem_bytes(p.r_pad, 2) <= per_block_2 ? 2 : 1;
    const size_t cap = p.blocks_per_sm == 2 ? per_block_2 : kSmemPerBlockMax;
    p.stages = 0;
    p.bytes = 0;
    for (int st = 4; st >= 2; --st)
        if (mass_smem_bytes(p.r_pad, st) <= cap) {
            p.stages = st;
            p.bytes = mass_smem_bytes(p.r_pad, st);
            break;
        }
    p.sp = plan_decode_split(heads, N, p.blocks_per_sm);
    return p;
}

struct MassWs {
    size_t tickets, part, stats, total;
};

MassWs mass_ws_layout(int64_t heads, int R, int splits)
{
    MassWs w;
    w.tickets = 256;
    w.part = w.tickets + align_up((size_t)heads * sizeof(unsigned), 256);
    w.stats = w.part + align_up((size_t)heads * splits * R * sizeof(float2), 256);
    w.total = w.stats + (size_t)heads * R * sizeof(float2);
    return w;
}

template <int PASS, int NTW>
think_status_t launch_mass_kernel(const CUtensorMap &mk, const MassArgs &a, const MassPlan &p, int heads,
                                  cudaStream_t st)
{
    auto kern = token_mass_kernel<PASS, NTW>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), p.bytes))
        return THINK_ERR_CUDA;
    dim3 grid(a.splits, heads);
    kern<<<grid, kMassThreads, p.bytes, st>>>(mk, a);
    return launch_status();
}

template <int NTW>
think_status_t launch_mass(const CUtensorMap &mk, const MassArgs &a, const MassPlan &p, int heads, cudaStream_t st)
{
    const think_status_t v = launch_mass_kernel<1, NTW>(mk, a, p, heads, st);
    if (v != THINK_OK) return v;
    return launch_mass_kernel<2, NTW>(mk, a, p, heads, st);
}

// The token mass on tcgen05 (mass_tc.cuh): R <= 256 window rows in MB = 1 or
// 2 blocks of 128, one block per SM, the deepest K ring (2..4 stages) that
// fits.  stages == 0: it does not apply (THINK_MASS_TC=0 also turns it off).
struct MassTcPlan {
    int mb, stages;
    size_t bytes;
    DecodeSplit sp;
};

MassTcPlan plan_mass_tc(int R, int64_t heads, int64_t N)
{
    MassTcPlan p{};
    if (R > 256 || env_int("THINK_MASS_TC", 1, 0, 1) == 0) return p;
    p.mb = R <= 128 ? 1 : 2;
    for (int st = 4; st >= 2; --st) {
        const size_t bytes = p.mb == 1 ? mass_tc_smem_bytes<1>(st) : mass_tc_smem_bytes<2>(st);
        if (bytes <= kSmemPerBlockMax) {
            p.stages = st;
            p.bytes = bytes;
            break;
        }
    }
    p.sp = plan_decode_split(heads, N, 1);
    return p;
}

template <int PASS, int MB>
think_status_t launch_mass_tc_kernel(const CUtensorMap &mk, const MassArgs &a, size_t bytes, int heads,
                                     cudaStream_t st)
{
    auto kern = token_mass_tc_kernel<PASS, MB>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), bytes))
        return THINK_ERR_CUDA;
    dim3 grid(a.splits, heads);
    kern<<<grid, MassTc<MB>::kThreads, bytes, st>>>(mk, a);
    return launch_status();
}

template <int MB>
think_status_t launch_mass_tc(const CUtensorMap &mk, const MassArgs &a, size_t bytes, int heads, cudaStream_t st)
{
    const think_status_t v = launch_mass_tc_kernel<1, MB>(mk, a, bytes, heads, st);
    if (v != THINK_OK) return v;
    return launch_mass_tc_kernel<2, MB>(mk, a, bytes, heads, st);
}

// ------------------------------------------------------------ 4-bit K' --

// Two blocks per SM of four consumer warps (32 tokens each) first: with one
// block per SM the dequantisation makes the consumers' latency, not the
// stream, the limit; at two blocks per SM four consumer warps beat eight of 16
// tokens, whose per-warp softmax and MMA set-up is paid twice per tile
// (long-context workload: 54.5 us against 56.7 us with eight warps, 66-71 us
// at one block per SM).
MmaPlan plan_decode_q4(int T, int G, int64_t heads, int64_t N)
{
    MmaPlan p;
    (void)heads;
    (void)N;
    const size_t per_block_2 = kSmemPerSM / 2 - kSmemReservedPerBlock;
    const int max_bps = env_int("THINK_DECODE_BLOCKS_PER_SM", 2, 1, 2);
    const int max_st = env_int("THINK_DECODE_STAGES", 6, 2, 6);
    p.warps = consumer_warps(4);
    for (int bps = max_bps; bps >= 1; --bps)
        for (int st = max_st; st >= 2; --st) {
            const size_t bytes = q4_smem_bytes(T, G, st, p.warps);
            if (bytes <= (bps == 2 ? per_block_2 : kSmemPerBlockMax)) {
                p.stages = st;
                p.blocks_per_sm = bps;
                p.bytes = bytes;
                return p;
            }
        }
    p.stages = 0;
    p.blocks_per_sm = 1;
    p.bytes = 0;
    return p;
}

template <int G, int CW>
think_status_t launch_decode_q4_gw(const CUtensorMap &mc, const CUtensorMap &mg, const CUtensorMap &mv,
                                   const DecodeArgs &a, size_t bytes, int heads, cudaStream_t st)
{
    auto kern = pruned_decode_q4_kernel<G, CW>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), bytes))
        return THINK_ERR_CUDA;
    dim3 grid(a.splits, heads);
    return launch_pdl(kern, grid, dim3(CW * 32 + 32), bytes, st, mc, mg, mv, a);
}

template <int G>
think_status_t launch_decode_q4_g(int cw, const CUtensorMap &mc, const CUtensorMap &mg, const CUtensorMap &mv,
                                  const DecodeArgs &a, size_t bytes, int heads, cudaStream_t st)
{
    return cw == 8 ? launch_decode_q4_gw<G, 8>(mc, mg, mv, a, bytes, heads, st)
                   : launch_decode_q4_gw<G, 4>(mc, mg, mv, a, bytes, heads, st);
}

think_status_t launch_decode_q4(int G, int cw, const CUtensorMap &mc, const CUtensorMap &mg,
                                const CUtensorMap &mv, const DecodeArgs &a, size_t bytes, int heads,
                                cudaStream_t st)
{
    switch (G) {
    case 1: return launch_decode_q4_g<1>(cw, mc, mg, mv, a, bytes, heads, st);
    case 2: return launch_decode_q4_g<2>(cw, mc, mg, mv, a, bytes, heads, st);
    case 4: return launch_decode_q4_g<4>(cw, mc, mg, mv, a, bytes, heads, st);
    case 8: return launch_decode_q4_g<8>(cw, mc, mg, mv, a, bytes, heads, st);
    default: return THINK_ERR_UNSUPPORTED;
    }
}

// --------------------------------------------------------- tcgen05 decode --

struct TcPlan {
    int stages_k, stages_v;
    size_t bytes;
};

// One block per SM: 4 V slots if possible, then as many K' slots (2..6) as
// fit.  THINK_DECODE_STAGES_V / THINK_DECODE_STAGES_K cap the choice (tuning).
TcPlan plan_decode_tc(int T)
{
    TcPlan p;
    const int max_v = env_int("THINK_DECODE_STAGES_V", 4, 2, 6);
    const int max_k = env_int("THINK_DECODE_STAGES_K", 6, 2, 8);
    for (int v = max_v; v >= 2; --v)
        for (int k = max_k; k >= 2; --k) {
            const size_t bytes = tc_layout(T, k, v).total + 1024;
            if (bytes <= kSmemPerBlockMax) {
                p.stages_k = k;
                p.stages_v = v;
                p.bytes = bytes;
                return p;
            }
        }
    p.stages_k = 0;
    p.stages_v = 0;
    p.bytes = 0;
    return p;
}

template <int G>
think_status_t launch_decode_tc_g(const CUtensorMap &mk, const CUtensorMap &mv, const DecodeArgs &a,
                                  size_t bytes, int heads, cudaStream_t st)
{
    auto kern = pruned_decode_tc_kernel<G>;
    if (!ensure_smem(reinterpret_cast<const void *>(kern), bytes))
        return THINK_ERR_CUDA;
    dim3 grid(a.splits, heads);
    kern<<<grid, kTcThreads, bytes, st>>>(mk, mv, a);
    return launch_status();
}

think_status_t launch_decode_tc(int G, const CUtensorMap &mk, const CUtensorMap &mv,
                                const DecodeArgs &a, size_t bytes, int heads, cudaStream_t st)
{
    switch (G) {
    case 1: return launch_decode_tc_g<1>(mk, mv, a, bytes, heads, st);
    case 2: return launch_decode_tc_g<2>(mk, mv, a, bytes, heads, st);
    case 4: return launch_decode_tc_g<4>(mk, mv, a, bytes, heads, st);
    case 8: return launch_decode_tc_g<8>(mk, mv, a, bytes, heads, st);
    default: return THINK_ERR_UNSUPPORTED;
    }
}

}  // namespace
}  // namespace think

// ------------------------------------------------------ decode without allocation --
// Callers that may not allocate device memory (a host framework that owns the
// whole device-memory budget, or a latency-critical path where an allocation,
// which can synchronise the device, is not allowed) use
// think_pruned_decode_attn_noalloc, whose scratch lives in this file-scope
// array.  Every GPU that loads the library holds it until the process exits.
namespace think {
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB
constexpr int kNoAllocMaxDevices = 64;
}  // namespace
}  // namespace think

static __device__ __align__(256) unsigned char g_noalloc_scratch[think::kNoAllocScratchBytes];

namespace think {
namespace {
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kNoAllocMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device, looked up once
// per device (with that device current).  In host code the array's name only
// stands for it; the kernel must be given this address.
cudaError_t noalloc_scratch(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}
}  // namespace
}  // namespace think

namespace think {
namespace {
struct SelectWs {
    int kpt, chunks;
    size_t hist, sel, cnt, total;
};

SelectWs select_ws_layout(int64_t heads, int64_t N)
{
    SelectWs w;
    // keys per thread: a multiple of kSelBatch, at most 1024 chunks per head
    w.kpt = (int)(kSelBatch * std::max<int64_t>(1, ceil_div(N, (int64_t)kSelThreads * 1024 * kSelBatch)));
    w.chunks = (int)std::max<int64_t>(1, ceil_div(N, (int64_t)kSelThreads * w.kpt));
    w.hist = 0;
    w.sel = align_up((size_t)4 * heads * 256 * sizeof(int), 256);
    w.cnt = w.sel + align_up((size_t)heads * 2 * sizeof(int), 256);
    w.total = w.cnt + (size_t)heads * w.chunks * 2 * sizeof(int);
    return w;
}
}  // namespace
}  // namespace think

using namespace think;

extern "C" {

const char *think_status_string(think_status_t s)
{
    switch (s) {
    case THINK_OK: return "THINK_OK";
    case THINK_ERR_INVALID_ARG: return "THINK_ERR_INVALID_ARG: invalid argument";
    case THINK_ERR_UNSUPPORTED: return "THINK_ERR_UNSUPPORTED: shape or dtype not built";
    case THINK_ERR_WORKSPACE: return "THINK_ERR_WORKSPACE: workspace missing or too small";
    case THINK_ERR_CUDA: return "THINK_ERR_CUDA: a CUDA call failed";
    case THINK_ERR_ALIGNMENT: return "THINK_ERR_ALIGNMENT: pointer or stride not 16-byte aligned";
    }
    return "THINK_ERR_UNKNOWN";
}

int think_t_from_lambda(int d, double lambda)
{
    if (d < 1 || !std::isfinite(lambda)) return 0;
    const double t = std::floor((1.0 - lambda) * (double)d + 0.5);
    if (t < 1.0) return 1;
    if (t > (double)d) return d;
    return (int)t;
}

int64_t think_pruned_ld(int64_t N, think_dtype_t dtype)
{
    if (N < 0 || !dtype_ok(dtype)) return -1;
    const int64_t q = (int64_t)(16 / esize(dtype));
    return ceil_div(N, q) * q;
}

size_t think_score_workspace_size(int B, int Hq, int Hkv, int64_t N, int d)
{
    if (B <= 0 || Hkv <= 0 || Hq < Hkv || Hq % Hkv != 0 || N < 0 || d != kD) return 0;
    const int64_t heads = (int64_t)B * Hkv;
    return score_ws_layout_max(heads, Hq / Hkv, N).total;
}

think_status_t think_score_channels(const void *q_win, const void *k, const int64_t k_strides[3],
                                    int B, int Hq, int Hkv, int64_t N, int S_obs, int d,
                                    think_dtype_t dtype, double *scores, void *workspace,
                                    size_t workspace_bytes, void *stream)
{
    const think_status_t v = validate_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, d, dtype,
                                            scores, workspace, workspace_bytes);
    if (v != THINK_OK || B == 0 || Hkv == 0) return v;
    return launch_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, dtype, 0, scores, nullptr,
                        workspace, static_cast<cudaStream_t>(stream));
}

think_status_t think_select_channels(const double *scores, int B, int Hkv, int d, int T,
                                     int32_t *idx, void *stream)
{
    if (B < 0 || Hkv < 0) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (T < 1 || T > d) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (!scores || !idx) return THINK_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(scores) & 7u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return THINK_ERR_ALIGNMENT;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > (int64_t)INT32_MAX / 2) return THINK_ERR_UNSUPPORTED;
    select_kernel<<<(unsigned)ceil_div(heads, 4), 128, 0, static_cast<cudaStream_t>(stream)>>>(
        scores, (int)heads, T, idx);
    return launch_status();
}

think_status_t think_compact_keys(const void *k, const int64_t k_strides[3], int B, int Hkv,
                                  int64_t N, int d, think_dtype_t dtype, const int32_t *idx,
                                  int T, void *k_pruned, int64_t ldk, void *stream)
{
    const think_status_t v = validate_compact(k, k_strides, B, Hkv, N, d, dtype, idx, T, k_pruned, ldk);
    if (v != THINK_OK || B == 0 || Hkv == 0 || N == 0) return v;
    return launch_compact(k, k_strides, B, Hkv, N, dtype, idx, T, k_pruned, ldk,
                          static_cast<cudaStream_t>(stream));
}

think_status_t think_append_keys(const void *k_new, const int64_t k_strides[3], int B, int Hkv,
                                 int64_t n_new, int d, think_dtype_t dtype, const int32_t *idx, int T,
                                 void *k_pruned, int64_t ldk, int64_t n_at, void *stream)
{
    if (n_new < 0 || n_at < 0) return THINK_ERR_INVALID_ARG;
    if (n_new > 0 && n_at > ldk - n_new) return THINK_ERR_INVALID_ARG;  // past the row capacity
    const think_status_t v = validate_compact(k_new, k_strides, B, Hkv, n_new, d, dtype, idx, T,
                                              k_pruned, ldk);
    if (v != THINK_OK || B == 0 || Hkv == 0 || n_new == 0) return v;
    return launch_compact(k_new, k_strides, B, Hkv, n_new, dtype, idx, T, k_pruned, ldk,
                          static_cast<cudaStream_t>(stream), n_at);
}

think_status_t think_prune(const void *q_win, const void *k, const int64_t k_strides[3], int B,
                           int Hq, int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype,
                           int T, double *scores, int32_t *idx, void *k_pruned, int64_t ldk,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    think_status_t v = validate_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, d, dtype, scores,
                                      workspace, workspace_bytes);
    if (v != THINK_OK) return v;
    if (T < 1 || T > d) return THINK_ERR_INVALID_ARG;
    if (B > 0 && Hkv > 0 && (!idx || (reinterpret_cast<uintptr_t>(idx) & 3u)))
        return idx ? THINK_ERR_ALIGNMENT : THINK_ERR_INVALID_ARG;
    v = validate_compact(k, k_strides, B, Hkv, N, d, dtype, idx, T, k_pruned, ldk);
    if (v != THINK_OK || B == 0 || Hkv == 0) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Two launches (score + select, then compact); THINK_PRUNE_FUSED=1 selects
    // for bf16 the one kernel that reads K about once (prune_fused_applies).
    // Both give the same bits.
    if (prune_fused_applies(dtype, (int64_t)B * Hkv, Hq / Hkv, N)) {
        v = launch_prune_fused(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, T, scores, idx, k_pruned,
                               ldk, workspace, st);
        if (v != THINK_ERR_UNSUPPORTED) return v;
    }
    v = launch_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, dtype, T, scores, idx, workspace, st);
    if (v != THINK_OK || N == 0) return v;
    if (dtype == THINK_BF16) {
        v = launch_compact_tma(k, k_strides, B, Hkv, N, idx, T, k_pruned, ldk, workspace, st);
        if (v != THINK_ERR_UNSUPPORTED) return v;
    }
    return launch_compact(k, k_strides, B, Hkv, N, dtype, idx, T, k_pruned, ldk, st);
}

size_t think_decode_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, think_dtype_t dtype)
{
    if (B <= 0 || Hkv <= 0 || Hq < Hkv || Hq % Hkv != 0 || N <= 0 || d != kD || !dtype_ok(dtype))
        return 0;
    const int64_t heads = (int64_t)B * Hkv;
    const int G = Hq / Hkv;
    const DecodeSplit sp = plan_decode_split(heads, N);
    const size_t slots = (size_t)heads * sp.splits * G;
    const size_t pe = dtype == THINK_F32 ? sizeof(double) : sizeof(float);  // fp32 caches: fp64 partials
    return kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256) + slots * kD * pe + slots * 2 * pe;
}

// fp32 caches: the fp64 decode (decode_f64.cuh), grid (splits, heads).
think_status_t launch_decode_f64(const void *q, const void *k_pruned, int64_t ldk, const void *v,
                                 const int64_t v_strides[3], const int32_t *idx, int B, int Hq, int Hkv,
                                 int64_t N, int T, float scale, float *out, void *workspace, cudaStream_t st)
{
    const int64_t heads = (int64_t)B * Hkv;
    const int G = Hq / Hkv;
    const DecodeSplit sp = plan_decode_split(heads, N);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t slots = (size_t)heads * sp.splits * G;
    DecodeF64Args a;
    a.q = static_cast<const float *>(q);
    a.kp = static_cast<const float *>(k_pruned);
    a.v = static_cast<const float *>(v);
    a.sb = v_strides[0];
    a.sh = v_strides[1];
    a.sn = v_strides[2];
    a.idx = idx;
    a.out = out;
    a.tickets = reinterpret_cast<unsigned *>(ws + kDecodeHeader);
    if (ready_counters(ws, kDecodeHeader, kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256),
                       st) != THINK_OK)
        return THINK_ERR_CUDA;
    a.part_o = reinterpret_cast<double *>(ws + kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256));
    a.part_ml = a.part_o + slots * kD;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.T = T;
    a.splits = sp.splits;
    a.tiles_per_split = sp.tiles_per_split;
    a.N = N;
    a.ldk = ldk;
    a.scale = (double)scale;
    const dim3 grid((unsigned)sp.splits, (unsigned)heads);
    switch (G) {
    case 1: pruned_decode_f64_kernel<1><<<grid, 256, 0, st>>>(a); break;
    case 2: pruned_decode_f64_kernel<2><<<grid, 256, 0, st>>>(a); break;
    case 4: pruned_decode_f64_kernel<4><<<grid, 256, 0, st>>>(a); break;
    default: pruned_decode_f64_kernel<8><<<grid, 256, 0, st>>>(a); break;
    }
    return launch_status();
}

think_status_t think_pruned_decode_attn(const void *q, const void *k_pruned, int64_t ldk,
                                        const void *v, const int64_t v_strides[3],
                                        const int32_t *idx, int B, int Hq, int Hkv, int64_t N,
                                        int d, int T, think_dtype_t dtype, float scale, float *out,
                                        void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0) return THINK_ERR_INVALID_ARG;
    if (!dtype_ok(dtype) || !std::isfinite(scale)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (T < 1 || T > d) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (Hq < Hkv || Hq % Hkv != 0) return THINK_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return THINK_ERR_UNSUPPORTED;
    if (N == 0 || ldk < N) return THINK_ERR_INVALID_ARG;
    if (!q || !k_pruned || !v || !v_strides || !idx || !out || !workspace)
        return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535 || N > (int64_t)INT32_MAX - kBN) return THINK_ERR_UNSUPPORTED;
    const size_t es = esize(dtype);
    if (!aligned16(q) || !aligned16(k_pruned) || !aligned16(v) || !aligned16(workspace) ||
        !aligned16(out) || !strides_ok(v_strides, es) || (ldk * (int64_t)es) % 16 != 0 ||
        (reinterpret_cast<uintptr_t>(idx) & 3u))
        return THINK_ERR_ALIGNMENT;
    const size_t need = think_decode_workspace_size(B, Hq, Hkv, N, d, dtype);
    if (workspace_bytes < need) return THINK_ERR_WORKSPACE;
    if (dtype == THINK_F32)
        return launch_decode_f64(q, k_pruned, ldk, v, v_strides, idx, B, Hq, Hkv, N, T, scale, out, workspace,
                                 static_cast<cudaStream_t>(stream));

    // bf16: warp-level tensor-core kernel (mma.sync) by default;
    // THINK_DECODE_TENSOR_CORES=1 selects the tcgen05 kernel and
    // THINK_DECODE_CUDA_CORES=1 the CUDA-core kernel (same results within
    // tolerance; for comparisons).  fp32 inputs use the fp64 decode above.
    enum { kSimt, kMma, kTc } kind = kSimt;
    if (dtype == THINK_BF16) {
        kind = kMma;
        if (env_flag("THINK_DECODE_TENSOR_CORES")) kind = kTc;
        else if (env_flag("THINK_DECODE_CUDA_CORES")) kind = kSimt;
    }
    const bool use_tc = kind == kTc;
    const TcPlan tp = plan_decode_tc(T);
    const MmaPlan mp = plan_decode_mma(T, G, heads, N);
    const DecodeSmem sm = plan_decode_smem(T, G, es);
    if (kind == kTc ? tp.stages_k == 0 : kind == kMma ? mp.stages == 0 : sm.bytes > kSmemPerBlockMax)
        return THINK_ERR_UNSUPPORTED;
    const int bps = kind == kTc ? kTcBlocksPerSM : kind == kMma ? mp.blocks_per_sm : kDecodeBlocksPerSM;
    const DecodeSplit sp = plan_decode_split(heads, N, bps);
    CUtensorMap mk, mv;
    if (kind != kSimt) {
        // K'^T in 64-token halves, V in 64-channel halves, 128-byte swizzle (the
        // tensor core's MN-major canonical layout)
        if (!make_map_4d(&mk, dtype, k_pruned, (uint64_t)N, (uint64_t)T, (uint64_t)Hkv, (uint64_t)B,
                         ldk, (int64_t)T * ldk, (int64_t)Hkv * T * ldk, 64, (uint32_t)T, true))
            return THINK_ERR_CUDA;
        if (!make_map_4d(&mv, dtype, v, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, v_strides[2],
                         v_strides[1], v_strides[0], 64, kBN, true))
            return THINK_ERR_CUDA;
    } else {
        // K'^T: x = token (pitch ldk), y = kept channel, z = KV head, w = batch
        if (!make_map_4d(&mk, dtype, k_pruned, (uint64_t)N, (uint64_t)T, (uint64_t)Hkv, (uint64_t)B,
                         ldk, (int64_t)T * ldk, (int64_t)Hkv * T * ldk, kBN, (uint32_t)T))
            return THINK_ERR_CUDA;
        // V: x = channel, y = token, z = KV head, w = batch
        if (!make_map_4d(&mv, dtype, v, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, v_strides[2],
                         v_strides[1], v_strides[0], kD, kBN))
            return THINK_ERR_CUDA;
    }

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t slots = (size_t)heads * sp.splits * G;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));  // Th = rowoff = null: one kept width for every head
    a.q = q;
    a.idx = idx;
    a.status = reinterpret_cast<unsigned *>(ws);
    a.tickets = reinterpret_cast<unsigned *>(ws + kDecodeHeader);
    if (ready_counters(ws, kDecodeHeader, kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256),
                       static_cast<cudaStream_t>(stream)) != THINK_OK)
        return THINK_ERR_CUDA;
    a.part_o = reinterpret_cast<float *>(ws + kDecodeHeader +
                                         align_up((size_t)heads * sizeof(unsigned), 256));
    a.out = out;
    a.part_ml = a.part_o + slots * kD;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.T = T;
    a.N = N;
    a.tiles_per_split = sp.tiles_per_split;
    a.splits = sp.splits;
    a.stages = use_tc ? tp.stages_k : kind == kMma ? mp.stages : sm.stages;
    a.stages_v = use_tc ? tp.stages_v : 0;
    a.prefetch = env_int("THINK_DECODE_PREFETCH", kDecodePrefetchTiles, 0, 64);
    a.early = env_int("THINK_DECODE_EARLY_PREFETCH", 1, 0, 1);
    a.staged_merge = env_int("THINK_DECODE_STAGED_MERGE", 1, 0, 1);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.stage_bytes = sm.stage_bytes;
    a.v_off = sm.v_off;
    a.tx_bytes = sm.tx_bytes;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (use_tc) return launch_decode_tc(G, mk, mv, a, tp.bytes, (int)heads, st);
    if (kind == kMma) return launch_decode_mma(G, mp.warps, mk, mv, a, mp.bytes, (int)heads, st);
    return launch_decode<__nv_bfloat16>(G, mk, mv, a, sm, (int)heads, st);
}

int64_t think_q4_ld(int64_t N)
{
    if (N < 0) return -1;
    return ceil_div(N, kQ4Group) * 64;
}

size_t think_q4_groups_bytes(int B, int Hkv, int64_t N, int T)
{
    if (B < 0 || Hkv < 0 || N < 0 || T < 1) return 0;
    return (size_t)B * Hkv * (size_t)ceil_div(N, kQ4Group) * (size_t)((T + 1) & ~1) * 2 * sizeof(float);
}

think_status_t think_quantize_keys_q4(const void *k_pruned, int64_t ldk, int B, int Hkv, int64_t N, int T,
                                      uint8_t *codes, int64_t ldq, float *groups, void *stream)
{
    if (B < 0 || Hkv < 0 || N < 0 || T < 1 || T > kD || ldk < N) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0 || N == 0) return THINK_OK;
    if (!k_pruned || !codes || !groups) return THINK_ERR_INVALID_ARG;
    if (ldq < think_q4_ld(N) || ldq % 64 != 0) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535 || ceil_div(N, kQ4Group) > INT32_MAX) return THINK_ERR_UNSUPPORTED;
    if (!aligned16(k_pruned) || !aligned16(codes) || !aligned16(groups) || (ldk * 2) % 16 != 0)
        return THINK_ERR_ALIGNMENT;
    dim3 grid((unsigned)ceil_div(N, kQ4Group), (unsigned)heads);
    quantize_q4_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(k_pruned), ldk, T, N, codes, ldq, reinterpret_cast<float2 *>(groups));
    return launch_status();
}

think_status_t think_pruned_decode_attn_q4(const void *q, const uint8_t *codes, int64_t ldq,
                                           const float *groups, const void *v, const int64_t v_strides[3],
                                           const int32_t *idx, int B, int Hq, int Hkv, int64_t N, int d, int T,
                                           float scale, float *out, void *workspace, size_t workspace_bytes,
                                           void *stream)
{
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0 || !std::isfinite(scale)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (T < 1 || T > d) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (Hq < Hkv || Hq % Hkv != 0) return THINK_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return THINK_ERR_UNSUPPORTED;
    if (N == 0 || ldq < think_q4_ld(N) || ldq % 64 != 0) return THINK_ERR_INVALID_ARG;
    if (!q || !codes || !groups || !v || !v_strides || !idx || !out || !workspace)
        return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535 || N > (int64_t)INT32_MAX - kBN) return THINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(codes) || !aligned16(groups) || !aligned16(v) || !aligned16(workspace) ||
        !aligned16(out) || !strides_ok(v_strides, 2) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return THINK_ERR_ALIGNMENT;
    if (workspace_bytes < think_decode_workspace_size(B, Hq, Hkv, N, d, THINK_BF16)) return THINK_ERR_WORKSPACE;

    const MmaPlan mp = plan_decode_q4(T, G, heads, N);
    if (mp.stages == 0) return THINK_ERR_UNSUPPORTED;
    const DecodeSplit sp = plan_decode_split(heads, N, mp.blocks_per_sm);
    const int64_t ng = ldq / 64;
    const uint64_t T2 = (uint64_t)((T + 1) & ~1);
    CUtensorMap mc, mg, mv;
    // codes: x = byte (two tokens), y = kept channel, z = KV head, w = batch; box 64 B x T
    if (!make_map_raw_4d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, (uint64_t)ldq, (uint64_t)T, (uint64_t)Hkv,
                         (uint64_t)B, (uint64_t)ldq, (uint64_t)T * ldq, (uint64_t)Hkv * T * ldq, 64,
                         (uint32_t)T))
        return THINK_ERR_CUDA;
    // group parameters: x = (scale, mn) of the T2 rows, y = group, z = KV head, w = batch
    if (!make_map_raw_4d(&mg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, groups, 2 * T2, (uint64_t)ng, (uint64_t)Hkv,
                         (uint64_t)B, 2 * T2 * 4, (uint64_t)ng * 2 * T2 * 4, (uint64_t)Hkv * ng * 2 * T2 * 4,
                         (uint32_t)(2 * T2), 1))
        return THINK_ERR_CUDA;
    if (!make_map_4d(&mv, THINK_BF16, v, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, v_strides[2],
                     v_strides[1], v_strides[0], 64, kBN, true))
        return THINK_ERR_CUDA;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t slots = (size_t)heads * sp.splits * G;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q;
    a.idx = idx;
    a.status = reinterpret_cast<unsigned *>(ws);
    a.tickets = reinterpret_cast<unsigned *>(ws + kDecodeHeader);
    if (ready_counters(ws, kDecodeHeader, kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256),
                       static_cast<cudaStream_t>(stream)) != THINK_OK)
        return THINK_ERR_CUDA;
    a.part_o = reinterpret_cast<float *>(ws + kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256));
    a.out = out;
    a.part_ml = a.part_o + slots * kD;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.T = T;
    a.N = N;
    a.tiles_per_split = sp.tiles_per_split;
    a.splits = sp.splits;
    a.stages = mp.stages;
    a.early = env_int("THINK_DECODE_EARLY_PREFETCH", 1, 0, 1);
    a.staged_merge = env_int("THINK_DECODE_STAGED_MERGE", 1, 0, 1);
    a.scale_log2 = scale * 1.4426950408889634f;
    return launch_decode_q4(G, mp.warps, mc, mg, mv, a, mp.bytes, (int)heads, static_cast<cudaStream_t>(stream));
}

int64_t think_ragged_rows(int B, int Hkv, int T_max)
{
    if (B < 0 || Hkv < 0 || T_max < 1 || T_max > kD) return -1;
    return (int64_t)B * Hkv * ((T_max + 15) & ~15);
}

think_status_t think_select_adaptive(const double *scores, int B, int Hkv, int d, double tau, int T_min,
                                     int T_max, int32_t *Th, int32_t *rowoff, int32_t *idx, void *stream)
{
    if (B < 0 || Hkv < 0) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (!(tau >= 0.0 && tau <= 1.0) || T_min < 1 || T_max < T_min || T_max > d) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (!scores || !Th || !rowoff || !idx) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535) return THINK_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(scores) & 7u) || (reinterpret_cast<uintptr_t>(Th) & 3u) ||
        (reinterpret_cast<uintptr_t>(rowoff) & 3u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return THINK_ERR_ALIGNMENT;
    select_adaptive_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(scores, (int)heads, tau, T_min,
                                                                             T_max, Th, rowoff, idx);
    return launch_status();
}

think_status_t think_compact_keys_ragged(const void *k, const int64_t k_strides[3], int B, int Hkv, int64_t N,
                                         int d, think_dtype_t dtype, const int32_t *idx, const int32_t *Th,
                                         const int32_t *rowoff, int T_max, void *k_pruned, int64_t ldk,
                                         void *stream)
{
    think_status_t v = validate_compact(k, k_strides, B, Hkv, N, d, dtype, idx, T_max, k_pruned, ldk);
    if (v != THINK_OK || B == 0 || Hkv == 0 || N == 0) return v;
    if (!Th || !rowoff) return THINK_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Th) & 3u) || (reinterpret_cast<uintptr_t>(rowoff) & 3u))
        return THINK_ERR_ALIGNMENT;
    return launch_compact(k, k_strides, B, Hkv, N, dtype, idx, T_max, k_pruned, ldk,
                          static_cast<cudaStream_t>(stream), 0, Th, rowoff);
}

think_status_t think_prune_adaptive(const void *q_win, const void *k, const int64_t k_strides[3], int B, int Hq,
                                    int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype, double tau,
                                    int T_min, int T_max, double *scores, int32_t *Th, int32_t *rowoff,
                                    int32_t *idx, void *k_pruned, int64_t ldk, void *workspace,
                                    size_t workspace_bytes, void *stream)
{
    think_status_t v = validate_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, d, dtype, scores, workspace,
                                      workspace_bytes);
    if (v != THINK_OK) return v;
    if (!(tau >= 0.0 && tau <= 1.0) || T_min < 1 || T_max < T_min || T_max > d) return THINK_ERR_INVALID_ARG;
    v = validate_compact(k, k_strides, B, Hkv, N, d, dtype, idx, T_max, k_pruned, ldk);
    if (v != THINK_OK || B == 0 || Hkv == 0) return v;
    if (!Th || !rowoff) return THINK_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Th) & 3u) || (reinterpret_cast<uintptr_t>(rowoff) & 3u))
        return THINK_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t heads = (int64_t)B * Hkv;
    v = launch_score(q_win, k, k_strides, B, Hq, Hkv, N, S_obs, dtype, 0, scores, nullptr, workspace, st);
    if (v != THINK_OK) return v;
    select_adaptive_kernel<<<1, 1024, 0, st>>>(scores, (int)heads, tau, T_min, T_max, Th, rowoff, idx);
    v = launch_status();
    if (v != THINK_OK || N == 0) return v;
    if (dtype == THINK_BF16) {
        v = launch_compact_tma(k, k_strides, B, Hkv, N, idx, T_max, k_pruned, ldk, workspace, st, Th, rowoff);
        if (v != THINK_ERR_UNSUPPORTED) return v;
    }
    return launch_compact(k, k_strides, B, Hkv, N, dtype, idx, T_max, k_pruned, ldk, st, 0, Th, rowoff);
}

think_status_t think_pruned_decode_attn_ragged(const void *q, const void *k_pruned, int64_t ldk, const void *v,
                                               const int64_t v_strides[3], const int32_t *idx,
                                               const int32_t *Th, const int32_t *rowoff, int T_max, int B, int Hq,
                                               int Hkv, int64_t N, int d, float scale, float *out,
                                               void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0 || !std::isfinite(scale)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (T_max < 1 || T_max > d) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (Hq < Hkv || Hq % Hkv != 0) return THINK_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return THINK_ERR_UNSUPPORTED;
    if (N == 0 || ldk < N) return THINK_ERR_INVALID_ARG;
    if (!q || !k_pruned || !v || !v_strides || !idx || !Th || !rowoff || !out || !workspace)
        return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535 || N > (int64_t)INT32_MAX - kBN) return THINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_pruned) || !aligned16(v) || !aligned16(workspace) || !aligned16(out) ||
        !strides_ok(v_strides, 2) || (ldk * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(Th) & 3u) || (reinterpret_cast<uintptr_t>(rowoff) & 3u))
        return THINK_ERR_ALIGNMENT;
    if (workspace_bytes < think_decode_workspace_size(B, Hq, Hkv, N, d, THINK_BF16)) return THINK_ERR_WORKSPACE;
    const MmaPlan mp = plan_decode_mma(T_max, G, heads, N);
    if (mp.stages == 0) return THINK_ERR_UNSUPPORTED;
    const DecodeSplit sp = plan_decode_split(heads, N, mp.blocks_per_sm);
    const int64_t rows = think_ragged_rows(B, Hkv, T_max);
    CUtensorMap mk, mv;
    // K' rows of every head in one 2-D range (x = token, y = row), 16-row boxes
    if (!make_map_4d(&mk, THINK_BF16, k_pruned, (uint64_t)N, (uint64_t)rows, 1, 1, ldk, rows * ldk, rows * ldk, 64,
                     16, true))
        return THINK_ERR_CUDA;
    if (!make_map_4d(&mv, THINK_BF16, v, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, v_strides[2], v_strides[1],
                     v_strides[0], 64, kBN, true))
        return THINK_ERR_CUDA;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t slots = (size_t)heads * sp.splits * G;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q;
    a.idx = idx;
    a.status = reinterpret_cast<unsigned *>(ws);
    a.tickets = reinterpret_cast<unsigned *>(ws + kDecodeHeader);
    if (ready_counters(ws, kDecodeHeader, kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256),
                       static_cast<cudaStream_t>(stream)) != THINK_OK)
        return THINK_ERR_CUDA;
    a.part_o = reinterpret_cast<float *>(ws + kDecodeHeader + align_up((size_t)heads * sizeof(unsigned), 256));
    a.out = out;
    a.part_ml = a.part_o + slots * kD;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.T = T_max;
    a.N = N;
    a.tiles_per_split = sp.tiles_per_split;
    a.splits = sp.splits;
    a.stages = mp.stages;
    a.early = env_int("THINK_DECODE_EARLY_PREFETCH", 1, 0, 1);
    a.staged_merge = env_int("THINK_DECODE_STAGED_MERGE", 1, 0, 1);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.Th = Th;
    a.rowoff = rowoff;
    return launch_decode_mma(G, mp.warps, mk, mv, a, mp.bytes, (int)heads, static_cast<cudaStream_t>(stream));
}

size_t think_token_mass_workspace_size(int B, int Hq, int Hkv, int64_t N, int S_obs)
{
    if (B < 0 || Hkv < 1 || Hq < Hkv || Hq % Hkv || N < 1 || S_obs < 1) return 0;
    const int64_t heads = (int64_t)B * Hkv;
    const int R = (Hq / Hkv) * S_obs;
    const MassPlan p = plan_mass(R, heads, N);
    return mass_ws_layout(heads, R, p.sp.splits).total;
}

think_status_t think_token_mass(const void *q_win, const void *k, const int64_t k_strides[3], int B, int Hq,
                                int Hkv, int64_t N, int S_obs, int d, think_dtype_t dtype, float scale, float *mass,
                                void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0 || S_obs < 0 || !std::isfinite(scale)) return THINK_ERR_INVALID_ARG;
    if (d != kD || dtype != THINK_BF16) return THINK_ERR_UNSUPPORTED;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (Hq < Hkv || Hq % Hkv != 0 || N < 1 || S_obs < 1) return THINK_ERR_INVALID_ARG;
    const int R = (Hq / Hkv) * S_obs;
    if (R > kMassRowsMax) return THINK_ERR_UNSUPPORTED;
    if (!q_win || !k || !k_strides || !mass || !workspace) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535 || N > (int64_t)INT32_MAX - kBN) return THINK_ERR_UNSUPPORTED;
    if (!aligned16(q_win) || !aligned16(k) || !aligned16(workspace) || !strides_ok(k_strides, 2) ||
        (reinterpret_cast<uintptr_t>(mass) & 3u))
        return THINK_ERR_ALIGNMENT;
    const MassPlan p = plan_mass(R, heads, N);
    if (p.stages == 0) return THINK_ERR_UNSUPPORTED;
    if (workspace_bytes < mass_ws_layout(heads, R, p.sp.splits).total) return THINK_ERR_WORKSPACE;
    // tcgen05 kernels when they apply (their one block per SM never needs more
    // splits, so the workspace sized for plan_mass holds their partials)
    const MassTcPlan tp = plan_mass_tc(R, heads, N);
    const bool use_tc = tp.stages > 0;
    const DecodeSplit sp = use_tc ? tp.sp : p.sp;
    const MassWs w = mass_ws_layout(heads, R, sp.splits);
    if (workspace_bytes < w.total) return THINK_ERR_WORKSPACE;
    CUtensorMap mk;
    // K as V is read by the decode: x = channel (two 64-channel halves), y = token
    if (!make_map_4d(&mk, THINK_BF16, k, kD, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B, k_strides[2], k_strides[1],
                     k_strides[0], 64, kBN, true))
        return THINK_ERR_CUDA;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    MassArgs a;
    a.qwin = static_cast<const __nv_bfloat16 *>(q_win);
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.S = S_obs;
    a.G = Hq / Hkv;
    a.R = R;
    a.r_pad = p.r_pad;
    a.N = N;
    a.tiles_per_split = sp.tiles_per_split;
    a.splits = sp.splits;
    a.stages = use_tc ? tp.stages : p.stages;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part = reinterpret_cast<float2 *>(ws + w.part);
    a.stats = reinterpret_cast<float2 *>(ws + w.stats);
    a.tickets = reinterpret_cast<unsigned *>(ws + w.tickets);
    a.status = reinterpret_cast<unsigned *>(ws);
    a.mass = mass;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (ready_counters(ws, w.tickets, w.part, st) != THINK_OK) return THINK_ERR_CUDA;
    if (use_tc)
        return tp.mb == 1 ? launch_mass_tc<1>(mk, a, tp.bytes, (int)heads, st)
                          : launch_mass_tc<2>(mk, a, tp.bytes, (int)heads, st);
    switch (p.ntw) {
    case 1: return launch_mass<1>(mk, a, p, (int)heads, st);
    case 2: return launch_mass<2>(mk, a, p, (int)heads, st);
    case 4: return launch_mass<4>(mk, a, p, (int)heads, st);
    default: return launch_mass<8>(mk, a, p, (int)heads, st);
    }
}

size_t think_select_tokens_workspace_size(int B, int Hkv, int64_t N)
{
    if (B <= 0 || Hkv <= 0 || N <= 0 || N > (int64_t)INT32_MAX) return 0;
    return select_ws_layout((int64_t)B * Hkv, N).total;
}

think_status_t think_select_tokens(const float *mass, int B, int Hkv, int64_t N, int M, int32_t *kept,
                                   void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || Hkv < 0 || N < 0) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    if (M < 1 || M > N || N > (int64_t)INT32_MAX) return THINK_ERR_INVALID_ARG;
    if (!mass || !kept || !workspace) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535) return THINK_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(mass) & 3u) || (reinterpret_cast<uintptr_t>(kept) & 3u) ||
        !aligned16(workspace))
        return THINK_ERR_ALIGNMENT;
    const SelectWs w = select_ws_layout(heads, N);
    if (workspace_bytes < w.total) return THINK_ERR_WORKSPACE;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    SelectArgs a;
    a.mass = mass;
    a.N = N;
    a.M = M;
    a.kpt = w.kpt;
    a.chunks = w.chunks;
    a.hist = reinterpret_cast<int *>(ws + w.hist);
    a.sel = reinterpret_cast<int *>(ws + w.sel);
    a.cnt = reinterpret_cast<int *>(ws + w.cnt);
    a.kept = kept;
    a.heads = (int)heads;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (ready_counters(ws, w.hist, w.sel, st) != THINK_OK) return THINK_ERR_CUDA;
    const dim3 grid((unsigned)w.chunks, (unsigned)heads);
    select_hist_kernel<0><<<grid, kSelThreads, 0, st>>>(a);
    select_hist_kernel<1><<<grid, kSelThreads, 0, st>>>(a);
    select_hist_kernel<2><<<grid, kSelThreads, 0, st>>>(a);
    select_hist_kernel<3><<<grid, kSelThreads, 0, st>>>(a);
    select_count_kernel<<<grid, kSelThreads, 0, st>>>(a);
    select_write_kernel<<<grid, kSelThreads, 0, st>>>(a);
    return launch_status();
}

think_status_t think_gather_tokens(const void *x, const int64_t x_strides[3], int B, int Hkv, int64_t N, int d,
                                   think_dtype_t dtype, const int32_t *kept, int M, void *out, void *stream)
{
    if (B < 0 || Hkv < 0 || N < 0 || M < 0 || !dtype_ok(dtype)) return THINK_ERR_INVALID_ARG;
    if (d != kD) return THINK_ERR_UNSUPPORTED;
    if (B == 0 || Hkv == 0 || M == 0) return THINK_OK;
    if (!x || !x_strides || !kept || !out) return THINK_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)B * Hkv;
    if (heads > 65535) return THINK_ERR_UNSUPPORTED;
    const size_t es = esize(dtype);
    if (!aligned16(x) || !aligned16(out) || !strides_ok(x_strides, es) || (reinterpret_cast<uintptr_t>(kept) & 3u))
        return THINK_ERR_ALIGNMENT;
    const int rows_per_block = 256 / (kD / (int)(16 / es));
    dim3 grid((unsigned)ceil_div(M, rows_per_block), (unsigned)heads);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == THINK_BF16)
        gather_tokens_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(x), x_strides[0], x_strides[1], x_strides[2], Hkv, M, kept, N,
            static_cast<__nv_bfloat16 *>(out));
    else
        gather_tokens_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(x), x_strides[0],
                                                          x_strides[1], x_strides[2], Hkv, M, kept, N,
                                                          static_cast<float *>(out));
    return launch_status();
}

think_status_t think_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace) return THINK_ERR_INVALID_ARG;
    if (workspace_bytes == 0) return THINK_OK;
    forget_counters(workspace);
    return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? THINK_OK
               : THINK_ERR_CUDA;
}

think_status_t think_read_device_status(const void *workspace, uint32_t *status, void *stream)
{
    if (!workspace || !status) return THINK_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
        return THINK_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? THINK_OK : THINK_ERR_CUDA;
}

size_t think_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

think_status_t think_pruned_decode_attn_noalloc(const void *q, const void *k_pruned, int64_t ldk,
                                                const void *v, const int64_t v_strides[3],
                                                const int32_t *idx, int B, int Hq, int Hkv,
                                                int64_t N, int d, int T, think_dtype_t dtype,
                                                float scale, float *out, void *stream)
{
    // Same validation as the workspace form; the problem must fit the array.
    if (B < 0 || Hq < 0 || Hkv < 0 || N < 0) return THINK_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0) return THINK_OK;
    const size_t need = think_decode_workspace_size(B, Hq, Hkv, N, d, dtype);
    if (need > kNoAllocScratchBytes) return THINK_ERR_WORKSPACE;
    if (need == 0)  // shape rejected by the sizing rules: let the full check name the reason
        return think_pruned_decode_attn(q, k_pruned, ldk, v, v_strides, idx, B, Hq, Hkv, N, d, T,
                                        dtype, scale, out, nullptr, 0, stream);
    void *ws = nullptr;
    if (noalloc_scratch(&ws) != cudaSuccess) return THINK_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word and the per-head arrival counters must start at zero
    const size_t zero = kDecodeHeader + align_up((size_t)B * Hkv * sizeof(unsigned), 256);
    if (cudaMemsetAsync(ws, 0, zero, st) != cudaSuccess) return THINK_ERR_CUDA;
    return think_pruned_decode_attn(q, k_pruned, ldk, v, v_strides, idx, B, Hq, Hkv, N, d, T, dtype,
                                    scale, out, ws, kNoAllocScratchBytes, stream);
}

think_status_t think_noalloc_read_device_status(uint32_t *status, void *stream)
{
    if (!status) return THINK_ERR_INVALID_ARG;
    void *ws = nullptr;
    if (noalloc_scratch(&ws) != cudaSuccess) return THINK_ERR_CUDA;
    return think_read_device_status(ws, status, stream);  // the status word is the array's first word
}

}  // extern "C"

"""Benchmark of the ThinK decode-time path on B200.

One step = one pass of the whole path over one layer of the long-context
workload (Mistral-7B-shaped GQA layer: B=1, 32 query / 8 KV heads, d=128,
N=131072, S_obs=64, lambda=0.6 -> T=51): score the key channels, select the
top T per KV head, compact K, then 256 decode steps of pruned-K attention, each
with a fresh query. Inputs are resident in HBM before the timed region and are
larger than L2 (K 268 MB; K'+V 375 MB read per decode step).

value = algorithmic bytes of the step (one read of K + K' written + Q_win +
idx, plus 256 x (K' + V + q + out + idx)) / device time of the step, in GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica on its own data: the path has no exchange step, so there is no
collective on the data path; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "pruned-K decode attention HBM GB/s (% of 8 TB/s); prune pass µs/layer"
WORKLOAD = "mistral_7b_long"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# default bf16 decode kernel, pruned_decode_mma_kernel<4, 4>, on the long-context
# workload: the capture of the 101st launch in a step's back-to-back loop with
# ncu's cache control off (profiles/pruned_decode_mma_kernel_mistral7b_long.md,
# "In the back-to-back loop"); reported only for that workload and to be reset
# to None whenever the kernel changes.
DECODE_TRAFFIC_BYTES = 375_471_360 + 9_629_696


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--e2e-steps", type=int, default=30)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the measurements outside the step (append, 4-bit and adaptive-width decode)")
    p.add_argument("--workload", default=WORKLOAD,
                   help="workload name from workloads.py (default: the "
                        "long-context layer the metric is quoted on)")
    p.add_argument("--hot", action="store_true",
                   help="one resident copy of the layer, so a layer that fits in L2 is read from L2 "
                        "(the default cycles through copies that together exceed L2 twice)")
    p.add_argument("--batch", type=int, default=None, help="override the workload's B")
    p.add_argument("--lam", type=float, default=None, help="override the workload's lambda")
    p.add_argument("--decode-steps", type=int, default=None,
                   help="override the workload's decode steps per bench step")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------ clocks ---

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: clocks stay unreported
            self.nv, self.error = None, repr(e)

    def _handle(self, idx):
        import torch
        nv = self.nv
        try:
            pr = torch.cuda.get_device_properties(idx)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.error = repr(e)
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": self.error or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------- multi-rank ---

def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_gbs(world: int, bytes_per_rank_step: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank moves bytes_per_rank_step per step."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ----------------------------------------------------------- workload ---

def workload(args):
    import workloads as W
    w = W.WORKLOADS[args.workload]
    kw = {}
    if args.batch is not None:
        kw["B"] = args.batch
    if args.lam is not None:
        kw["lam"] = args.lam
    if args.decode_steps is not None:
        kw["decode_steps"] = args.decode_steps
    return w.with_(**kw) if kw else w


def default_workload(args):
    return (args.workload == WORKLOAD and args.batch is None and args.lam is None
            and args.decode_steps is None)


L2_BYTES = 126 * 1000 * 1000


def resident_layers(w, T):
    """How many layers' buffers a step cycles through: all layers of a
    multi-layer workload, else enough copies of the one layer that a pass over
    them reads at least twice the L2 capacity (so no step finds its K, K' or V
    in L2 from the previous one)."""
    if w.layers > 1:
        return w.layers
    e = torch_elem_size(w.dtype)
    heads = w.B * w.Hkv
    footprint = heads * w.N * (2 * w.d + T) * e        # K + V + K'
    return max(1, -(-2 * L2_BYTES // footprint))


def torch_elem_size(dtype):
    import torch
    return torch.empty((), dtype=dtype).element_size()


def step_bytes(w, T):
    import workloads as W
    return W.prune_bytes(w, T) + w.decode_steps * W.decode_bytes(w, T)


def measure_read_probe(dev, stream, gib=4, reps=10):
    """Context for the decode's fraction of the copy peak: the read bandwidth
    of a plain read-only stream (torch's max reduction, a library kernel, over
    a buffer larger than L2), next to the driver's read+write copy peak."""
    import torch
    buf = torch.ones((gib << 30) // 4, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            torch.amax(buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            torch.amax(buf)
        e1.record(stream)
    stream.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = buf.numel() * 4
    del buf
    return {"gbs": nbytes / (us * 1e-6) / 1e9, "bytes": nbytes,
            "kernel": "torch.amax over a 4 GiB int32 buffer (read-only stream, library kernel; context only)"}


def measure_append(w, T, dev, stream, qw_d, k_d, chunk=4096, reps=50):
    """Growing cache, outside the timed step: device time of appending one new
    token's keys (all heads) and a chunk of new tokens' keys to a pruned cache
    with room for them (the new keys are views of cached ones)."""
    import torch
    import query_driven_key_b200 as qdk
    chunk = min(chunk, w.N)
    cache = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, T, w.d, dtype=w.dtype, device=dev,
                            capacity=w.N + chunk)
    cache.prune(qw_d, k_d, stream=stream)

    def timed(n_new):
        knew = k_d[:, :, :n_new]
        for _ in range(3):
            qdk.think_append_keys(knew, cache.idx, cache.k_pruned, cache.ldk, w.N, stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            qdk.think_append_keys(knew, cache.idx, cache.k_pruned, cache.ldk, w.N, stream)
        e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) * 1e3 / reps

    e = torch_elem_size(w.dtype)
    one_us, chunk_us = timed(1), timed(chunk)
    chunk_bytes = w.B * w.Hkv * chunk * (w.d + T) * e + w.B * w.Hkv * T * 4
    return {"one_token_us": one_us, "chunk_tokens": chunk, "chunk_us": chunk_us,
            "chunk_gbs": chunk_bytes / (chunk_us * 1e-6) / 1e9,
            "note": "think_append_keys, device time per call (CUDA events), not part of the step"}


def measure_q4(w, T, stream, cache, qs_d, v_d, outs, bf16_us, peak):
    """The 4-bit thinner cache on the same layer, outside the timed step:
    device time of quantising K' and of the step's decode calls over the codes."""
    import torch
    import workloads as W
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        cache.quantize_q4(stream)
    e0, e1 = ev(), ev()
    e0.record(stream)
    cache.quantize_q4(stream)
    e1.record(stream)
    for s in range(3):
        cache.decode_q4(qs_d[s], v_d, outs[s], stream=stream)
    e2, e3 = ev(), ev()
    e2.record(stream)
    for s in range(w.decode_steps):
        cache.decode_q4(qs_d[s], v_d, outs[s], stream=stream)
    e3.record(stream)
    stream.synchronize()
    us = e2.elapsed_time(e3) * 1e3 / w.decode_steps
    nbytes = W.decode_bytes_q4(w, T)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"decode_us_per_step": us, "decode_gbs": gbs, "frac_of_measured_peak": gbs / peak,
            "algorithmic_bytes_per_launch": nbytes, "speedup_vs_bf16_decode": bf16_us / us,
            "quantize_us": e0.elapsed_time(e1) * 1e3,
            "kernel": "pruned_decode_q4_kernel (think_pruned_decode_attn_q4), not part of the step"}


def measure_adaptive(w, dev, stream, qw_d, k_d, qs_d, v_d, outs, peak, tau=0.9, T_min=8, T_max=128):
    """A kept width per head on the same layer, outside the timed step: prune
    with the adaptive rule, then the step's decode calls over the ragged cache."""
    import torch
    import query_driven_key_b200 as qdk
    cache = qdk.AdaptiveCache(w.B, w.Hq, w.Hkv, w.N, tau, T_min, T_max, w.d, dtype=w.dtype, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        cache.prune(qw_d, k_d, stream=stream)
    e0, e1 = ev(), ev()
    e0.record(stream)
    cache.prune(qw_d, k_d, stream=stream)
    e1.record(stream)
    for s in range(3):
        cache.decode(qs_d[s], v_d, outs[s], stream=stream)
    e2, e3 = ev(), ev()
    e2.record(stream)
    for s in range(w.decode_steps):
        cache.decode(qs_d[s], v_d, outs[s], stream=stream)
    e3.record(stream)
    stream.synchronize()
    Th = cache.Th.cpu()
    kept = int(Th.sum())
    heads = w.B * w.Hkv
    nbytes = (kept * w.N * 2 + heads * w.N * w.d * 2 + w.B * w.Hq * w.d * 2 + w.B * w.Hq * w.d * 4 + kept * 4)
    us = e2.elapsed_time(e3) * 1e3 / w.decode_steps
    return {"tau": tau, "T_min": T_min, "T_max": T_max, "T_per_head": Th.tolist(),
            "mean_T": kept / heads, "prune_us": e0.elapsed_time(e1) * 1e3, "decode_us_per_step": us,
            "decode_gbs": nbytes / (us * 1e-6) / 1e9, "frac_of_measured_peak": nbytes / (us * 1e-6) / 1e9 / peak,
            "algorithmic_bytes_per_launch": nbytes,
            "kernel": "pruned_decode_mma_kernel, ragged mode (think_pruned_decode_attn_ragged), not part of the step"}


def measure_evict(w, T, dev, stream, qw_d, k_d, v_d, qs_d, outs, peak, keep=0.25):
    """Token eviction then channel pruning on the same layer, outside the timed
    step: the M = keep * N tokens of largest window attention mass are kept,
    then pruned to T channels; device time of that whole prune and of the
    step's decode calls over the M kept tokens."""
    import torch
    import query_driven_key_b200 as qdk
    import workloads as W
    M = max(1, int(w.N * keep))
    cache = qdk.EvictedCache(w.B, w.Hq, w.Hkv, w.N, w.S_obs, M, T, w.d, dtype=w.dtype, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        cache.prune(qw_d, k_d, v_d, stream=stream)
    e0, e1 = ev(), ev()
    e0.record(stream)
    cache.prune(qw_d, k_d, v_d, stream=stream)
    e1.record(stream)
    for s in range(3):
        cache.decode(qs_d[s], outs[s], stream=stream)
    e2, e3 = ev(), ev()
    e2.record(stream)
    for s in range(w.decode_steps):
        cache.decode(qs_d[s], outs[s], stream=stream)
    e3.record(stream)
    stream.synchronize()
    wm = w.with_(N=M)
    nbytes = W.decode_bytes(wm, T)
    us = e2.elapsed_time(e3) * 1e3 / w.decode_steps
    return {"kept_tokens": M, "T": T, "evict_and_prune_us": e0.elapsed_time(e1) * 1e3,
            "decode_us_per_step": us, "decode_gbs": nbytes / (us * 1e-6) / 1e9,
            "frac_of_measured_peak": nbytes / (us * 1e-6) / 1e9 / peak, "algorithmic_bytes_per_launch": nbytes,
            "note": "token_mass (2 launches) + select_tokens + 2 gathers + prune; decode over the kept tokens; "
                    "not part of the step"}


def data_recipe(w):
    if w.k_kind == "lowrank":
        keys = f"rank-{w.k_rank} N(0,1) factors + {w.k_noise} N(0,1) noise, LogNormal(0,{w.k_sigma}) channel scales"
    else:
        keys = f"LogNormal(0,{w.k_sigma}) channel-scaled N(0,1) keys"
    return f"synthetic (seeded {keys}, N(0,1) values/queries)"


def l2_note(w, T, R, hot=False):
    e = torch_elem_size(w.dtype)
    heads = w.B * w.Hkv
    kvp = heads * w.N * (w.d + T) * e
    k = heads * w.N * w.d * e
    if hot:
        return (f"hot: 1 resident layer (K {k / 1e6:.0f} MB, K'+V {kvp / 1e6:.0f} MB), read again every step "
                f"with no flush, so what fits in L2 is served from it")
    return (f"inputs larger than L2: {R} resident layer(s); a pass over them reads "
            f"K {R * k / 1e6:.0f} MB (prune) and K'+V {R * kvp / 1e6:.0f} MB (decode), no flush")


def decode_kernel_name(w):
    import torch
    if w.dtype == torch.bfloat16:
        return f"pruned_decode_mma_kernel<{w.G}, 4>"
    return f"pruned_decode_kernel<float, {w.G}>"


def cpu_baseline(w, T, seed_layer=0, budget_s=12.0):
    """The fp64 oracle as it stands, on this host's cores, on a bounded sample
    of the workload: the whole prune pass plus as many of the 256 decode steps
    as fit in about budget_s seconds (at least 4)."""
    import torch
    import oracle
    import workloads as W

    q_win, k, v = W.gen_layer(w, seed_layer)
    f64 = lambda t: t.to(torch.float64).numpy()
    qw, kk, vv = f64(q_win), f64(k), f64(v)
    o = oracle.default_oracle()
    t0 = time.perf_counter()
    _, idx, kp = o.prune(qw, kk, T)
    steps = 0
    while steps < w.decode_steps and (steps < 4 or time.perf_counter() - t0 < budget_s):
        o.decode(f64(W.gen_decode_q(w, steps, seed_layer)), kp, vv, idx)
        steps += 1
    dt = time.perf_counter() - t0
    nbytes = W.prune_bytes(w, T) + steps * W.decode_bytes(w, T)
    out = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": o.num_threads(), "kind": "oracle",
           "sample": f"prune of all {w.B * w.Hkv} KV heads + {steps} of {w.decode_steps} decode "
                     f"steps, fp64 C loops (OpenMP over heads), {dt:.2f} s"}
    # the same oracle on one thread: one KV head (its query group) of the
    # first batch item, prune + one decode step
    w1 = w.with_(B=1, Hkv=1, Hq=w.G)
    cores = o.num_threads()
    o.set_num_threads(1)
    try:
        t1 = time.perf_counter()
        _, idx1, kp1 = o.prune(qw[:1, :w.G], kk[:1, :1], T)
        o.decode(f64(W.gen_decode_q(w, 0, seed_layer))[:1, :w.G], kp1, vv[:1, :1], idx1)
        dt1 = time.perf_counter() - t1
    finally:
        o.set_num_threads(cores)
    nb1 = W.prune_bytes(w1, T) + W.decode_bytes(w1, T)
    out["one_thread"] = {"value": nb1 / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                         "sample": f"one KV head (group of {w.G} query heads): prune + 1 decode step, "
                                   f"{dt1:.2f} s"}
    return out


# ----------------------------------------------------- reference arm ---

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    import oracle
    import workloads as W

    w = workload(args)
    T = oracle.t_from_lambda(w.d, w.lam)
    q_win, k, v = W.gen_layer(w)
    f64 = lambda t: t.to(torch.float64).numpy()
    qw, kk, vv = f64(q_win), f64(k), f64(v)
    o = oracle.default_oracle()
    times = []
    for i in range(args.warmup + args.steps):
        q = f64(W.gen_decode_q(w, i))
        t0 = time.perf_counter()
        _, idx, kp = o.prune(qw, kk, T)
        o.decode(q, kp, vv, idx)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    nbytes = W.prune_bytes(w, T) + W.decode_bytes(w, T)
    sec = sum(times) / len(times)
    value = nbytes / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, bf16-rounded inputs)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "S_obs": w.S_obs, "lambda": w.lam, "T": T,
                   "sample": "each step: prune pass + 1 of the 256 decode steps"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": o.num_threads(), "kind": "oracle",
                         "sample": "prune of all KV heads + 1 decode step per timed step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------- native arm ---

def run_native(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import query_driven_key_b200 as qdk
    import workloads as W

    w = workload(args)
    T = qdk.think_t_from_lambda(w.d, w.lam)
    R = 1 if args.hot else resident_layers(w, T)
    # each rank: an independent replica on its own data; one generated layer
    # is copied into R device buffers (distinct addresses, so L2 cannot serve
    # one layer's reads from another's)
    q_win, k, v = W.gen_layer(w, layer=rank)
    qs = torch.stack([W.gen_decode_q(w, s, layer=rank) for s in range(w.decode_steps)])
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        qw_d = [q_win.to(dev) for _ in range(R)]
        k_d = [k.to(dev) for _ in range(R)]
        v_d = [v.to(dev) for _ in range(R)]
        qs_d = qs.to(dev)
        caches = [qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, T, w.d, dtype=w.dtype, device=dev)
                  for _ in range(R)]
        outs = torch.empty((w.decode_steps, R, w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    stream.synchronize()

    # prune: score+select, compact; one kernel per decode
    launches_per_step = R * (2 + w.decode_steps)

    # the per-step views of the decode queries and outputs are made once, so
    # that the host loop issuing short decodes does only the calls
    out_views = [[outs[s, r] for r in range(R)] for s in range(w.decode_steps)]
    q_views = {}

    def one_step(ev=None, bufs=None):
        qw_b, k_b, v_b, qs_b = bufs if bufs is not None else (qw_d, k_d, v_d, qs_d)
        qv = q_views.get(id(qs_b))
        if qv is None:
            qv = q_views[id(qs_b)] = (qs_b, [qs_b[s] for s in range(w.decode_steps)])
        qv = qv[1]
        if ev is not None:
            ev[0].record(stream)
        for r in range(R):
            caches[r].prune(qw_b[r], k_b[r], stream=stream)
        if ev is not None:
            ev[1].record(stream)
        for s in range(w.decode_steps):
            q_s, o_s = qv[s], out_views[s]
            for r in range(R):
                caches[r].decode(q_s, v_b[r], o_s[r], stream=stream)
        if ev is not None:
            ev[2].record(stream)

    def device_status():
        return max(max(qdk.think_read_device_status(c.decode_ws, stream),
                       qdk.think_read_device_status(c.score_ws, stream)) for c in caches)

    for _ in range(args.warmup):
        one_step()
    stream.synchronize()
    assert device_status() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            one_step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    prune_ms = [e[0].elapsed_time(e[1]) for e in evs]
    decode_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms, prune_sum, decode_sum = max_over_ranks([total_ms, sum(prune_ms), sum(decode_ms)], dev)
    assert device_status() == 0

    ms_per_step = total_ms / args.steps
    nbytes = R * step_bytes(w, T)
    value = aggregate_gbs(world, nbytes, ms_per_step)
    dec_bytes = W.decode_bytes(w, T)
    dec_us = decode_sum / args.steps / (w.decode_steps * R) * 1e3
    prune_us = prune_sum / args.steps / R * 1e3
    achieved = dec_bytes / (dec_us * 1e-6) / 1e9
    peak, peak_kind = measured_peaks()

    # ---------------------------------------------- end to end (host buffers)
    # Every step copies its inputs (window queries, K, V, the decode queries)
    # from pinned host memory and reads its outputs (decode outputs, kept
    # channels) back, inside the timed region.  With one resident layer the
    # device inputs are double-buffered: a copy stream fills one set while the
    # compute stream works on the other (events order them), as a server that
    # prefetches the next request would.
    e2e = None
    if args.e2e_steps > 0:
        pin = lambda t: t.pin_memory()
        h_qw, h_k, h_v, h_qs = pin(q_win), pin(k), pin(v), pin(qs)
        h_out = torch.empty(outs.shape, dtype=torch.float32).pin_memory()
        h_idx = torch.empty((R,) + tuple(caches[0].idx.shape), dtype=torch.int32).pin_memory()
        h2d = R * sum(t.numel() * t.element_size() for t in (h_qw, h_k, h_v)) \
            + h_qs.numel() * h_qs.element_size()
        d2h = h_out.numel() * 4 + h_idx.numel() * 4
        sets = [(qw_d, k_d, v_d, qs_d)]
        if R == 1:
            with torch.cuda.stream(stream):
                sets.append(([t.clone() for t in qw_d], [t.clone() for t in k_d], [t.clone() for t in v_d],
                             qs_d.clone()))
        copy_stream = torch.cuda.Stream(device=dev)
        free = [torch.cuda.Event() for _ in sets]
        ready = [torch.cuda.Event() for _ in sets]
        for e in free:
            e.record(stream)

        def copy_in(i):
            qw_b, k_b, v_b, qs_b = sets[i]
            copy_stream.wait_event(free[i])
            with torch.cuda.stream(copy_stream):
                for r in range(R):
                    qw_b[r].copy_(h_qw, non_blocking=True)
                    k_b[r].copy_(h_k, non_blocking=True)
                    v_b[r].copy_(h_v, non_blocking=True)
                qs_b.copy_(h_qs, non_blocking=True)
            ready[i].record(copy_stream)

        def e2e_steps(n):
            copy_in(0)
            for j in range(n):
                i = j % len(sets)
                if j + 1 < n:
                    copy_in((j + 1) % len(sets))   # the next step's inputs, while this one computes
                stream.wait_event(ready[i])
                with torch.cuda.stream(stream):
                    one_step(bufs=sets[i])
                    h_out.copy_(outs, non_blocking=True)
                    for r in range(R):
                        h_idx[r].copy_(caches[r].idx, non_blocking=True)
                free[i].record(stream)

        e2e_steps(2)
        stream.synchronize()
        copy_stream.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_stream.wait_event(e0)
        e2e_steps(args.e2e_steps)
        e1.record(stream)
        stream.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], dev)[0]
        e2e = {"value": aggregate_gbs(world, nbytes, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": args.e2e_steps, "input_buffers": len(sets)}

    extras = rank == 0 and not args.no_extras
    append = measure_append(w, T, dev, stream, qw_d[0], k_d[0]) if extras else None
    q4 = (measure_q4(w, T, stream, caches[0], qs_d, v_d[0], outs[:, 0], dec_us, peak)
          if extras and w.dtype == torch.bfloat16 else None)
    adaptive = (measure_adaptive(w, dev, stream, qw_d[0], k_d[0], qs_d, v_d[0], outs[:, 0], peak)
                if extras and w.dtype == torch.bfloat16 else None)
    evict = (measure_evict(w, T, dev, stream, qw_d[0], k_d[0], v_d[0], qs_d, outs[:, 0], peak)
             if extras and w.dtype == torch.bfloat16 else None)
    read_probe = measure_read_probe(dev, stream) if extras else None
    prune_1read, prune_2read = W.prune_bytes(w, T), W.prune_bytes(w, T, k_reads=2)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": data_recipe(w),
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "S_obs": w.S_obs, "lambda": w.lam, "T": T, "decode_steps_per_step": w.decode_steps,
                   "layers_per_step": R,
                   "parallelism": f"{world} independent replica(s), no collective",
                   "l2": l2_note(w, T, R, args.hot)},
        "pct_of_8tbs": value / world / NOMINAL_HBM_GBS * 100.0,
        "decode_gbs": achieved,
        "decode_pct_of_8tbs": achieved / NOMINAL_HBM_GBS * 100.0,
        "decode_us_per_step": dec_us,
        "prune_us_per_layer": prune_us,
        "prune_gbs_1read": prune_1read / (prune_us * 1e-6) / 1e9,
        "prune_frac_1read": prune_1read / (prune_us * 1e-6) / 1e9 / peak,
        "prune_gbs_2read": prune_2read / (prune_us * 1e-6) / 1e9,
        "prune_frac_2read": prune_2read / (prune_us * 1e-6) / 1e9 / peak,
        "roofline": {"kernel": f"{decode_kernel_name(w)} (think_pruned_decode_attn, one launch), "
                               f"CUDA events around each step's {w.decode_steps * R} decode calls",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "traffic": DECODE_TRAFFIC_BYTES if default_workload(args) else None},
        "append": append,
        "q4": q4,
        "adaptive": adaptive,
        "evict": evict,
        "read_probe": read_probe,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, T)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())

"""Seeded synthetic inputs for the ThinK decode-time path.

This module only draws random numbers; it holds none of the method's
arithmetic (no scoring, selection, compaction or attention). Both the CUDA
path's tests/bench and the CPU oracle's tests take their inputs from here.

The workloads stand in for the Llama/Mistral long-context evaluations of
"ThinK: Thinner Key Cache by Query-Driven Pruning" (experiments section), whose
models and datasets are not available here. Only their shapes are used. Keys
get uneven per-channel magnitudes (LogNormal channel scales), mirroring the
page's observation that key channels have an uneven magnitude distribution;
one workload also gives K a low-rank structure.

Every (layer, batch item) slice of a workload is drawn by its own CPU
``torch.Generator`` with a fixed seed, in a fixed order: window queries, key
factors, channel scales, values. Decode queries have their own seed per step.
Values are drawn in fp32 and rounded once to the workload dtype; every consumer
sees the same rounded tensors.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    label: str                     # the model shape it stands for; name adds the sizes
    seed: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    S_obs: int
    lam: float
    dtype: torch.dtype
    decode_steps: int
    layers: int = 1
    k_kind: str = "lognormal"      # "lognormal" or "lowrank"
    k_sigma: float = 1.0           # sigma of the LogNormal channel scales
    k_rank: int = 16               # rank of the low-rank key factors
    k_noise: float = 0.1           # noise added to the low-rank keys

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def name(self) -> str:
        """The label and the sizes the workload has now (with_ keeps them in step)."""
        dt = {torch.bfloat16: "bf16", torch.float32: "fp32"}.get(self.dtype, str(self.dtype))
        s = (f"{self.label}: B{self.B} Hq{self.Hq} Hkv{self.Hkv} d{self.d} N{self.N} S_obs{self.S_obs} "
             f"lambda{self.lam} {dt}")
        if self.layers > 1:
            s += f", {self.layers} layers"
        if self.k_kind == "lowrank":
            s += ", low-rank K"
        return s

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads (shapes of one decoder layer's attention, or 32 layers).
WORKLOADS = {
    "tiny_fp32": Workload("tiny single head", 0,
                          B=1, Hq=1, Hkv=1, N=512, d=128, S_obs=32, lam=0.5,
                          dtype=torch.float32, decode_steps=1),
    "llama2_7b_mha": Workload("llama2-7b-shaped MHA", 1,
                              B=1, Hq=32, Hkv=32, N=4096, d=128, S_obs=32, lam=0.4,
                              dtype=torch.bfloat16, decode_steps=64),
    "llama3_8b_gqa": Workload("llama3-8b-shaped GQA", 2,
                              B=4, Hq=32, Hkv=8, N=32768, d=128, S_obs=32, lam=0.5,
                              dtype=torch.bfloat16, decode_steps=1, k_kind="lowrank"),
    "mistral_7b_long": Workload("mistral-7b-shaped GQA long context", 3,
                                B=1, Hq=32, Hkv=8, N=131072, d=128, S_obs=64, lam=0.6,
                                dtype=torch.bfloat16, decode_steps=256, k_sigma=1.5),
    "sweep_32l": Workload("32-layer sweep", 4,
                          B=1, Hq=32, Hkv=8, N=8192, d=128, S_obs=32, lam=0.4,
                          dtype=torch.bfloat16, decode_steps=1, layers=32),
}
SWEEP_BATCHES = (1, 4, 16, 32)
SWEEP_LAMBDAS = (0.0, 0.4, 0.6)


def _slice_seed(w: Workload, layer: int, b: int) -> int:
    return (w.seed * 1_000_003 + layer * 10_007 + b) & 0x7FFF_FFFF_FFFF


def _step_seed(w: Workload, layer: int, step: int) -> int:
    return (w.seed * 1_000_003 + 7_777_777 + layer * 10_007 + step) & 0x7FFF_FFFF_FFFF


def gen_slice(w: Workload, layer: int, b: int):
    """One batch item of one layer: (q_win [Hq,S,d], k [Hkv,N,d], v [Hkv,N,d])."""
    g = torch.Generator(device="cpu")
    g.manual_seed(_slice_seed(w, layer, b))
    f32 = torch.float32
    q_win = torch.randn((w.Hq, w.S_obs, w.d), generator=g, dtype=f32)
    if w.k_kind == "lowrank":
        a = torch.randn((w.Hkv, w.N, w.k_rank), generator=g, dtype=f32)
        bf = torch.randn((w.Hkv, w.d, w.k_rank), generator=g, dtype=f32)
        k = torch.bmm(a, bf.transpose(1, 2))
        k += w.k_noise * torch.randn((w.Hkv, w.N, w.d), generator=g, dtype=f32)
    else:
        k = torch.randn((w.Hkv, w.N, w.d), generator=g, dtype=f32)
    scales = torch.exp(w.k_sigma * torch.randn((w.Hkv, 1, w.d), generator=g, dtype=f32))
    k *= scales
    v = torch.randn((w.Hkv, w.N, w.d), generator=g, dtype=f32)
    return q_win.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def gen_layer(w: Workload, layer: int = 0):
    """All batch items of one layer: q_win [B,Hq,S,d], k [B,Hkv,N,d], v [B,Hkv,N,d]."""
    qs, ks, vs = [], [], []
    for b in range(w.B):
        q, k, v = gen_slice(w, layer, b)
        qs.append(q)
        ks.append(k)
        vs.append(v)
    return torch.stack(qs), torch.stack(ks), torch.stack(vs)


def gen_decode_q(w: Workload, step: int, layer: int = 0) -> torch.Tensor:
    """The decode query of one step: q [B,Hq,d] ~ N(0,1)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(_step_seed(w, layer, step))
    return torch.randn((w.B, w.Hq, w.d), generator=g, dtype=torch.float32).to(w.dtype)


def decode_bytes(w: Workload, T: int) -> int:
    """Algorithmic HBM bytes of one decode step: K' (unpadded) + V + q + out(fp32) + idx."""
    e = torch.empty((), dtype=w.dtype).element_size()
    heads = w.B * w.Hkv
    return (heads * w.N * T * e + heads * w.N * w.d * e + w.B * w.Hq * w.d * e
            + w.B * w.Hq * w.d * 4 + heads * T * 4)


def decode_bytes_q4(w: Workload, T: int) -> int:
    """Algorithmic HBM bytes of one decode step over the 4-bit thinner cache:
    codes (half a byte per kept element) + group parameters (8 bytes per kept
    channel and 128 tokens) + V + q + out(fp32) + idx."""
    heads = w.B * w.Hkv
    return (heads * w.N * T // 2 + heads * (-(-w.N // 128)) * T * 8 + heads * w.N * w.d * 2
            + w.B * w.Hq * w.d * 2 + w.B * w.Hq * w.d * 4 + heads * T * 4)


def prune_bytes(w: Workload, T: int, k_reads: int = 1) -> int:
    """Algorithmic HBM bytes of one prune pass: K read k_reads times + K' written +
    Q_win read + idx written."""
    e = torch.empty((), dtype=w.dtype).element_size()
    heads = w.B * w.Hkv
    return (k_reads * heads * w.N * w.d * e + heads * w.N * T * e
            + w.B * w.Hq * w.S_obs * w.d * e + heads * T * 4)

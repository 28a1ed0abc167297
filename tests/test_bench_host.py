"""Host-side logic of bench.py (no GPU): workload overrides and how many
resident layer copies a bench step cycles through so that its reads exceed L2."""
import argparse

import pytest

import bench
import workloads as W


def _args(**kw):
    base = dict(workload=bench.WORKLOAD, batch=None, lam=None, decode_steps=None)
    base.update(kw)
    return argparse.Namespace(**base)


def _T(w):
    import oracle
    return oracle.t_from_lambda(w.d, w.lam)


def test_default_workload_is_the_long_context_layer():
    a = _args()
    w = bench.workload(a)
    assert w is W.WORKLOADS["mistral_7b_long"]
    assert bench.default_workload(a)
    assert not bench.default_workload(_args(batch=1))


def test_overrides():
    w = bench.workload(_args(workload="sweep_32l", batch=16, lam=0.0, decode_steps=2))
    assert (w.B, w.lam, w.decode_steps, w.layers) == (16, 0.0, 2, 32)


@pytest.mark.parametrize("name,expect", [("mistral_7b_long", 1), ("llama3_8b_gqa", 1),
                                         ("llama2_7b_mha", 3), ("sweep_32l", 32)])
def test_resident_layers(name, expect):
    w = W.WORKLOADS[name]
    R = bench.resident_layers(w, _T(w))
    assert R == expect
    # a pass over the resident layers reads at least twice L2 (or is all layers)
    per_layer = w.B * w.Hkv * w.N * (2 * w.d + _T(w)) * 2
    assert w.layers > 1 or R * per_layer >= 2 * bench.L2_BYTES
    assert R == 1 or w.layers > 1 or (R - 1) * per_layer < 2 * bench.L2_BYTES


def test_l2_note_and_kernel_name():
    w = W.WORKLOADS["mistral_7b_long"]
    note = bench.l2_note(w, _T(w), 1)
    assert "K 268 MB" in note and "K'+V 375 MB" in note
    assert bench.decode_kernel_name(w) == "pruned_decode_mma_kernel<4, 4>"
    assert bench.decode_kernel_name(W.WORKLOADS["tiny_fp32"]).startswith("pruned_decode_kernel<float")

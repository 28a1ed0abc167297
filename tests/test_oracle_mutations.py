"""Planted mistakes: each plausible slip in the oracle must fail at least one pin.

Each case copies the oracle's C source, plants one mistake (a dropped term, a
wrong sign, index or scale, a transposed operand, a flipped tie rule), compiles
the copy into a temporary library and runs the pins of test_oracle_pins.py
against it. The committed oracle is never modified.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "think_oracle.c")
GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))

MUTATIONS = {
    "squares_replaced_by_abs": ("kn2[c] += x * x;", "kn2[c] += fabs(x);"),
    "group_sum_dropped": ("s += sqrt(qn2) * sqrt(kn2[c]);", "s = sqrt(qn2) * sqrt(kn2[c]);"),
    "group_rows_concatenated": ("s += sqrt(qn2) * sqrt(kn2[c]);", "s += qn2 * kn2[c];"),
    "tie_to_higher_index": ("    return (a > b) - (a < b);\n}\n\nstatic int ascending",
                            "    return (b > a) - (b < a);\n}\n\nstatic int ascending"),
    "kept_list_not_reordered": ("qsort(order, (size_t)T, sizeof(int), ascending_int);\n        for (int t = 0; t < T; ++t) idx[(size_t)bh * T + t]",
                                "for (int t = 0; t < T; ++t) idx[(size_t)bh * T + t]"),
    "gather_uses_position": ("k[((size_t)bh * N + (size_t)n) * d + ih[t]];",
                             "k[((size_t)bh * N + (size_t)n) * d + t];"),
    "gather_transposed": ("k[((size_t)bh * N + (size_t)n) * d + ih[t]];",
                          "k[((size_t)bh * N + (size_t)(ih[t] % N)) * d + (n % d)];"),
    "scale_of_kept_width": ("\n        z[n] = dot * scale;", "\n        z[n] = dot * scale * sqrt((double)d / W);"),
    "softmax_sign": ("\n        z[n] = exp(z[n] - m);", "\n        z[n] = exp(m - z[n]);"),
    "softmax_not_normalised": ("const double p = z[n] / l;", "const double p = z[n];"),
    "gqa_head_mapping_modulo": ("kv = h / G;\n        const size_t kvh = (size_t)b * Hkv + (size_t)kv;\n"
                                "        const int32_t *ih",
                                "kv = h % Hkv;\n        const size_t kvh = (size_t)b * Hkv + (size_t)kv;\n"
                                "        const int32_t *ih"),
    "query_not_gathered": ("qp[t] = q[(size_t)bhq * d + ih[t]];", "qp[t] = q[(size_t)bhq * d + t];"),
    "q4_step_of_16_levels": ("const float scale = (mx - mn) / 15.0f;", "const float scale = (mx - mn) / 16.0f;"),
    "q4_truncated_codes": ("c = rintf((x - mn) / scale);", "c = floorf((x - mn) / scale);"),
    "q4_min_not_added": ("bf16_round(fmaf(c, gs[gi], gs[gi + 1]))", "bf16_round(c * gs[gi])"),
    "q4_group_index_of_next_group": ("(((size_t)bh * ng + n / group) * T + t) * 2;",
                                     "(((size_t)bh * ng + (n + 1) / group) * T + t) * 2;"),
    "adaptive_strict_threshold": ("if (k >= T_min && cum >= tau * E) {", "if (k >= T_min && cum > tau * E) {"),
    "adaptive_energy_unsquared": ("cum += s[order[k - 1]] * s[order[k - 1]];", "cum += s[order[k - 1]];"),
    "mass_without_scale": ("z[n] = dot * scale;\n                        if (z[n] > m) m = z[n];",
                           "z[n] = dot;\n                        if (z[n] > m) m = z[n];"),
    "mass_not_normalised": ("for (int n = 0; n < N; ++n) mh[n] += z[n] / l;",
                            "for (int n = 0; n < N; ++n) mh[n] += z[n];"),
    "adaptive_offsets_not_advanced": ("        rows += T;\n    }\n    off[B * Hkv] = rows;",
                                      "    }\n    off[B * Hkv] = rows;"),
    "tokens_kept_list_not_reordered": ("        qsort(order, (size_t)M, sizeof(int), ascending_int);\n", ""),
    "tokens_first_m_by_index": ("qsort(order, (size_t)N, sizeof(int), by_score_desc);",
                                "qsort(order, (size_t)N, sizeof(int), ascending_int);"),
}


def _pins(o: oracle.Oracle):
    """Yield (name, passed) for the core pins, run against oracle instance o."""
    r = np.random.default_rng(5)
    # factorised score == explicit Frobenius norm (with a GQA group)
    q_win = r.standard_normal((1, 4, 3, 8))
    k = r.standard_normal((1, 2, 7, 8)) * r.lognormal(0, 1, (1, 1, 1, 8))
    yield "frobenius", np.allclose(o.score(q_win, k), o.score_explicit(q_win, k), rtol=1e-12, atol=0)
    g = GOLDEN["score_mha"]
    s = o.score(g["q_win"], g["k"])
    ok = np.allclose(s[0, 0], [math.sqrt(5), 3 * math.sqrt(2), 2 * math.sqrt(2), math.sqrt(5)], rtol=1e-15)
    ok &= all(o.select(s, int(T))[0, 0].tolist() == v for T, v in g["select"].items())
    yield "golden_mha", ok
    g = GOLDEN["score_gqa"]
    s = o.score(g["q_win"], g["k"])
    ok = np.allclose(s[0], g["scores"], rtol=1e-15)
    ok &= all(o.select(s, int(T))[0, 0].tolist() == v for T, v in g["select"].items())
    yield "golden_gqa", ok
    # selection order against Python's sort
    sc = r.integers(0, 5, size=(1, 2, 16)).astype(np.float64)
    ok = True
    for T in (3, 9):
        idx = o.select(sc, T)
        for h in range(2):
            order = sorted(range(16), key=lambda c: (-sc[0, h, c], c))
            ok &= idx[0, h].tolist() == sorted(order[:T])
    yield "select_sort", ok
    # compaction against numpy's gather
    kk = r.standard_normal((1, 2, 9, 16))
    idx = np.array([[[1, 5, 6], [0, 2, 15]]], dtype=np.int32)
    ref = np.take_along_axis(kk, np.broadcast_to(idx[:, :, None, :], (1, 2, 9, 3)), axis=3)
    yield "compact_gather", np.array_equal(o.compact(kk, idx), ref)
    # hand-worked decode
    g = GOLDEN["decode"]
    out = o.decode(g["q"], o.compact(g["k"], g["idx"]), g["v"], g["idx"])
    yield "golden_decode", np.allclose(out, g["out"], rtol=0, atol=1e-12)
    # pruned decode == torch SDPA on masked K (GQA group of 2)
    B, Hkv, N, d, T, G = 1, 2, 13, 8, 3, 2
    q = r.standard_normal((B, Hkv * G, d))
    k = r.standard_normal((B, Hkv, N, d)) * 2
    v = r.standard_normal((B, Hkv, N, d))
    idx = np.array([[[0, 3, 6], [1, 2, 7]]], dtype=np.int32)
    out = o.decode(q, o.compact(k, idx), v, idx)
    mask = np.zeros((B, Hkv, 1, d))
    for h in range(Hkv):
        mask[0, h, 0, idx[0, h]] = 1
    qt = torch.from_numpy(q)[:, :, None, :]
    kt = torch.from_numpy(k * mask).repeat_interleave(G, 1)
    vt = torch.from_numpy(v).repeat_interleave(G, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[:, :, 0].numpy()
    yield "sdpa_masked", np.allclose(out, ref, rtol=1e-12, atol=1e-13)
    # 4-bit thinner K: grid values are exact; min -> 0 and max -> 15; error bound
    kgrid = np.zeros((1, 1, 130, 2))
    kq = r.integers(0, 16, size=(130, 2))
    kq[0], kq[1], kq[128], kq[129] = 0, 15, 0, 15
    kgrid[0, 0] = -1.0 + kq / 8.0
    codes, gs = o.quantize_q4(kgrid)
    ok = np.array_equal(codes[0, 0], kq) and np.array_equal(o.dequantize_q4(codes, gs), kgrid)
    yield "q4_grid", ok
    kr = torch.from_numpy(r.standard_normal((1, 1, 200, 3)) * 2).to(torch.bfloat16).double().numpy()
    codes, gs = o.quantize_q4(kr)
    khat = o.dequantize_q4(codes, gs)
    step = np.repeat(gs[..., 0], 128, axis=2)[:, :, :200].astype(np.float64)
    yield "q4_bound", bool(np.all(np.abs(khat - kr) <= 0.5 * step * (1 + 1e-5) + np.abs(khat) * 2.0 ** -8))
    # adaptive kept width: hand-worked thresholds and ragged offsets
    sc2 = np.array([[[3.0, 4.0, 0.0, 0.0], [1.0, 1.0, 1.0, 1.0]]])
    ok = True
    for tau, T0, T1 in [(0.64, 1, 3), (0.65, 2, 3), (0.26, 1, 2)]:
        Th, off, ix = o.select_adaptive(sc2, tau, 1, 4)
        ok &= Th.tolist() == [[T0, T1]] and list(off) == [0, T0, T0 + T1]
        ok &= list(ix[:T0]) == ([1] if T0 == 1 else [0, 1])
    yield "adaptive_hand", bool(ok)
    # token mass against torch's softmax, and its row-sum closed form
    qw = r.standard_normal((1, 2, 3, 8))
    kk = r.standard_normal((1, 1, 11, 8))
    mass = o.token_mass(qw, kk)
    p = torch.softmax(torch.from_numpy(qw[0].reshape(6, 8)) @ torch.from_numpy(kk[0, 0]).T / math.sqrt(8), -1)
    yield "mass_softmax", bool(np.allclose(mass[0, 0], p.sum(0).numpy(), rtol=1e-12, atol=1e-15))
    # token selection against Python's sort (largest mass, ties to the lower
    # index, kept indices ascending), with many exact ties
    ms = r.integers(0, 4, size=(1, 2, 20)).astype(np.float64)
    ok = True
    for M in (1, 7, 20):
        kept = o.select_tokens(ms, M)
        for h in range(2):
            order = sorted(range(20), key=lambda n: (-ms[0, h, n], n))
            ok &= kept[0, h].tolist() == sorted(order[:M])
    yield "select_tokens_sort", bool(ok)


def _all_pass(o):
    return {name: bool(ok) for name, ok in _pins(o)}


def test_committed_oracle_passes_every_pin():
    res = _all_pass(oracle.default_oracle())
    assert all(res.values()), res


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/present"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(mutated), out=str(tmp_path / "libmutant.so"))
    res = _all_pass(oracle.Oracle(so))
    assert not all(res.values()), f"planted mistake {name} passed every pin: {res}"

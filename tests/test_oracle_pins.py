"""Pins of the fp64 CPU oracle against things other than itself.

The ThinK page ("ThinK: Thinner Key Cache by Query-Driven Pruning") prints no
worked example and no formula, so the oracle is pinned by:

* the closed form behind the score: the Frobenius norm of a rank-one outer
  product equals the product of the two vector norms (checked against the
  explicit matrix and against numpy's matrix norm);
* hand-worked examples (tests/golden/hand_worked.json, derivations inside);
* the abstract's objective, by brute force over all channel subsets at d=8,
  including the orthogonal-query and orthogonal-key special cases, where the
  norm ranking is provably the exact minimiser of the attention-weight loss;
* library routines: Python's sort for the selection order, numpy's gather for
  the compaction, torch's fp64 scaled_dot_product_attention for decode;
* invariants: lambda = 0 reproduces dense attention bit for bit, softmax
  weights sum to one, all-zero channels make pruning lossless;
* growing cache: appending keys chunk by chunk equals compacting the whole
  cache at once, lambda = 0 over a grown cache equals dense attention over all
  keys, and an appended token that dominates the logits takes the whole
  softmax weight (closed form).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- score ---

@pytest.mark.parametrize("G", [1, 2, 4])
def test_score_closed_form_equals_explicit_frobenius(G):
    r = rng(10 + G)
    B, Hkv, S, N, d = 2, 2, 5, 11, 8
    q_win = r.standard_normal((B, Hkv * G, S, d))
    k = r.standard_normal((B, Hkv, N, d)) * r.lognormal(0, 1, (1, 1, 1, d))
    fast = oracle.oracle_score(q_win, k)
    slow = oracle.oracle_score_explicit(q_win, k)
    np.testing.assert_allclose(fast, slow, rtol=1e-12, atol=0)
    # and against numpy's Frobenius norm of the explicit outer product
    for b in range(B):
        for kv in range(Hkv):
            for c in range(d):
                ref = sum(np.linalg.norm(np.outer(q_win[b, kv * G + g, :, c], k[b, kv, :, c]), "fro")
                          for g in range(G))
                assert math.isclose(fast[b, kv, c], ref, rel_tol=1e-12)


def test_score_hand_worked_mha():
    g = GOLDEN["score_mha"]
    s = oracle.oracle_score(g["q_win"], g["k"])[0, 0]
    expect = [math.sqrt(5), 3 * math.sqrt(2), 2 * math.sqrt(2), math.sqrt(5)]
    np.testing.assert_allclose(s, expect, rtol=1e-15)
    for T, idx in g["select"].items():
        got = oracle.oracle_select(s[None, None, :], int(T))[0, 0].tolist()
        assert got == idx, (T, got, idx)


def test_score_hand_worked_gqa_group_sum():
    g = GOLDEN["score_gqa"]
    s = oracle.oracle_score(g["q_win"], g["k"])[0]
    np.testing.assert_allclose(s, g["scores"], rtol=1e-15)
    for T, idx in g["select"].items():
        got = oracle.oracle_select(s[None], int(T))[0, 0].tolist()
        assert got == idx, (T, got, idx)


def test_score_empty_window_and_empty_cache():
    # Norms of empty vectors are zero; every channel ties and the lowest indices win.
    q_win = np.zeros((1, 2, 0, 8))
    k = rng(1).standard_normal((1, 1, 5, 8))
    s = oracle.oracle_score(q_win, k)
    assert np.all(s == 0)
    assert oracle.oracle_select(s, 3)[0, 0].tolist() == [0, 1, 2]
    s2 = oracle.oracle_score(rng(2).standard_normal((1, 1, 3, 8)), np.zeros((1, 1, 0, 8)))
    assert np.all(s2 == 0)


# --------------------------------------------------------------- select ---

@pytest.mark.parametrize("seed", range(6))
def test_select_matches_python_sort(seed):
    r = rng(100 + seed)
    B, Hkv, d = 2, 3, 16
    s = r.integers(0, 6, size=(B, Hkv, d)).astype(np.float64)  # many exact ties
    s += (seed % 2) * r.random((B, Hkv, d))
    for T in (1, 5, 8, 15, 16):
        idx = oracle.oracle_select(s, T)
        for b in range(B):
            for h in range(Hkv):
                order = sorted(range(d), key=lambda c: (-s[b, h, c], c))
                assert idx[b, h].tolist() == sorted(order[:T])


def test_select_rejects_bad_T():
    with pytest.raises(ValueError):
        oracle.oracle_select(np.zeros((1, 1, 8)), 0)
    with pytest.raises(ValueError):
        oracle.oracle_select(np.zeros((1, 1, 8)), 9)


# -------------------------------------------- objective vs brute force ---

def _orthonormal(r, rows, cols):
    a = r.standard_normal((rows, cols))
    qm, _ = np.linalg.qr(a)
    return qm[:, :cols]


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("T", [2, 3, 4, 5, 6])
def test_norm_ranking_is_optimal_for_orthogonal_queries(seed, T):
    # With orthogonal window-query columns the cross terms of
    # ||sum_{c not kept} q_c k_c^T||_F^2 vanish, leaving sum |q_c|^2 |k_c|^2:
    # keeping the largest |q_c||k_c| is then exactly optimal.
    r = rng(1000 + seed)
    d, S, N = 8, 10, 12
    Q = _orthonormal(r, S, d) * r.lognormal(0, 1, d)
    K = r.standard_normal((N, d)) * r.lognormal(0, 1, d)
    s = oracle.oracle_score(Q[None, None], K[None, None])
    idx = tuple(oracle.oracle_select(s, T)[0, 0].tolist())
    best, argmins = oracle.bruteforce_best_subset(Q, K, T)
    assert idx in argmins
    assert math.isclose(oracle.attention_loss(Q, K, idx), best, rel_tol=1e-12, abs_tol=1e-12)


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("T", [2, 4, 6])
def test_norm_ranking_is_optimal_for_orthogonal_keys(seed, T):
    r = rng(2000 + seed)
    d, S, N = 8, 6, 16
    Q = r.standard_normal((S, d))
    K = _orthonormal(r, N, d) * r.lognormal(0, 1, d)
    s = oracle.oracle_score(Q[None, None], K[None, None])
    idx = tuple(oracle.oracle_select(s, T)[0, 0].tolist())
    best, argmins = oracle.bruteforce_best_subset(Q, K, T)
    assert idx in argmins


def test_norm_ranking_on_random_inputs_is_near_optimal():
    # The ranking is a greedy stand-in for the abstract's objective; on random
    # inputs it is not always the exact minimiser. Record how close it gets:
    # its loss must beat the median subset and stay within 2x of the optimum.
    r = rng(3000)
    d, S, N = 8, 8, 16
    hits, ratios = 0, []
    for trial in range(20):
        Q = r.standard_normal((S, d))
        K = r.standard_normal((N, d)) * r.lognormal(0, 1, d)
        T = 2 + trial % 5
        s = oracle.oracle_score(Q[None, None], K[None, None])
        idx = tuple(oracle.oracle_select(s, T)[0, 0].tolist())
        best, argmins = oracle.bruteforce_best_subset(Q, K, T)
        loss = oracle.attention_loss(Q, K, idx)
        allloss = sorted(oracle.attention_loss(Q, K, c) for c in itertools.combinations(range(d), T))
        assert loss <= allloss[len(allloss) // 2]
        ratios.append(loss / best)
        hits += idx in argmins
    assert max(ratios) < 2.0
    assert hits >= 10, f"greedy hit the optimum {hits}/20 times"


# -------------------------------------------------------------- compact ---

def test_compact_equals_numpy_gather():
    r = rng(7)
    B, Hkv, N, d, T = 2, 3, 9, 16, 5
    k = r.standard_normal((B, Hkv, N, d))
    idx = np.stack([np.stack([np.sort(r.choice(d, T, replace=False)) for _ in range(Hkv)])
                    for _ in range(B)]).astype(np.int32)
    kp = oracle.oracle_compact(k, idx)
    ref = np.take_along_axis(k, np.broadcast_to(idx[:, :, None, :], (B, Hkv, N, T)), axis=3)
    assert np.array_equal(kp, ref)


def test_compact_rejects_out_of_range_index():
    with pytest.raises(ValueError):
        oracle.oracle_compact(np.zeros((1, 1, 2, 4)), np.array([[[0, 4]]], dtype=np.int32))


# --------------------------------------------------------------- decode ---

def test_decode_hand_worked():
    g = GOLDEN["decode"]
    kp = oracle.oracle_compact(g["k"], g["idx"])
    out = oracle.oracle_decode(g["q"], kp, g["v"], g["idx"])
    np.testing.assert_allclose(out, g["out"], rtol=0, atol=1e-12)


def test_decode_gqa_head_mapping():
    r = rng(8)
    B, Hq, Hkv, N, d, T = 1, 4, 2, 7, 8, 3
    q = r.standard_normal((B, Hq, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = np.ones((B, Hkv, N, d))
    v[:, 1] = 2.0
    idx = np.array([[[0, 3, 5], [1, 2, 7]]], dtype=np.int32)
    out = oracle.oracle_decode(q, oracle.oracle_compact(k, idx), v, idx)
    expect = GOLDEN["gqa_mapping"]["out_row_values"]
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], expect[h], rtol=0, atol=1e-12)


def _sdpa(q, k, v, G):
    # torch's fp64 attention on CPU; default scale 1/sqrt(last dim of q).
    qt = torch.from_numpy(q)[:, :, None, :]                       # [B,Hq,1,d]
    kt = torch.from_numpy(k)
    vt = torch.from_numpy(v)
    kt = kt.repeat_interleave(G, dim=1)
    vt = vt.repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[:, :, 0, :].numpy()


@pytest.mark.parametrize("G", [1, 4])
def test_pruned_decode_equals_sdpa_on_masked_keys(G):
    # Attending with K' and q' equals full attention on K with the dropped
    # channels zeroed, at the full-width scale 1/sqrt(d).
    r = rng(20 + G)
    B, Hkv, N, d, T = 2, 2, 37, 16, 6
    Hq = Hkv * G
    q = r.standard_normal((B, Hq, d))
    k = r.standard_normal((B, Hkv, N, d)) * 2
    v = r.standard_normal((B, Hkv, N, d))
    q_win = r.standard_normal((B, Hq, 4, d))
    _, idx, kp = oracle.oracle_prune(q_win, k, T)
    out = oracle.oracle_decode(q, kp, v, idx)
    mask = np.zeros((B, Hkv, 1, d))
    for b in range(B):
        for h in range(Hkv):
            mask[b, h, 0, idx[b, h]] = 1.0
    ref = _sdpa(q, k * mask, v, G)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("G", [1, 2])
def test_dense_decode_equals_sdpa(G):
    r = rng(30 + G)
    B, Hkv, N, d = 2, 3, 50, 8
    q = r.standard_normal((B, Hkv * G, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    np.testing.assert_allclose(oracle.oracle_dense_decode(q, k, v), _sdpa(q, k, v, G),
                               rtol=1e-12, atol=1e-13)


def test_lambda_zero_reproduces_dense_bit_for_bit():
    r = rng(40)
    B, Hq, Hkv, S, N, d = 2, 4, 2, 8, 33, 16
    q_win = r.standard_normal((B, Hq, S, d))
    k = r.standard_normal((B, Hkv, N, d)) * r.lognormal(0, 1, (1, 1, 1, d))
    v = r.standard_normal((B, Hkv, N, d))
    q = r.standard_normal((B, Hq, d))
    T = oracle.t_from_lambda(d, 0.0)
    assert T == d
    _, idx, kp = oracle.oracle_prune(q_win, k, T)
    assert np.array_equal(idx, np.broadcast_to(np.arange(d, dtype=np.int32), (B, Hkv, d)))
    assert np.array_equal(kp, k)
    assert np.array_equal(oracle.oracle_decode(q, kp, v, idx), oracle.oracle_dense_decode(q, k, v))


def test_softmax_weights_sum_to_one():
    r = rng(50)
    B, Hq, Hkv, N, d, T = 1, 2, 1, 64, 16, 5
    q = r.standard_normal((B, Hq, d)) * 4
    k = r.standard_normal((B, Hkv, N, d)) * 4
    idx = np.array([[[1, 4, 6, 9, 15]]], dtype=np.int32)
    kp = oracle.oracle_compact(k, idx)
    ones = np.ones((B, Hkv, N, d))
    np.testing.assert_allclose(oracle.oracle_decode(q, kp, ones, idx), 1.0, rtol=0, atol=1e-12)
    # with V = identity rows the output is the weight vector itself: compare to torch.softmax
    eye = np.zeros((B, Hkv, N, N))
    eye[0, 0] = np.eye(N)
    w = oracle.oracle_decode(np.pad(q, ((0, 0), (0, 0), (0, N - d))), kp, eye, idx,
                             scale=1 / math.sqrt(d))
    for h in range(Hq):
        z = torch.from_numpy(kp[0, 0] @ q[0, h, idx[0, 0]]) / math.sqrt(d)
        np.testing.assert_allclose(w[0, h], torch.softmax(z, 0).numpy(), rtol=1e-12, atol=1e-15)
        assert math.isclose(w[0, h].sum(), 1.0, rel_tol=1e-12)


def test_zero_channels_make_pruning_lossless():
    # K with exactly d-T all-zero channels: those channels score 0, pruning them
    # loses nothing, and the pruned decode equals the dense decode.
    r = rng(60)
    B, Hq, Hkv, S, N, d, T = 1, 4, 2, 6, 40, 16, 7
    keep = [np.sort(r.choice(d, T, replace=False)) for _ in range(Hkv)]
    k = r.standard_normal((B, Hkv, N, d))
    for h in range(Hkv):
        drop = np.setdiff1d(np.arange(d), keep[h])
        k[0, h, :, drop] = 0.0
    q_win = r.standard_normal((B, Hq, S, d))
    v = r.standard_normal((B, Hkv, N, d))
    q = r.standard_normal((B, Hq, d))
    _, idx, kp = oracle.oracle_prune(q_win, k, T)
    for h in range(Hkv):
        assert idx[0, h].tolist() == keep[h].tolist()
    np.testing.assert_allclose(oracle.oracle_decode(q, kp, v, idx),
                               oracle.oracle_dense_decode(q, k, v), rtol=1e-14, atol=1e-15)


def test_decode_rejects_empty_cache():
    with pytest.raises(ValueError):
        oracle.oracle_decode(np.zeros((1, 1, 4)), np.zeros((1, 1, 0, 2)), np.zeros((1, 1, 0, 4)),
                             np.array([[[0, 1]]], dtype=np.int32))


def test_t_from_lambda_rule():
    for d, lam, T in GOLDEN["t_from_lambda"]["cases"]:
        assert oracle.t_from_lambda(d, lam) == T, (d, lam)


# -------------------------------------------------------- growing cache ---

def test_append_in_chunks_equals_compacting_everything():
    r = rng(70)
    B, Hkv, N, d, T = 2, 3, 41, 16, 6
    k = r.standard_normal((B, Hkv, N, d))
    idx = np.sort(np.stack([np.stack([r.choice(d, T, replace=False) for _ in range(Hkv)])
                            for _ in range(B)]), axis=-1).astype(np.int32)
    kp = oracle.oracle_compact(k[:, :, :10], idx)
    for a, b in [(10, 11), (11, 18), (18, 18), (18, 40), (40, 41)]:
        kp = oracle.oracle_append(kp, k[:, :, a:b], idx)
    assert kp.shape == (B, Hkv, N, T)
    assert np.array_equal(kp, oracle.oracle_compact(k, idx))
    assert np.array_equal(kp, np.take_along_axis(k, idx[:, :, None, :].repeat(N, 2), axis=3))


def test_grown_cache_at_lambda_zero_is_dense_attention():
    r = rng(71)
    B, Hq, Hkv, N0, n, d = 1, 4, 2, 20, 13, 8
    q = r.standard_normal((B, Hq, d))
    k = r.standard_normal((B, Hkv, N0 + n, d))
    v = r.standard_normal((B, Hkv, N0 + n, d))
    idx = np.broadcast_to(np.arange(d, dtype=np.int32), (B, Hkv, d)).copy()
    kp = oracle.oracle_append(oracle.oracle_compact(k[:, :, :N0], idx), k[:, :, N0:], idx)
    np.testing.assert_array_equal(oracle.oracle_decode(q, kp, v, idx), oracle.oracle_dense_decode(q, k, v))
    np.testing.assert_allclose(oracle.oracle_decode(q, kp, v, idx), _sdpa(q, k, v, Hq // Hkv),
                               rtol=1e-12, atol=1e-13)


def test_dominant_appended_token_takes_all_weight():
    # the appended token's key on the kept channels is 800 q' / |q'|^2, so its
    # logit is 800 / sqrt(16) = 200; the cached keys are tiny (logits ~ 0.01),
    # so every other softmax weight is below e^-190
    r = rng(72)
    B, Hq, Hkv, N0, d, T = 1, 1, 1, 30, 16, 4
    idx = np.array([[[2, 5, 11, 13]]], dtype=np.int32)
    q = r.standard_normal((B, Hq, d))
    k_old = 0.01 * r.standard_normal((B, Hkv, N0, d))
    k_new = np.zeros((B, Hkv, 1, d))
    qk = q[0, 0, idx[0, 0]]
    k_new[0, 0, 0, idx[0, 0]] = 800.0 * qk / np.dot(qk, qk)
    v = r.standard_normal((B, Hkv, N0 + 1, d))
    kp = oracle.oracle_append(oracle.oracle_compact(k_old, idx), k_new, idx)
    out = oracle.oracle_decode(q, kp, v, idx)
    np.testing.assert_allclose(out[0, 0], v[0, 0, N0], rtol=0, atol=1e-12)


# ------------------------------------------------------- 4-bit thinner K ---

def _bf16_values(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def test_q4_codes_span_each_group():
    r = rng(80)
    B, Hkv, N, T, group = 2, 2, 300, 5, 128
    kp = _bf16_values(r.standard_normal((B, Hkv, N, T)) * r.lognormal(0, 1, (1, 1, 1, T)))
    codes, gs = oracle.oracle_quantize_q4(kp, group)
    assert codes.max() <= 15
    for g0 in range(0, N, group):
        blk = kp[:, :, g0:g0 + group]
        cb = codes[:, :, g0:g0 + group]
        gi = g0 // group
        # the group's parameters are its own min and (max - min) / 15
        np.testing.assert_array_equal(gs[:, :, gi, :, 1], blk.min(axis=2).astype(np.float32))
        np.testing.assert_array_equal(gs[:, :, gi, :, 0],
                                      ((blk.max(axis=2) - blk.min(axis=2)).astype(np.float32) / np.float32(15)))
        # the minimum maps to code 0 and the maximum to code 15
        amin, amax = blk.argmin(axis=2), blk.argmax(axis=2)
        assert np.all(np.take_along_axis(cb, amin[:, :, None, :], 2) == 0)
        assert np.all(np.take_along_axis(cb, amax[:, :, None, :], 2) == 15)


def test_q4_error_is_within_half_a_step_plus_bf16_rounding():
    r = rng(81)
    B, Hkv, N, T = 1, 3, 257, 7
    kp = _bf16_values(r.standard_normal((B, Hkv, N, T)) * 3)
    codes, gs = oracle.oracle_quantize_q4(kp)
    khat = oracle.oracle_dequantize_q4(codes, gs)
    scale = np.repeat(gs[..., 0], 128, axis=2)[:, :, :N].astype(np.float64)
    bound = 0.5 * scale * (1 + 1e-5) + np.abs(khat) * 2.0 ** -8
    assert np.all(np.abs(khat - kp) <= bound)
    # a dequantised key is a bf16 value
    np.testing.assert_array_equal(_bf16_values(khat), khat)


def test_q4_constant_group_is_exact():
    kp = np.full((1, 1, 100, 3), 0.3125)
    kp[0, 0, :, 1] = -2.5
    codes, gs = oracle.oracle_quantize_q4(kp)
    assert np.all(codes == 0) and np.all(gs[..., 0] == 0)
    np.testing.assert_array_equal(oracle.oracle_dequantize_q4(codes, gs), kp)


def test_q4_values_on_the_grid_are_exact():
    # values mn + k * s with s = 1/8 and k covering 0..15: the step is s exactly,
    # every value is a grid point, so codes are k and dequantisation is exact
    r = rng(82)
    k = r.integers(0, 16, size=(1, 2, 128, 4))
    k[0, :, 0, :], k[0, :, 1, :] = 0, 15
    kp = -1.0 + k / 8.0
    codes, gs = oracle.oracle_quantize_q4(kp)
    np.testing.assert_array_equal(gs[..., 0], 0.125)
    np.testing.assert_array_equal(codes, k)
    np.testing.assert_array_equal(oracle.oracle_dequantize_q4(codes, gs), kp)


def test_q4_last_group_uses_only_its_tokens():
    # N = 130: the second group holds two tokens, its range is theirs alone
    kp = np.zeros((1, 1, 130, 1))
    kp[0, 0, :128, 0] = np.linspace(-4, 4, 128)
    kp[0, 0, 128:, 0] = [1.0, 2.5]
    kp = _bf16_values(kp)
    codes, gs = oracle.oracle_quantize_q4(kp)
    assert gs.shape == (1, 1, 2, 1, 2)
    assert gs[0, 0, 1, 0, 1] == 1.0 and gs[0, 0, 1, 0, 0] == np.float32(1.5) / np.float32(15)
    assert list(codes[0, 0, 128:, 0]) == [0, 15]


# ----------------------------------------------------- adaptive kept width ---

def test_adaptive_width_hand_worked():
    # scores (3, 4, 0, 0): squared 16 and 9 of E = 25, rank order channel 1, 0
    s = np.array([[[3.0, 4.0, 0.0, 0.0]]])
    for tau, T, idx in [(0.5, 1, [1]), (0.64, 1, [1]), (0.65, 2, [0, 1]), (1.0, 2, [0, 1]), (0.0, 1, [1])]:
        Th, off, ix = oracle.oracle_select_adaptive(s, tau, 1, 4)
        assert Th[0, 0] == T and list(ix) == idx and list(off) == [0, T], (tau, Th, ix)
    # clamps: T_min = 3 keeps the two zero channels by index; T_max = 1 caps
    Th, _, ix = oracle.oracle_select_adaptive(s, 0.5, 3, 4)
    assert Th[0, 0] == 3 and list(ix) == [0, 1, 2]
    Th, _, ix = oracle.oracle_select_adaptive(s, 1.0, 1, 1)
    assert Th[0, 0] == 1 and list(ix) == [1]
    # all-zero scores keep T_min channels, lowest indices first
    Th, _, ix = oracle.oracle_select_adaptive(np.zeros((1, 1, 4)), 0.9, 2, 4)
    assert Th[0, 0] == 2 and list(ix) == [0, 1]


def test_adaptive_width_ragged_offsets_and_monotone_in_tau():
    r = rng(90)
    s = np.abs(r.standard_normal((2, 3, 16))) * r.lognormal(0, 1, (2, 3, 16))
    prev = None
    for tau in (0.0, 0.3, 0.6, 0.9, 0.99, 1.0):
        Th, off, ix = oracle.oracle_select_adaptive(s, tau, 2, 12)
        assert np.all((Th >= 2) & (Th <= 12))
        assert list(off) == [0] + list(np.cumsum(Th.ravel()))
        for bh in range(6):
            seg = ix[off[bh]:off[bh + 1]]
            assert np.all(np.diff(seg) > 0)
            # the kept channels are the top T_h of the ranking
            order = sorted(range(16), key=lambda c: (-s.reshape(6, 16)[bh, c], c))
            assert sorted(order[:Th.ravel()[bh]]) == list(seg)
        if prev is not None:
            assert np.all(Th >= prev)
        prev = Th


def test_adaptive_width_is_the_fewest_channels_within_the_loss_budget():
    # one query head with orthogonal window queries: the squared attention loss
    # of dropping a set of channels is the sum of their squared scores, so the
    # chosen width must be the smallest subset size (over every subset, brute
    # force) whose loss^2 is within (1 - tau) of the total
    r = rng(91)
    d, S, N = 8, 8, 12
    q, _ = np.linalg.qr(r.standard_normal((S, S)))
    q_win = (q[:, :d] * r.lognormal(0, 1, d))[None, None]
    k = r.standard_normal((1, 1, N, d)) * r.lognormal(0, 1, (1, 1, 1, d))
    s = oracle.oracle_score(q_win, k)
    total = oracle.attention_loss(q_win[0, 0], k[0, 0], [])
    for tau in (0.5, 0.8, 0.95):
        Th, _, ix = oracle.oracle_select_adaptive(s, tau, 1, d)
        kept_loss = oracle.attention_loss(q_win[0, 0], k[0, 0], list(ix))
        assert kept_loss ** 2 <= (1 - tau) * total ** 2 * (1 + 1e-9)
        best = min(T for T in range(1, d + 1)
                   if any(oracle.attention_loss(q_win[0, 0], k[0, 0], list(c)) ** 2 <= (1 - tau) * total ** 2 * (1 + 1e-9)
                          for c in itertools.combinations(range(d), T)))
        assert Th[0, 0] == best, (tau, Th, best)


def test_ragged_decode_equals_per_head_pruned_decode():
    r = rng(92)
    B, Hq, Hkv, N, d = 2, 4, 2, 20, 8
    q = r.standard_normal((B, Hq, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    Th = np.array([[3, 5], [8, 1]], dtype=np.int32)
    off = np.array([0, 3, 8, 16, 17], dtype=np.int32)
    idx = np.array([0, 4, 7, 1, 2, 3, 5, 6, 0, 1, 2, 3, 4, 5, 6, 7, 2], dtype=np.int32)
    out = oracle.oracle_decode_ragged(q, k, v, Th, off, idx)
    # head (1, 0) keeps every channel: dense attention for its two query heads
    np.testing.assert_allclose(out[1, 0:2], oracle.oracle_dense_decode(q[1:2, 0:2], k[1:2, 0:1], v[1:2, 0:1])[0],
                               rtol=1e-12, atol=1e-13)
    # head (0, 0): masked-key SDPA with channels {0, 4, 7}
    mask = np.zeros(d)
    mask[[0, 4, 7]] = 1
    np.testing.assert_allclose(out[0, 0:2], _sdpa(q[0:1, 0:2], k[0:1, 0:1] * mask, v[0:1, 0:1], 2)[0],
                               rtol=1e-12, atol=1e-13)


# ------------------------------------------------------- token eviction ---

def test_token_mass_equals_torch_softmax_and_sums_to_rows():
    r = rng(100)
    B, Hq, Hkv, S, N, d = 2, 4, 2, 5, 37, 16
    q_win = r.standard_normal((B, Hq, S, d)) * 2
    k = r.standard_normal((B, Hkv, N, d))
    mass = oracle.oracle_token_mass(q_win, k)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            qg = torch.from_numpy(q_win[b, h * G:(h + 1) * G].reshape(G * S, d))
            p = torch.softmax(qg @ torch.from_numpy(k[b, h]).T / math.sqrt(d), dim=-1)
            np.testing.assert_allclose(mass[b, h], p.sum(0).numpy(), rtol=1e-12, atol=1e-15)
    # every softmax row sums to one: the mass of a head sums to G * S
    np.testing.assert_allclose(mass.sum(-1), G * S, rtol=1e-12)


def test_token_mass_of_equal_keys_is_uniform():
    r = rng(101)
    q_win = r.standard_normal((1, 2, 3, 8))
    k = np.broadcast_to(r.standard_normal(8), (1, 1, 9, 8)).copy()
    np.testing.assert_allclose(oracle.oracle_token_mass(q_win, k), 2 * 3 / 9, rtol=1e-13)


def test_select_tokens_matches_python_sort():
    r = rng(102)
    mass = r.integers(0, 6, size=(2, 3, 40)).astype(np.float64)  # many exact ties
    for M in (1, 7, 40):
        kept = oracle.oracle_select_tokens(mass, M)
        for b in range(2):
            for h in range(3):
                order = sorted(range(40), key=lambda n: (-mass[b, h, n], n))
                assert kept[b, h].tolist() == sorted(order[:M])


def test_keeping_every_token_is_the_plain_prune():
    r = rng(103)
    q_win = r.standard_normal((1, 4, 6, 16))
    k = r.standard_normal((1, 2, 25, 16)) * r.lognormal(0, 1, (1, 1, 1, 16))
    kept, scores, idx, kp = oracle.oracle_evict_and_prune(q_win, k, 25, 6)
    assert np.array_equal(kept, np.broadcast_to(np.arange(25), (1, 2, 25)))
    s2, i2, kp2 = oracle.oracle_prune(q_win, k, 6)
    assert np.array_equal(scores, s2) and np.array_equal(idx, i2) and np.array_equal(kp, kp2)


def test_eviction_keeps_the_attended_token():
    # a key aligned with every window query gets almost all of the mass
    r = rng(104)
    d = 16
    q_win = np.abs(r.standard_normal((1, 2, 4, d)))
    k = 0.01 * r.standard_normal((1, 1, 30, d))
    k[0, 0, 17] = 8.0
    kept = oracle.oracle_select_tokens(oracle.oracle_token_mass(q_win, k), 1)
    assert kept[0, 0, 0] == 17

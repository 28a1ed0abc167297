"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every input comes from the seeded generators in workloads.py;
every expected value comes from the oracle on the same (bf16-rounded) inputs.
Kept channels and the thinner key cache must match bit for bit (near-ties at the
cut excepted, see tests/helpers.py); decode outputs within the stated
tolerances. The full-size workloads run in the same launch configuration as
bench.py (the launch plan depends only on the shape).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import (NEAR_TIE_REL, TOL, check_out, check_scores, f64, idx_mismatch_heads, kp_logical,
                           width_is_near_tie)

pytestmark = pytest.mark.gpu

qdk = pytest.importorskip("query_driven_key_b200")
import workloads as W  # noqa: E402

DEV = "cuda"


def _prune_gpu(q_win, k, T):
    B, Hq, S, d = q_win.shape
    _, Hkv, N, _ = k.shape
    cache = qdk.PrunedCache(B, Hq, Hkv, N, T, d, dtype=k.dtype)
    cache.prune(q_win, k)
    assert qdk.think_read_device_status(cache.score_ws) == 0
    return cache


def _full_path_check(w, q_win, k, v, steps, T=None):
    T = qdk.think_t_from_lambda(w.d, w.lam) if T is None else T
    assert T == oracle.t_from_lambda(w.d, w.lam)
    qd, kd, vd = q_win.to(DEV), k.to(DEV), v.to(DEV)
    cache = _prune_gpu(qd, kd, T)
    torch.cuda.synchronize()
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k), T)
    check_scores(cache.scores, ora_scores, dtype=w.dtype)
    gpu_idx = cache.idx.cpu().numpy()
    ties = idx_mismatch_heads(gpu_idx, ora_idx, ora_scores, T)
    if ties:
        # Near-tie heads: compact and decode again from the oracle's kept set so
        # both sides attend over the same channels.
        cache.idx.copy_(torch.from_numpy(ora_idx))
        qdk.think_compact_keys(kd, cache.idx, cache.k_pruned, cache.ldk)
    assert np.array_equal(kp_logical(cache.k_pruned, w.N), ora_kp), "thinner key cache differs"
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    fv = f64(v)
    for step in steps:
        q = W.gen_decode_q(w, step)
        cache.decode(q.to(DEV), vd, out)
        torch.cuda.synchronize()
        ora = oracle.oracle_decode(f64(q), ora_kp, fv, ora_idx)
        check_out(out, ora, w.dtype, where=f"{w.name} step {step}")
    assert qdk.think_read_device_status(cache.decode_ws) == 0
    return cache


def test_tiny_fp32():
    w = W.WORKLOADS["tiny_fp32"]
    q_win, k, v = W.gen_layer(w)
    _full_path_check(w, q_win, k, v, steps=range(w.decode_steps))


def test_llama2_mha_all_steps():
    w = W.WORKLOADS["llama2_7b_mha"]
    q_win, k, v = W.gen_layer(w)
    _full_path_check(w, q_win, k, v, steps=range(w.decode_steps))


def test_llama3_gqa_lowrank():
    w = W.WORKLOADS["llama3_8b_gqa"]
    q_win, k, v = W.gen_layer(w)
    _full_path_check(w, q_win, k, v, steps=[0, 1, 2])


def test_mistral_long_context():
    # the bench workload, full size: prune + decode steps {0, 1, 2, last}
    w = W.WORKLOADS["mistral_7b_long"]
    q_win, k, v = W.gen_layer(w)
    _full_path_check(w, q_win, k, v, steps=[0, 1, 2, w.decode_steps - 1])


@pytest.mark.parametrize("layer", [0, 31])
def test_sweep_32_layers(layer):
    # Each (B, lambda) of the sweep on one layer; the GPU runs the whole batch,
    # the oracle checks the first and last batch items.
    base = W.WORKLOADS["sweep_32l"]
    for B in W.SWEEP_BATCHES:
        w = base.with_(B=B)
        q_win, k, v = W.gen_layer(w, layer)
        qd, kd, vd = q_win.to(DEV), k.to(DEV), v.to(DEV)
        q = W.gen_decode_q(w, 0, layer)
        for lam in W.SWEEP_LAMBDAS:
            T = qdk.think_t_from_lambda(w.d, lam)
            cache = _prune_gpu(qd, kd, T)
            out = torch.empty((B, w.Hq, w.d), dtype=torch.float32, device=DEV)
            cache.decode(q.to(DEV), vd, out)
            torch.cuda.synchronize()
            gpu_idx = cache.idx.cpu().numpy()
            for b in sorted({0, B - 1}):
                ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win[b:b + 1]), f64(k[b:b + 1]), T)
                check_scores(cache.scores[b:b + 1], ora_scores)
                assert not idx_mismatch_heads(gpu_idx[b:b + 1], ora_idx, ora_scores, T)
                assert np.array_equal(kp_logical(cache.k_pruned[b:b + 1], w.N), ora_kp)
                ora = oracle.oracle_decode(f64(q[b:b + 1]), ora_kp, f64(v[b:b + 1]), ora_idx)
                check_out(out[b:b + 1], ora, w.dtype, where=f"layer {layer} B{B} lam{lam} b{b}")
                if lam == 0.0:
                    assert np.array_equal(ora_idx[0], np.broadcast_to(np.arange(w.d), (w.Hkv, w.d)))
                    assert np.array_equal(kp_logical(cache.k_pruned[b:b + 1], w.N), f64(k[b:b + 1]))
                    dense = oracle.oracle_dense_decode(f64(q[b:b + 1]), f64(k[b:b + 1]), f64(v[b:b + 1]))
                    check_out(out[b:b + 1], dense, w.dtype, where="lambda=0 vs dense")


# ------------------------------------------------------------ edge cases ---

def _random_case(seed, B, Hq, Hkv, N, S, dtype, k_pad=0, v_pad=0):
    g = torch.Generator().manual_seed(seed)
    d = 128
    q_win = torch.randn((B, Hq, S, d), generator=g).to(dtype)
    kbig = torch.randn((B, Hkv, N + k_pad, d), generator=g) * torch.exp(torch.randn((B, Hkv, 1, d), generator=g))
    vbig = torch.randn((B, Hkv, N + v_pad, d), generator=g)
    q = torch.randn((B, Hq, d), generator=g).to(dtype)
    # strided views when padded: the token axis of a bigger buffer
    return q_win, kbig.to(dtype)[:, :, :N], vbig.to(dtype)[:, :, :N], q


EDGE = [
    # (B, Hq, Hkv, N, S, T)
    (1, 1, 1, 1, 1, 1),
    (1, 2, 1, 7, 3, 128),
    (2, 4, 2, 100, 5, 127),
    (1, 8, 1, 129, 4, 51),
    (3, 8, 4, 1000, 8, 77),
    (1, 16, 2, 4097, 16, 64),
    (2, 32, 4, 2049, 32, 1),
    (1, 4, 4, 257, 0, 13),     # empty window: all scores zero, channels 0..T-1 kept
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("case", EDGE)
def test_edge_shapes(case, dtype):
    B, Hq, Hkv, N, S, T = case
    q_win, k, v, q = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, S, dtype, k_pad=8, v_pad=16)
    kd, vd = k.to(DEV), v.to(DEV)
    # keep the strided layout on the device
    kd = torch.empty((B, Hkv, N + 8, 128), dtype=dtype, device=DEV)[:, :, :N].copy_(k)
    vd = torch.empty((B, Hkv, N + 16, 128), dtype=dtype, device=DEV)[:, :, :N].copy_(v)
    cache = _prune_gpu(q_win.to(DEV), kd, T)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
    cache.decode(q.to(DEV), vd, out)
    torch.cuda.synchronize()
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k), T)
    check_scores(cache.scores, ora_scores, dtype=dtype)
    assert not idx_mismatch_heads(cache.idx.cpu().numpy(), ora_idx, ora_scores, T)
    assert np.array_equal(kp_logical(cache.k_pruned, N), ora_kp)
    check_out(out, oracle.oracle_decode(f64(q), ora_kp, f64(v), ora_idx), dtype, where=str(case))
    if S == 0:
        assert np.array_equal(cache.idx.cpu().numpy()[0, 0], np.arange(T))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_growing_cache(dtype):
    # prune on the first N0 tokens, then append new tokens' keys in chunks of
    # odd sizes (unaligned columns included) and decode after every append
    B, Hq, Hkv, N0, S, T = 2, 8, 2, 300, 16, 51
    chunks = [1, 7, 64, 100, 1, 500, 3]
    n_tot = N0 + sum(chunks)
    q_win, k, v, q = _random_case(77, B, Hq, Hkv, n_tot, S, dtype)
    kd, vd, qd = k.to(DEV), v.to(DEV), q.to(DEV)
    cache = qdk.PrunedCache(B, Hq, Hkv, N0, T, dtype=dtype, capacity=n_tot + 5)
    cache.k_pruned.fill_(7.0)
    cache.prune(q_win.to(DEV), kd[:, :, :N0])
    torch.cuda.synchronize()
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k[:, :, :N0]), T)
    if idx_mismatch_heads(cache.idx.cpu().numpy(), ora_idx, ora_scores, T):
        cache.idx.copy_(torch.from_numpy(ora_idx))
        qdk.think_compact_keys(kd[:, :, :N0], cache.idx, cache.k_pruned, cache.ldk)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
    n = N0
    for c in chunks:
        cache.append(kd[:, :, n:n + c])
        ora_kp = oracle.oracle_append(ora_kp, f64(k[:, :, n:n + c]), ora_idx)
        n += c
        assert cache.n == n
        cache.decode(qd, vd, out)
        torch.cuda.synchronize()
        assert np.array_equal(kp_logical(cache.k_pruned, n), ora_kp), f"K' after growing to {n}"
        assert torch.all(cache.k_pruned[..., n:] == 7.0), "columns past the cache length are not written"
        check_out(out, oracle.oracle_decode(f64(q), ora_kp, f64(v[:, :, :n]), ora_idx), dtype,
                  where=f"grown to {n}")
    with pytest.raises(qdk.ThinkError):  # past the capacity of a K' row
        qdk.think_append_keys(kd[:, :, :cache.ldk - n + 1], cache.idx, cache.k_pruned, cache.ldk, n)
    assert qdk.think_read_device_status(cache.decode_ws) == 0


def _q4_codes_logical(cache, N):
    """GPU codes [B,Hkv,T,ldq] (two tokens per byte) -> [B,Hkv,N,T] uint8."""
    c = cache.codes.cpu().numpy()
    both = np.stack([c & 15, c >> 4], axis=-1).reshape(c.shape[:3] + (-1,))[..., :N]
    return np.ascontiguousarray(both.transpose(0, 1, 3, 2))


def _q4_check(cache, q_win, k, v, q, T, where):
    B, Hkv, N, _ = k.shape
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k), T)
    if idx_mismatch_heads(cache.idx.cpu().numpy(), ora_idx, ora_scores, T):
        cache.idx.copy_(torch.from_numpy(ora_idx))
        qdk.think_compact_keys(k.to(DEV), cache.idx, cache.k_pruned, cache.ldk)
    cache.quantize_q4()
    torch.cuda.synchronize()
    codes, gs = oracle.oracle_quantize_q4(ora_kp)
    assert np.array_equal(_q4_codes_logical(cache, N), codes), f"{where}: 4-bit codes differ"
    ng = -(-N // 128)
    gpu_gs = cache.groups[:, :, :ng, :T].cpu().numpy()
    assert np.array_equal(gpu_gs, gs), f"{where}: group parameters differ"
    out = torch.empty((B, q.shape[1], 128), dtype=torch.float32, device=DEV)
    cache.decode_q4(q.to(DEV), v.to(DEV), out)
    torch.cuda.synchronize()
    khat = oracle.oracle_dequantize_q4(codes, gs)
    check_out(out, oracle.oracle_decode(f64(q), khat, f64(v), ora_idx), torch.bfloat16, where=where)
    assert qdk.think_read_device_status(cache.decode_ws) == 0


@pytest.mark.parametrize("case", [(1, 32, 8, 20000, 51), (2, 8, 2, 1000, 64), (1, 4, 4, 130, 13),
                                  (1, 8, 1, 5000, 128), (2, 16, 8, 257, 1), (3, 16, 8, 128, 77)])
def test_q4_thinner_cache(case):
    B, Hq, Hkv, N, T = case
    q_win, k, v, q = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, 16, torch.bfloat16)
    cache = _prune_gpu(q_win.to(DEV), k.to(DEV), T)
    _q4_check(cache, q_win, k, v, q, T, str(case))


@pytest.mark.parametrize("warps", ["4", "8"])
def test_q4_consumer_warp_variants(warps, monkeypatch):
    monkeypatch.setenv("THINK_DECODE_WARPS", warps)
    for case in [(1, 32, 8, 3000, 51), (2, 8, 1, 1000, 128), (1, 16, 8, 300, 1)]:
        B, Hq, Hkv, N, T = case
        q_win, k, v, q = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, 16, torch.bfloat16)
        cache = _prune_gpu(q_win.to(DEV), k.to(DEV), T)
        _q4_check(cache, q_win, k, v, q, T, f"{case} warps={warps}")


def test_q4_long_context_full_size():
    # the bench workload at full size: codes, parameters and one decode step
    w = W.WORKLOADS["mistral_7b_long"]
    T = qdk.think_t_from_lambda(w.d, w.lam)
    q_win, k, v = W.gen_layer(w)
    cache = _prune_gpu(q_win.to(DEV), k.to(DEV), T)
    _q4_check(cache, q_win, k, v, W.gen_decode_q(w, 0), T, "mistral_7b_long q4")


def _adaptive_against_oracle_scores(ora_scores, Th, gidx, rowoff, out, q, kf, vf, tau, T_min, T_max):
    B, Hkv = Th.shape
    oTh, ooff, oidx = oracle.oracle_select_adaptive(ora_scores, tau, T_min, T_max)
    agree = np.zeros((B, Hkv), dtype=bool)
    for bh in range(B * Hkv):
        b, h = divmod(bh, Hkv)
        s = ora_scores[b, h]
        kg, ko = int(Th[b, h]), int(oTh[b, h])
        if kg != ko:
            assert width_is_near_tie(s, tau, T_min, T_max, kg, ko), (
                f"head {bh}: width {kg} on the GPU, {ko} from the oracle's scores, not a near-tie")
            continue
        gi = gidx[rowoff[bh]:rowoff[bh] + kg]
        oi = oidx[ooff[bh]:ooff[bh] + ko]
        if not np.array_equal(gi, oi):
            cut = np.sort(s)[::-1][kg - 1]
            for c in np.setxor1d(gi, oi):
                assert abs(s[c] - cut) <= NEAR_TIE_REL * abs(cut), f"head {bh}: channel {c} not a near-tie"
            continue
        agree[b, h] = True
    assert agree.any() or B * Hkv == 0
    ora_out = oracle.oracle_decode_ragged(f64(q), kf, vf, oTh, ooff, oidx)
    G = out.shape[1] // Hkv
    rows = np.repeat(agree, G, axis=1)  # [B, Hq]: query heads of agreeing KV heads
    g = f64(out)
    if rows.any():
        check_out(torch.from_numpy(g[rows]), ora_out[rows], torch.bfloat16, where="adaptive, oracle scores")


@pytest.mark.parametrize("case", [(1, 32, 8, 20000, 0.9, 16, 96), (2, 8, 2, 1000, 0.5, 1, 128),
                                  (1, 16, 8, 300, 1.0, 8, 64), (2, 32, 32, 257, 0.0, 4, 40),
                                  (1, 8, 8, 2000, 0.8, 33, 33), (3, 8, 1, 129, 0.95, 1, 17)])
def test_adaptive_width(case):
    B, Hq, Hkv, N, tau, T_min, T_max = case
    q_win, k, v, q = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, 16, torch.bfloat16, k_pad=8)
    kd = torch.empty((B, Hkv, N + 8, 128), dtype=torch.bfloat16, device=DEV)[:, :, :N].copy_(k)
    cache = qdk.AdaptiveCache(B, Hq, Hkv, N, tau, T_min, T_max)
    cache.k_pruned.fill_(7.0)
    cache.prune(q_win.to(DEV), kd)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
    cache.decode(q.to(DEV), v.to(DEV), out)
    torch.cuda.synchronize()
    ora_scores = oracle.oracle_score(f64(q_win), f64(k))
    check_scores(cache.scores, ora_scores)
    # the width rule decides on the GPU's scores: the oracle's rule on the same
    # scores must give the same widths and kept channels
    oTh, ooff, oidx = oracle.oracle_select_adaptive(f64(cache.scores), tau, T_min, T_max)
    Th = cache.Th.cpu().numpy().reshape(B, Hkv)
    assert np.array_equal(Th, oTh), (Th, oTh)
    rowoff = cache.rowoff.cpu().numpy()
    assert np.array_equal(rowoff, np.concatenate([[0], np.cumsum((oTh.ravel() + 15) // 16 * 16)]))
    gidx = cache.idx.cpu().numpy()
    kp = cache.k_pruned.cpu()
    kf = f64(k)
    for bh in range(B * Hkv):
        b, h = divmod(bh, Hkv)
        T = int(Th[b, h])
        ih = oidx[ooff[bh]:ooff[bh] + T]
        assert np.array_equal(gidx[rowoff[bh]:rowoff[bh] + T], ih)
        rows = f64(kp[rowoff[bh]:rowoff[bh + 1], :N])
        assert np.array_equal(rows[:T], kf[b, h][:, ih].T), f"K' rows of head {bh}"
        assert np.all(rows[T:] == 0), "pad rows are zero"
    assert torch.all(kp[rowoff[-1]:, :N] == 7.0) if rowoff[-1] < kp.shape[0] else True
    check_out(out, oracle.oracle_decode_ragged(f64(q), kf, f64(v), oTh, ooff, oidx), torch.bfloat16,
              where=str(case))
    assert qdk.think_read_device_status(cache.decode_ws) == 0
    assert qdk.think_read_device_status(cache.score_ws) == 0
    # From the inputs: the oracle's rule on the oracle's own scores.
    _adaptive_against_oracle_scores(ora_scores, Th, gidx, rowoff, out, q, kf, f64(v), tau, T_min, T_max)
    # the one-entry prune (TMA compaction in the ragged layout) gives the
    # outputs of the three separate calls (register compaction) bit for bit
    step = qdk.AdaptiveCache(B, Hq, Hkv, N, tau, T_min, T_max)
    step.k_pruned.fill_(7.0)
    step.prune_stepwise(q_win.to(DEV), kd)
    torch.cuda.synchronize()
    for name in ("scores", "Th", "rowoff"):
        assert torch.equal(getattr(step, name), getattr(cache, name)), name
    sidx = step.idx.cpu().numpy()
    for bh in range(B * Hkv):  # kept entries (a head's pad entries of idx are unspecified)
        T = int(Th.ravel()[bh])
        assert np.array_equal(sidx[rowoff[bh]:rowoff[bh] + T], gidx[rowoff[bh]:rowoff[bh] + T])
    assert torch.equal(step.k_pruned[:, :N], cache.k_pruned[:, :N])


@pytest.mark.parametrize("tc", ["1", "0"])
@pytest.mark.parametrize("case", [(1, 32, 8, 3000, 64), (1, 32, 8, 1300, 50), (2, 16, 8, 777, 48),
                                  (1, 8, 2, 129, 16)])
def test_token_mass_both_kernels(case, tc, monkeypatch):
    # the window attention masses from the tcgen05 kernel (default up to 256
    # window rows: here 256, 200 with padding rows, 96 and 64 rows) and from
    # the mma.sync kernel, against the fp64 oracle; ragged last tiles
    monkeypatch.setenv("THINK_MASS_TC", tc)
    B, Hq, Hkv, N, S = case
    q_win, k, _, _ = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, S, torch.bfloat16)
    mass = torch.full((B, Hkv, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.zeros(qdk.think_token_mass_workspace_size(B, Hq, Hkv, N, S), dtype=torch.uint8, device=DEV)
    for _ in range(2):  # twice on the same workspace
        qdk.think_token_mass(q_win.to(DEV), k.to(DEV), mass, ws)
    torch.cuda.synchronize()
    assert qdk.think_read_device_status(ws) == 0
    ora = oracle.oracle_token_mass(f64(q_win), f64(k))
    np.testing.assert_allclose(f64(mass), ora, rtol=2e-4, atol=1e-6 * (Hq // Hkv) * S)
    np.testing.assert_allclose(f64(mass).sum(axis=-1), (Hq // Hkv) * S, rtol=1e-5)


@pytest.mark.parametrize("case", [(1, 1, 1, 1, "grid"), (1, 3, 4097, 4097, "grid"), (2, 4, 131072, 32768, "grid"),
                                  (1, 2, 70001, 1, "grid"), (1, 1, 5_000_000, 1_000_000, "grid"),
                                  (1, 8, 20000, 6000, "cont"), (3, 2, 9000, 8999, "cont")])
def test_select_tokens_multi_block(case):
    # the chunked radix selection against the oracle's rule on the same masses:
    # coarse-grid masses (many exact ties, zeros included) and continuous ones,
    # N = M, M = 1, chunk boundaries, and more keys per thread than the default
    # (N > 256 * 1024 * 16); a second call checks that the histograms were
    # left at zero
    B, Hkv, N, M, kind = case
    g = torch.Generator().manual_seed(N + M)
    if kind == "grid":
        mass = torch.randint(0, 50, (B, Hkv, N), generator=g).float() * 0.125
    else:
        mass = torch.rand((B, Hkv, N), generator=g) * 3.0
    want = oracle.oracle_select_tokens(mass.double().numpy(), M)
    md = mass.to(DEV)
    ws = torch.zeros(max(256, qdk.think_select_tokens_workspace_size(B, Hkv, N)), dtype=torch.uint8, device=DEV)
    kept = torch.empty((B, Hkv, M), dtype=torch.int32, device=DEV)
    for _ in range(2):
        kept.fill_(-1)
        qdk.think_select_tokens(md, M, kept, ws)
        torch.cuda.synchronize()
        assert np.array_equal(kept.cpu().numpy(), want), case


@pytest.mark.parametrize("case", [(1, 32, 8, 5000, 32, 1000, 51), (2, 8, 2, 1000, 16, 300, 64),
                                  (1, 4, 4, 300, 64, 300, 13), (1, 8, 1, 2049, 64, 129, 128),
                                  (2, 16, 8, 700, 8, 1, 32), (1, 64, 8, 1500, 64, 500, 40)])
def test_token_eviction_then_prune(case):
    B, Hq, Hkv, N, S, M, T = case
    q_win, k, v, q = _random_case(hash(case) & 0xFFFF, B, Hq, Hkv, N, S, torch.bfloat16, k_pad=8)
    kd = torch.empty((B, Hkv, N + 8, 128), dtype=torch.bfloat16, device=DEV)[:, :, :N].copy_(k)
    cache = qdk.EvictedCache(B, Hq, Hkv, N, S, M, T)
    cache.prune(q_win.to(DEV), kd, v.to(DEV))
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
    cache.decode(q.to(DEV), out)
    torch.cuda.synchronize()
    assert qdk.think_read_device_status(cache.mass_ws) == 0
    # masses: fp32 sums of exp2-approximated weights against the fp64 oracle
    ora_mass = oracle.oracle_token_mass(f64(q_win), f64(k))
    gm = f64(cache.mass)
    np.testing.assert_allclose(gm, ora_mass, rtol=2e-4, atol=1e-6 * (Hq // Hkv) * S)
    # the selection on the GPU's masses is the oracle's selection on the same masses
    kept = cache.kept.cpu().numpy()
    assert np.array_equal(kept, oracle.oracle_select_tokens(gm, M))
    # against the oracle's own masses it may differ only at near-ties of the cut
    ora_kept = oracle.oracle_select_tokens(ora_mass, M)
    for b in range(B):
        for h in range(Hkv):
            diff = set(kept[b, h]) ^ set(ora_kept[b, h])
            if diff:
                cut = np.sort(ora_mass[b, h])[::-1][M - 1]
                assert all(abs(ora_mass[b, h, n] - cut) <= 5e-4 * cut for n in diff), (b, h, diff)
    # gathers are exact copies; the prune and decode run on the kept tokens
    kk = oracle.oracle_gather_tokens(f64(k), kept)
    assert np.array_equal(f64(cache.k_kept), kk)
    assert np.array_equal(f64(cache.v_kept), oracle.oracle_gather_tokens(f64(v), kept))
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), kk, T)
    check_scores(cache.pruned.scores, ora_scores)
    if idx_mismatch_heads(cache.pruned.idx.cpu().numpy(), ora_idx, ora_scores, T):
        cache.pruned.idx.copy_(torch.from_numpy(ora_idx))
        qdk.think_compact_keys(cache.k_kept, cache.pruned.idx, cache.pruned.k_pruned, cache.pruned.ldk)
        cache.decode(q.to(DEV), out)
        torch.cuda.synchronize()
    assert np.array_equal(kp_logical(cache.pruned.k_pruned, M), ora_kp)
    check_out(out, oracle.oracle_decode(f64(q), ora_kp, oracle.oracle_gather_tokens(f64(v), kept), ora_idx),
              torch.bfloat16, where=str(case))


def test_ldk_larger_than_needed_and_exact_ties():
    # duplicate channels give exact score ties: lower index must win on both sides
    B, Hq, Hkv, N, S, T = 1, 4, 2, 300, 6, 40
    q_win, k, v, q = _random_case(5, B, Hq, Hkv, N, S, torch.bfloat16)
    k[..., 64:96] = k[..., 0:32]
    q_win[..., 64:96] = q_win[..., 0:32]
    kd = k.contiguous().to(DEV)
    ldk = 512
    scores = torch.empty((B, Hkv, 128), dtype=torch.float64, device=DEV)
    ws = torch.zeros(qdk.think_score_workspace_size(B, Hq, Hkv, N), dtype=torch.uint8, device=DEV)
    idx = torch.empty((B, Hkv, T), dtype=torch.int32, device=DEV)
    kp = torch.full((B, Hkv, T, ldk), 7.0, dtype=torch.bfloat16, device=DEV)
    qdk.think_score_channels(q_win.to(DEV), kd, scores, ws)
    qdk.think_select_channels(scores, T, idx)
    qdk.think_compact_keys(kd, idx, kp, ldk)
    torch.cuda.synchronize()
    s, oi, okp = oracle.oracle_prune(f64(q_win), f64(k), T)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.array_equal(kp_logical(kp, N), okp)
    assert torch.all(kp[..., N:] == 7.0), "columns beyond N must not be written"


def test_fused_prune_equals_stepwise_calls():
    w = W.WORKLOADS["llama3_8b_gqa"].with_(B=2, N=5000)
    q_win, k, _ = W.gen_layer(w)
    qd, kd = q_win.to(DEV), k.to(DEV)
    a = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, 64, dtype=k.dtype)
    b = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, 64, dtype=k.dtype)
    a.prune(qd, kd)
    b.prune_stepwise(qd, kd)
    torch.cuda.synchronize()
    assert torch.equal(a.scores, b.scores)
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.k_pruned[..., : w.N], b.k_pruned[..., : w.N])
    # counters are left at zero: a second call gives the same result
    a.prune(qd, kd)
    torch.cuda.synchronize()
    assert torch.equal(a.idx, b.idx)


PRUNE_ENV_KEYS = ("THINK_PRUNE_FUSED", "THINK_PRUNE_STAGES", "THINK_PRUNE_CSTAGES", "THINK_PRUNE_HINTS",
                  "THINK_PRUNE_LAG", "THINK_PRUNE_PREFETCH", "THINK_SCORE_PLAN_ROUNDS",
                  "THINK_SCORE_TMA", "THINK_SCORE_STAGES", "THINK_COMPACT_TMA", "THINK_COMPACT_STAGES",
                  "THINK_COMPACT_TILES")


FUSED = {"THINK_PRUNE_FUSED": "1", "THINK_SCORE_PLAN_ROUNDS": "1"}


@pytest.mark.parametrize("env", [FUSED,
                                 dict(FUSED, THINK_PRUNE_STAGES="2", THINK_PRUNE_CSTAGES="2"),
                                 dict(FUSED, THINK_PRUNE_STAGES="10", THINK_PRUNE_CSTAGES="2"),
                                 dict(FUSED, THINK_PRUNE_STAGES="3", THINK_PRUNE_CSTAGES="5", THINK_PRUNE_LAG="1"),
                                 dict(FUSED, THINK_PRUNE_HINTS="0", THINK_PRUNE_LAG="5"),
                                 dict(FUSED, THINK_PRUNE_HINTS="7", THINK_PRUNE_PREFETCH="8"),
                                 {"THINK_SCORE_PLAN_ROUNDS": "1", "THINK_SCORE_TMA": "0"},
                                 {"THINK_SCORE_TMA": "0"},
                                 {"THINK_SCORE_STAGES": "2"},
                                 {"THINK_SCORE_STAGES": "8"},
                                 {"THINK_COMPACT_TMA": "0"},
                                 {"THINK_COMPACT_STAGES": "2", "THINK_COMPACT_TILES": "1"},
                                 {"THINK_COMPACT_STAGES": "8", "THINK_COMPACT_TILES": "37"}])
def test_prune_schedules_give_identical_results(env, monkeypatch):
    # the default two-launch prune (TMA-staged score and compaction tiles)
    # against the register-pipelined score and compaction kernels, other ring
    # depths and run lengths, and -- on the round split plan, which the
    # one-kernel prune needs -- the one-kernel prune (which compacts each round
    # of heads from L2 while it scores the next; several ring depths, lags, L2
    # hints and prefetch distances): bit for bit the same for the same split
    # plan (same order of additions, pure copies).  Shapes: one round, several
    # rounds of one and of several heads (two runs per block), a head too long
    # for the one-kernel prune (two launches on both sides)
    shapes = [(2, 32, 8, 5000, 64), (1, 8, 1, 70, 51), (4, 4, 4, 3000, 128), (3, 16, 8, 1, 1),
              (1, 32, 8, 40000, 51), (2, 32, 8, 60000, 51), (1, 8, 2, 200000, 40)]
    for i, (B, Hq, Hkv, N, T) in enumerate(shapes):
        q_win, k, _, _ = _random_case(100 + i, B, Hq, Hkv, N, 32, torch.bfloat16, k_pad=8)
        kd = torch.empty((B, Hkv, N + 8, 128), dtype=torch.bfloat16, device=DEV)[:, :, :N].copy_(k)
        qd = q_win.to(DEV)
        for key in PRUNE_ENV_KEYS:
            monkeypatch.delenv(key, raising=False)
        if "THINK_SCORE_PLAN_ROUNDS" in env:  # the reference uses the same split plan
            monkeypatch.setenv("THINK_SCORE_PLAN_ROUNDS", env["THINK_SCORE_PLAN_ROUNDS"])
        a = _prune_gpu(qd, kd, T)
        for key, val in env.items():
            monkeypatch.setenv(key, val)
        b = _prune_gpu(qd, kd, T)
        b.prune(qd, kd)  # a second call on the same workspace: counters and flags were reset
        torch.cuda.synchronize()
        assert qdk.think_read_device_status(b.score_ws) == 0
        assert torch.equal(a.scores, b.scores), (env, B, Hq, Hkv, N, T)
        assert torch.equal(a.idx, b.idx)
        assert torch.equal(a.k_pruned[..., :N], b.k_pruned[..., :N])
        ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k), T)
        check_scores(a.scores, ora_scores)
        assert not idx_mismatch_heads(a.idx.cpu().numpy(), ora_idx, ora_scores, T)
        assert np.array_equal(kp_logical(a.k_pruned, N), ora_kp)


def test_one_workspace_serves_every_shape(monkeypatch):
    # One score workspace and one decode workspace, sized for the largest
    # shape, serve prunes (both prune paths, whose split plans differ) and
    # decodes of several shapes in turn.  The arrival counters of each call sit
    # where the previous call left scratch values; every call must still give
    # the results of a fresh workspace, with a clear status.
    shapes = [(1, 32, 8, 40000, 51), (2, 16, 8, 3000, 64), (1, 8, 2, 60000, 40), (1, 32, 8, 40000, 51)]
    s_bytes = max(qdk.think_score_workspace_size(B, Hq, Hkv, N) for B, Hq, Hkv, N, _ in shapes)
    d_bytes = max(qdk.think_decode_workspace_size(B, Hq, Hkv, N) for B, Hq, Hkv, N, _ in shapes)
    sws = torch.empty(s_bytes, dtype=torch.uint8, device=DEV)
    dws = torch.empty(d_bytes, dtype=torch.uint8, device=DEV)
    qdk.think_workspace_init(sws)
    qdk.think_workspace_init(dws)
    for i, (B, Hq, Hkv, N, T) in enumerate(shapes):
        q_win, k, v, q = _random_case(300 + i, B, Hq, Hkv, N, 32, torch.bfloat16)
        qd, kd, vd, qq = q_win.to(DEV), k.to(DEV), v.to(DEV), q.to(DEV)
        for fused in ("0", "1"):
            monkeypatch.setenv("THINK_PRUNE_FUSED", fused)
            fresh = _prune_gpu(qd, kd, T)
            ref = torch.empty((B, Hq, 128), dtype=torch.float32, device=DEV)
            fresh.decode(qq, vd, ref)
            scores = torch.empty_like(fresh.scores)
            idx = torch.empty_like(fresh.idx)
            kp = torch.empty_like(fresh.k_pruned)
            qdk.think_prune(qd, kd, T, scores, idx, kp, fresh.ldk, sws)
            out = torch.empty_like(ref)
            qdk.think_pruned_decode_attn(qq, kp, fresh.ldk, vd, idx, out, dws)
            torch.cuda.synchronize()
            assert qdk.think_read_device_status(sws) == 0 and qdk.think_read_device_status(dws) == 0
            where = (B, Hq, Hkv, N, T, fused)
            assert torch.equal(scores, fresh.scores) and torch.equal(idx, fresh.idx), where
            assert torch.equal(kp[..., :N], fresh.k_pruned[..., :N]), where
            assert torch.equal(out, ref), where
    monkeypatch.delenv("THINK_PRUNE_FUSED")


@pytest.mark.parametrize("kernel", ["warp_mma", "warp_mma_8_warps", "cuda_cores", "tensor_cores"])
def test_every_bf16_decode_kernel(kernel, monkeypatch):
    # the bf16 decode kernels on the same inputs: warp-level mma (default; four
    # and eight consumer warps), CUDA cores, tcgen05
    for key in ("THINK_DECODE_TENSOR_CORES", "THINK_DECODE_CUDA_CORES", "THINK_DECODE_WARPS"):
        monkeypatch.delenv(key, raising=False)
    if kernel == "tensor_cores":
        monkeypatch.setenv("THINK_DECODE_TENSOR_CORES", "1")
    elif kernel == "cuda_cores":
        monkeypatch.setenv("THINK_DECODE_CUDA_CORES", "1")
    elif kernel == "warp_mma_8_warps":
        monkeypatch.setenv("THINK_DECODE_WARPS", "8")
    w = W.WORKLOADS["mistral_7b_long"].with_(N=20000)
    q_win, k, v = W.gen_layer(w)
    _full_path_check(w, q_win, k, v, steps=[0, 1])
    for G, Hq in [(1, 8), (2, 16), (8, 64)]:
        wg = w.with_(Hq=Hq, N=3000)
        q_win, k, v = W.gen_layer(wg)
        _full_path_check(wg, q_win, k, v, steps=[0])


# (B, Hq, Hkv, N): the 32-layer sweep's layer (8 heads of 64 tiles), the
# llama2-shaped MHA layer (32 heads of 32 tiles), 9 tiles (clusters of up to
# 16 with empty splits), 3 tiles with a ragged tail (16 heads: clusters of 4,
# which are always resident).  Whether the first three use clusters depends
# on how many clusters of a size the device keeps resident.
CLUSTER_SHAPES = [(1, 32, 8, 8192), (1, 32, 32, 4096), (1, 64, 8, 1100), (2, 16, 8, 300)]


@pytest.mark.parametrize("warps", ["4", "8"])
@pytest.mark.parametrize("shape", CLUSTER_SHAPES)
def test_cluster_split_merge(shape, warps, monkeypatch):
    # The warp-MMA decode merges a short head's splits inside a thread-block
    # cluster (distributed shared memory): every cluster size cap gives the
    # oracle's output within tolerance, and the capped-off global merge (cap 0)
    # too.  With clusters on, the workspace's split partials stay untouched.
    for key in ("THINK_DECODE_TENSOR_CORES", "THINK_DECODE_CUDA_CORES"):
        monkeypatch.delenv(key, raising=False)
    monkeypatch.setenv("THINK_DECODE_WARPS", warps)
    B, Hq, Hkv, N = shape
    w = W.WORKLOADS["sweep_32l"].with_(B=B, Hq=Hq, Hkv=Hkv, N=N, layers=1)
    q_win, k, v = W.gen_layer(w)
    T = qdk.think_t_from_lambda(w.d, w.lam)
    ora_scores, ora_idx, ora_kp = oracle.oracle_prune(f64(q_win), f64(k), T)
    cache = _prune_gpu(q_win.to(DEV), k.to(DEV), T)
    cache.idx.copy_(torch.from_numpy(ora_idx))
    qdk.think_compact_keys(k.to(DEV), cache.idx, cache.k_pruned, cache.ldk)
    q = W.gen_decode_q(w, 0)
    ora = oracle.oracle_decode(f64(q), ora_kp, f64(v), ora_idx)
    vd, qd = v.to(DEV), q.to(DEV)
    heads = B * Hkv
    part0 = 256 + (heads * 4 + 255) // 256 * 256  # status header, tickets, then the partials
    outs = {}
    for cap in ["0", "2", "4", "8", "16"]:
        monkeypatch.setenv("THINK_DECODE_CLUSTER", cap)
        ws = torch.empty(qdk.think_decode_workspace_size(B, Hq, Hkv, N), dtype=torch.uint8, device=DEV)
        qdk.think_workspace_init(ws)
        ws[part0:].fill_(0xA5)
        out = torch.full((B, Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
        for _ in range(2):  # the same workspace twice
            qdk.think_pruned_decode_attn(qd, cache.k_pruned, cache.ldk, vd, cache.idx, out, ws)
        torch.cuda.synchronize()
        assert qdk.think_read_device_status(ws) == 0
        check_out(out, ora, w.dtype, where=f"cluster cap {cap}")
        untouched = bool(torch.all(ws[part0:] == 0xA5))
        if cap == "0":
            assert not untouched, "the global merge writes split partials"
        elif cap in ("4", "16") and shape == (2, 16, 8, 300):
            assert untouched, "a clustered decode writes no split partials"
        outs[cap] = out.clone()
    monkeypatch.delenv("THINK_DECODE_CLUSTER")


def test_scores_are_deterministic():
    w = W.WORKLOADS["llama2_7b_mha"]
    q_win, k, _ = W.gen_slice(w, 0, 0)
    qd, kd = q_win[None].to(DEV), k[None].to(DEV)
    a = _prune_gpu(qd, kd, 77)
    b = _prune_gpu(qd, kd, 77)
    torch.cuda.synchronize()
    assert torch.equal(a.scores, b.scores)
    assert torch.equal(a.idx, b.idx)


# ------------------------------------------------------------ validation ---

def test_host_validation_errors_launch_nothing():
    B, Hq, Hkv, N = 1, 4, 2, 64
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device=DEV)
    v = torch.zeros((B, Hkv, N, 128), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((B, Hkv, 4), dtype=torch.int32, device=DEV)
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device=DEV)
    kp = torch.zeros((B, Hkv, 4, 64), dtype=torch.bfloat16, device=DEV)
    ws_n = qdk.think_decode_workspace_size(B, Hq, Hkv, N)
    ws = torch.zeros(ws_n, dtype=torch.uint8, device=DEV)
    with pytest.raises(qdk.ThinkError) as e:
        qdk.think_pruned_decode_attn(q, kp, 64, v, idx, out, ws[: ws_n - 16])
    assert e.value.code == qdk.THINK_ERR_WORKSPACE
    with pytest.raises(qdk.ThinkError) as e:
        qdk.think_pruned_decode_attn(q, kp, 60, v, idx, out, ws)   # pitch not 16-byte multiple
    assert e.value.code in (qdk.THINK_ERR_ALIGNMENT, qdk.THINK_ERR_INVALID_ARG)
    q3 = torch.zeros((B, 6, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qdk.ThinkError) as e:
        qdk.think_pruned_decode_attn(q3, kp, 64, v, idx, torch.zeros((B, 6, 128), device=DEV),
                                     torch.zeros(1 << 20, dtype=torch.uint8, device=DEV))
    assert e.value.code == qdk.THINK_ERR_UNSUPPORTED          # group of 3
    torch.cuda.synchronize()
    assert torch.all(out == 0)

"""GPU integration: the calls inside a captured CUDA graph, concurrent calls on
two streams, and the later pipelines at many heads.  Inputs come from the
seeded generators; expected values from the eager calls (bit-identical: every
kernel adds in a fixed order) or from the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import check_out, f64, idx_mismatch_heads

pytestmark = pytest.mark.gpu

qdk = pytest.importorskip("query_driven_key_b200")
import workloads as W  # noqa: E402

DEV = "cuda"


def _layer(name, **kw):
    w = W.WORKLOADS[name].with_(**kw)
    q_win, k, v = W.gen_layer(w)
    return w, q_win.to(DEV), k.to(DEV), v.to(DEV)


def test_prune_and_decode_inside_a_cuda_graph():
    w, qd, kd, vd = _layer("mistral_7b_long", N=5000)
    T = qdk.think_t_from_lambda(w.d, w.lam)
    qs = [W.gen_decode_q(w, s).to(DEV) for s in range(3)]
    eager = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, T)
    eager.prune(qd, kd)
    ref = []
    for q in qs:
        o = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
        eager.decode(q, vd, o)
        ref.append(o)
    torch.cuda.synchronize()

    cache = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, T)
    outs = [torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV) for _ in qs]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        cache.prune(qd, kd)
        for q, o in zip(qs, outs):
            cache.decode(q, vd, o)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cache.prune(qd, kd)
        for q, o in zip(qs, outs):
            cache.decode(q, vd, o)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(cache.idx, eager.idx) and torch.equal(cache.scores, eager.scores)
    for o, r in zip(outs, ref):
        assert torch.equal(o, r)
    assert qdk.think_read_device_status(cache.decode_ws) == 0


def test_two_streams_at_once():
    # two layers with their own caches, decoded alternately on two streams
    w1, q1, k1, v1 = _layer("llama3_8b_gqa", B=2, N=6000)
    w2, q2, k2, v2 = _layer("mistral_7b_long", N=9000)
    T1 = qdk.think_t_from_lambda(w1.d, w1.lam)
    T2 = qdk.think_t_from_lambda(w2.d, w2.lam)
    c1 = qdk.PrunedCache(w1.B, w1.Hq, w1.Hkv, w1.N, T1)
    c2 = qdk.PrunedCache(w2.B, w2.Hq, w2.Hkv, w2.N, T2)
    qa = [W.gen_decode_q(w1, s).to(DEV) for s in range(4)]
    qb = [W.gen_decode_q(w2, s).to(DEV) for s in range(4)]
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    o1 = [torch.empty((w1.B, w1.Hq, 128), dtype=torch.float32, device=DEV) for _ in qa]
    o2 = [torch.empty((w2.B, w2.Hq, 128), dtype=torch.float32, device=DEV) for _ in qb]
    torch.cuda.synchronize()
    c1.prune(q1, k1, stream=s1)
    c2.prune(q2, k2, stream=s2)
    for i in range(4):
        c1.decode(qa[i], v1, o1[i], stream=s1)
        c2.decode(qb[i], v2, o2[i], stream=s2)
    torch.cuda.synchronize()
    # the same calls one after the other on the default stream
    for c, qw, kk, vv, qs, outs, w in ((c1, q1, k1, v1, qa, o1, w1), (c2, q2, k2, v2, qb, o2, w2)):
        ref = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, c.T)
        ref.prune(qw, kk)
        for q, o in zip(qs, outs):
            r = torch.empty_like(o)
            ref.decode(q, vv, r)
            torch.cuda.synchronize()
            assert torch.equal(o, r)
    assert qdk.think_read_device_status(c1.decode_ws) == 0 and qdk.think_read_device_status(c2.decode_ws) == 0


def test_adaptive_width_at_256_heads():
    w, qd, kd, vd = _layer("sweep_32l", B=32, N=2000)
    cache = qdk.AdaptiveCache(w.B, w.Hq, w.Hkv, w.N, 0.9, 4, 96)
    cache.prune(qd, kd)
    q = W.gen_decode_q(w, 0).to(DEV)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=DEV)
    cache.decode(q, vd, out)
    torch.cuda.synchronize()
    oTh, ooff, oidx = oracle.oracle_select_adaptive(f64(cache.scores), 0.9, 4, 96)
    assert np.array_equal(cache.Th.cpu().numpy().reshape(w.B, w.Hkv), oTh)
    # decode of the first and last batch items against the oracle
    for b in (0, w.B - 1):
        sl = slice(b * w.Hkv, (b + 1) * w.Hkv)
        ooff_b = ooff[sl.start:sl.stop + 1] - ooff[sl.start]
        ora = oracle.oracle_decode_ragged(f64(q[b:b + 1]), f64(kd[b:b + 1]), f64(vd[b:b + 1]), oTh[b:b + 1],
                                          ooff_b, oidx[ooff[sl.start]:ooff[sl.stop]])
        check_out(out[b:b + 1], ora, torch.bfloat16, where=f"adaptive b={b}")


def test_eviction_at_128_heads():
    w, qd, kd, vd = _layer("sweep_32l", B=16, N=3000, S_obs=16)
    M, T = 700, 51
    cache = qdk.EvictedCache(w.B, w.Hq, w.Hkv, w.N, w.S_obs, M, T)
    cache.prune(qd, kd, vd)
    torch.cuda.synchronize()
    gm = f64(cache.mass)
    kept = cache.kept.cpu().numpy()
    assert np.array_equal(kept, oracle.oracle_select_tokens(gm, M))
    np.testing.assert_allclose(gm.sum(-1), (w.Hq // w.Hkv) * w.S_obs, rtol=1e-4)
    for b in (0, w.B - 1):
        ora_mass = oracle.oracle_token_mass(f64(qd[b:b + 1]), f64(kd[b:b + 1]))
        np.testing.assert_allclose(gm[b:b + 1], ora_mass, rtol=2e-4, atol=1e-6 * (w.Hq // w.Hkv) * w.S_obs)
        kk = oracle.oracle_gather_tokens(f64(kd[b:b + 1]), kept[b:b + 1])
        assert np.array_equal(f64(cache.k_kept[b:b + 1]), kk)
        s, i, _ = oracle.oracle_prune(f64(qd[b:b + 1]), kk, T)
        assert not idx_mismatch_heads(cache.pruned.idx[b:b + 1].cpu().numpy(), i, s, T)

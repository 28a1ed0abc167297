"""The decode entry point that allocates nothing, against the workspace form.

think_pruned_decode_attn_noalloc serves callers that may not allocate device
memory (a host framework that owns the device-memory budget, or a
latency-critical path where an allocation could synchronise the device): it
runs the same decode with the library's built-in scratch array instead of a
caller workspace. Two calls in a row are compared with the workspace form
through the C ABI: the same kernel with the same split plan, so the outputs
must be equal bit for bit, and the device status word read back from the
array must be zero after each call. This file
sorts last so that a run stopping at the first failure has run everything
else first; it also passes on its own in a fresh process.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

qdk = pytest.importorskip("query_driven_key_b200")
import workloads as W  # noqa: E402


@pytest.mark.parametrize("name,N", [("mistral_7b_long", 20000), ("llama2_7b_mha", 4096)])
def test_noalloc_decode_matches_workspace_decode(name, N):
    w = W.WORKLOADS[name].with_(N=N)
    T = qdk.think_t_from_lambda(w.d, w.lam)
    q_win, k, v = W.gen_layer(w)
    dev = "cuda"
    cache = qdk.PrunedCache(w.B, w.Hq, w.Hkv, w.N, T, w.d, dtype=w.dtype, device=dev)
    cache.prune(q_win.to(dev), k.to(dev))
    vd = v.to(dev)
    assert qdk.think_decode_workspace_size(w.B, w.Hq, w.Hkv, w.N) <= qdk.lib.think_noalloc_scratch_bytes()
    for step in (0, 1):  # two calls in a row share the built-in scratch
        q = W.gen_decode_q(w, step).to(dev)
        ref = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
        got = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=dev)
        cache.decode(q, vd, ref)
        qdk.think_pruned_decode_attn_noalloc(q, cache.k_pruned, cache.ldk, vd, cache.idx, got, N=w.N)
        assert qdk.think_noalloc_read_device_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (step, (got - ref).abs().max().item())


def test_noalloc_rejects_a_problem_larger_than_its_scratch():
    B, Hq, Hkv, N = 130, 64, 8, 1000   # 1040 KV heads x 8 query heads: over 4 MiB of partials
    assert qdk.think_decode_workspace_size(B, Hq, Hkv, N) > qdk.lib.think_noalloc_scratch_bytes()
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((B, Hkv, N, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((B, Hkv, 4), dtype=torch.int32, device="cuda")
    kp = torch.zeros((B, Hkv, 4, 1008), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(qdk.ThinkError) as e:
        qdk.think_pruned_decode_attn_noalloc(q, kp, 1008, v, idx, out, N=N)
    assert e.value.code == qdk.THINK_ERR_WORKSPACE

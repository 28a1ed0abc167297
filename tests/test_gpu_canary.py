"""Out-of-bounds write checks with canary regions (the device memory checker is
not available on the GPUs these tests run on).

Every output buffer and workspace of a call is carved from a larger device
buffer whose tail (and, for the thinner key cache, the token columns past N
and the rows past the last head) holds a byte pattern; after the call the
pattern must be intact.  Small odd shapes put ragged tiles at the edges.
"""
import os

import pytest
import torch

pytestmark = pytest.mark.gpu

qdk = pytest.importorskip("query_driven_key_b200")
if os.environ.get("THINK_DEBUG_LIB") == "1":
    assert qdk.LIB_PATH.endswith("libthink_debug.so"), qdk.LIB_PATH

DEV = "cuda"
PAT = 0xA5
PAD = 4096  # canary bytes after each buffer


class Canary:
    """A device tensor of `shape` carved from the front of a byte buffer whose
    last PAD bytes hold the pattern."""

    def __init__(self, shape, dtype, fill=None):
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((self.nbytes + PAD,), PAT, dtype=torch.uint8, device=DEV)
        self.t = self.raw[: self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self):
        return bool(torch.all(self.raw[self.nbytes:] == PAT))


def _ws(nbytes):
    c = Canary((max(256, nbytes),), torch.uint8)
    qdk.think_workspace_init(c.t)
    return c


def _inputs(B, Hq, Hkv, N, S, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q_win = torch.randn((B, Hq, S, 128), generator=g).to(dtype).to(DEV)
    k = (torch.randn((B, Hkv, N, 128), generator=g) *
         torch.exp(torch.randn((B, Hkv, 1, 128), generator=g))).to(dtype).to(DEV)
    v = torch.randn((B, Hkv, N, 128), generator=g).to(dtype).to(DEV)
    q = torch.randn((B, Hq, 128), generator=g).to(dtype).to(DEV)
    return q_win, k, v, q


SHAPES = [(2, 8, 2, 1000, 5, 51), (1, 4, 4, 129, 3, 128), (3, 16, 2, 70, 1, 1)]


@pytest.mark.parametrize("fused", ["0", "1"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", SHAPES)
def test_prune_and_decode_stay_in_bounds(shape, dtype, fused, monkeypatch):
    if fused == "1" and dtype != torch.bfloat16:
        pytest.skip("the one-kernel prune is bf16 only")
    monkeypatch.setenv("THINK_PRUNE_FUSED", fused)
    B, Hq, Hkv, N, S, T = shape
    q_win, k, v, q = _inputs(B, Hq, Hkv, N, S, dtype, hash(shape) & 0xFFFF)
    ldk = qdk.think_pruned_ld(N + 40, dtype)          # room past N: must stay untouched
    scores = Canary((B, Hkv, 128), torch.float64)
    idx = Canary((B, Hkv, T), torch.int32)
    kp = Canary((B, Hkv, T, ldk), dtype, fill=7.0)
    sws = _ws(qdk.think_score_workspace_size(B, Hq, Hkv, N))
    for _ in range(2):  # a second call on the same workspace
        qdk.think_prune(q_win, k, T, scores.t, idx.t, kp.t, ldk, sws.t)
    out = Canary((B, Hq, 128), torch.float32)
    dws = _ws(qdk.think_decode_workspace_size(B, Hq, Hkv, N, dtype=dtype))
    for _ in range(2):
        qdk.think_pruned_decode_attn(q, kp.t, ldk, v, idx.t, out.t, dws.t)
    torch.cuda.synchronize()
    assert qdk.think_read_device_status(sws.t) == 0 and qdk.think_read_device_status(dws.t) == 0
    for name, c in [("scores", scores), ("idx", idx), ("K'", kp), ("score ws", sws), ("out", out),
                    ("decode ws", dws)]:
        assert c.intact(), name
    assert torch.all(kp.t[..., N:] == 7.0), "K' columns past N"
    assert torch.isfinite(out.t).all()


@pytest.mark.parametrize("shape", SHAPES[:2])
def test_append_q4_adaptive_and_eviction_stay_in_bounds(shape):
    B, Hq, Hkv, N, S, T = shape
    dtype = torch.bfloat16
    q_win, k, v, q = _inputs(B, Hq, Hkv, N, S, dtype, 7 + N)
    # growing cache: append 37 tokens after a prune of N - 37
    n0 = N - 37
    cap = qdk.think_pruned_ld(N, dtype)
    idx = Canary((B, Hkv, T), torch.int32)
    scores = Canary((B, Hkv, 128), torch.float64)
    kp = Canary((B, Hkv, T, cap), dtype, fill=3.0)
    sws = _ws(qdk.think_score_workspace_size(B, Hq, Hkv, n0))
    qdk.think_prune(q_win, k[:, :, :n0], T, scores.t, idx.t, kp.t, cap, sws.t)
    qdk.think_append_keys(k[:, :, n0:], idx.t, kp.t, cap, n0)
    # 4-bit thinner cache and its decode
    ldq = qdk.think_q4_ld(N)
    codes = Canary((B, Hkv, T, ldq), torch.uint8)
    groups = Canary((qdk.think_q4_groups_bytes(B, Hkv, N, T) // 4,), torch.float32)
    qdk.think_quantize_keys_q4(kp.t, cap, N, codes.t, ldq, groups.t)
    out = Canary((B, Hq, 128), torch.float32)
    dws = _ws(qdk.think_decode_workspace_size(B, Hq, Hkv, N))
    qdk.think_pruned_decode_attn_q4(q, codes.t, ldq, groups.t, v, idx.t, out.t, dws.t, N=N)
    # adaptive kept width per head
    rows = qdk.think_ragged_rows(B, Hkv, 96)
    a_scores = Canary((B, Hkv, 128), torch.float64)
    Th = Canary((B * Hkv,), torch.int32)
    rowoff = Canary((B * Hkv + 1,), torch.int32)
    a_idx = Canary((rows,), torch.int32)
    a_kp = Canary((rows, cap), dtype, fill=5.0)
    a_ws = _ws(qdk.think_score_workspace_size(B, Hq, Hkv, N))
    qdk.think_prune_adaptive(q_win, k, 0.9, 4, 96, a_scores.t, Th.t, rowoff.t, a_idx.t, a_kp.t, cap, a_ws.t)
    a_out = Canary((B, Hq, 128), torch.float32)
    a_dws = _ws(qdk.think_decode_workspace_size(B, Hq, Hkv, N))
    qdk.think_pruned_decode_attn_ragged(q, a_kp.t, cap, v, a_idx.t, Th.t, rowoff.t, 96, a_out.t, a_dws.t)
    # token eviction: masses, kept tokens, gathered rows
    M = max(1, N // 3)
    mass = Canary((B, Hkv, N), torch.float32)
    mws = _ws(qdk.think_token_mass_workspace_size(B, Hq, Hkv, N, S))
    qdk.think_token_mass(q_win, k, mass.t, mws.t)
    kept = Canary((B, Hkv, M), torch.int32)
    tws = _ws(qdk.think_select_tokens_workspace_size(B, Hkv, N))
    qdk.think_select_tokens(mass.t, M, kept.t, tws.t)
    kk = Canary((B, Hkv, M, 128), dtype)
    qdk.think_gather_tokens(k, kept.t, kk.t)
    torch.cuda.synchronize()
    for ws in (sws, dws, a_ws, a_dws, mws):
        assert qdk.think_read_device_status(ws.t) == 0
    for name, c in [("idx", idx), ("scores", scores), ("K'", kp), ("codes", codes), ("groups", groups),
                    ("q4 out", out), ("q4 ws", dws), ("adaptive scores", a_scores), ("Th", Th),
                    ("rowoff", rowoff), ("adaptive idx", a_idx), ("ragged K'", a_kp), ("adaptive ws", a_ws),
                    ("ragged out", a_out), ("ragged ws", a_dws), ("mass", mass), ("mass ws", mws),
                    ("kept", kept), ("select ws", tws), ("gathered K", kk)]:
        assert c.intact(), name

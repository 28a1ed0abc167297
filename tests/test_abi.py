"""CPU checks of the C ABI: the library loads, exports every entry point the
header declares, and its host-side logic (T rule, pitch, workspace sizes,
argument validation) behaves as documented. No kernel is launched here: every
call below is rejected by host validation before any CUDA call, or is a pure
host function."""
import ctypes
import os
import re

import pytest

import oracle

qdk = pytest.importorskip("query_driven_key_b200")
lib = qdk.lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "think.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(think_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in think.h but not exported"
    assert set(names) == set(qdk.EXPORTED)


def test_library_is_built_for_sm100a_in_tree():
    assert os.path.dirname(qdk.LIB_PATH) == os.path.dirname(qdk.__file__)


@pytest.mark.parametrize("d", [1, 8, 10, 128])
def test_t_from_lambda_matches_oracle_rule(d):
    for i in range(0, 101):
        lam = i / 100
        assert qdk.think_t_from_lambda(d, lam) == oracle.t_from_lambda(d, lam), (d, lam)
    assert lib.think_t_from_lambda(0, 0.5) == 0
    assert lib.think_t_from_lambda(128, float("nan")) == 0


def test_pruned_pitch():
    import torch
    assert qdk.think_pruned_ld(0) == 0
    assert qdk.think_pruned_ld(1) == 8
    assert qdk.think_pruned_ld(131072) == 131072
    assert qdk.think_pruned_ld(4097) == 4104
    assert qdk.think_pruned_ld(5, torch.float32) == 8
    assert lib.think_pruned_ld(-1, 1) == -1


def test_workspace_sizes():
    assert qdk.think_score_workspace_size(1, 32, 8, 131072) > 0
    assert qdk.think_score_workspace_size(1, 32, 8, 131072, d=64) == 0
    assert qdk.think_score_workspace_size(1, 30, 8, 100) == 0
    n4 = qdk.think_decode_workspace_size(1, 32, 8, 131072)
    assert n4 >= 256 + 8 * 4 * 130 * 4
    assert qdk.think_decode_workspace_size(1, 32, 8, 0) == 0
    assert qdk.think_decode_workspace_size(1, 30, 8, 100) == 0       # Hq not a multiple of Hkv


def test_status_strings():
    for code in range(6):
        assert lib.think_status_string(code).startswith(b"THINK_")
    assert lib.think_status_string(99) == b"THINK_ERR_UNKNOWN"


I64x3 = ctypes.c_int64 * 3
FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: validation rejects first
MISALIGNED = ctypes.c_void_p(0x10008)


def test_score_validation():
    st = (128 * 64, 128 * 64, 128)
    s = I64x3(*st)
    f = lib.think_score_channels
    assert f(FAKE, FAKE, s, 1, 4, 2, 64, 8, 64, 1, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, s, 0, 4, 2, 64, 8, 128, 1, FAKE, FAKE, 0, None) == qdk.THINK_OK   # empty
    assert f(FAKE, None, s, 1, 4, 2, 64, 8, 128, 1, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, FAKE, s, 1, 6, 4, 64, 8, 128, 1, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, FAKE, s, 1, 4, 2, 64, 8, 128, 7, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, MISALIGNED, s, 1, 4, 2, 64, 8, 128, 1, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_ALIGNMENT
    bad = I64x3(128 * 64, 128 * 64, 130)
    assert f(FAKE, FAKE, bad, 1, 4, 2, 64, 8, 128, 1, FAKE, FAKE, 1 << 20, None) == qdk.THINK_ERR_ALIGNMENT
    assert f(FAKE, FAKE, s, 1, 4, 2, 64, 8, 128, 1, FAKE, FAKE, 16, None) == qdk.THINK_ERR_WORKSPACE


def test_prune_validation():
    st = I64x3(128 * 64, 128 * 64, 128)
    f = lib.think_prune
    ok_ws = qdk.think_score_workspace_size(1, 4, 2, 64)
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 1, 0, FAKE, FAKE, FAKE, 64, FAKE, ok_ws, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 1, 10, FAKE, None, FAKE, 64, FAKE, ok_ws, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 1, 10, FAKE, FAKE, FAKE, 63, FAKE, ok_ws, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 1, 10, FAKE, FAKE, FAKE, 64, FAKE, ok_ws - 8, None) == qdk.THINK_ERR_WORKSPACE
    assert f(FAKE, FAKE, st, 0, 4, 2, 64, 8, 128, 1, 10, FAKE, FAKE, FAKE, 64, FAKE, 0, None) == qdk.THINK_OK


def test_select_validation():
    f = lib.think_select_channels
    assert f(FAKE, 1, 2, 128, 0, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 128, 129, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 96, 10, FAKE, None) == qdk.THINK_ERR_UNSUPPORTED
    assert f(None, 1, 2, 128, 10, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 0, 2, 128, 10, FAKE, None) == qdk.THINK_OK


def test_compact_validation():
    s = I64x3(128 * 64, 128 * 64, 128)
    f = lib.think_compact_keys
    assert f(FAKE, s, 1, 2, 64, 128, 1, FAKE, 10, FAKE, 63, None) == qdk.THINK_ERR_INVALID_ARG   # ldk < N
    assert f(FAKE, s, 1, 2, 64, 128, 1, FAKE, 10, FAKE, 68, None) == qdk.THINK_ERR_ALIGNMENT     # 136 B pitch
    assert f(FAKE, s, 1, 2, 64, 128, 1, FAKE, 0, FAKE, 64, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, s, 1, 2, 0, 128, 1, FAKE, 10, FAKE, 0, None) == qdk.THINK_OK                  # N == 0


def test_append_validation():
    s = I64x3(128 * 64, 128 * 64, 128)
    f = lib.think_append_keys
    # (k_new, strides, B, Hkv, n_new, d, dtype, idx, T, k_pruned, ldk, n_at, stream)
    assert f(FAKE, s, 1, 2, 8, 128, 1, FAKE, 10, FAKE, 64, 57, None) == qdk.THINK_ERR_INVALID_ARG  # past capacity
    assert f(FAKE, s, 1, 2, -1, 128, 1, FAKE, 10, FAKE, 64, 0, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, s, 1, 2, 8, 128, 1, FAKE, 10, FAKE, 64, -1, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, s, 1, 2, 8, 96, 1, FAKE, 10, FAKE, 64, 56, None) == qdk.THINK_ERR_UNSUPPORTED
    assert f(FAKE, s, 1, 2, 8, 128, 1, FAKE, 0, FAKE, 64, 56, None) == qdk.THINK_ERR_INVALID_ARG    # T = 0
    assert f(FAKE, s, 1, 2, 8, 128, 1, FAKE, 10, FAKE, 68, 60, None) == qdk.THINK_ERR_ALIGNMENT     # 136 B pitch
    assert f(FAKE, s, 1, 2, 8, 128, 1, None, 10, FAKE, 64, 56, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, s, 1, 2, 0, 128, 1, FAKE, 10, FAKE, 64, 64, None) == qdk.THINK_OK              # nothing to append


def test_q4_sizes_and_validation():
    assert qdk.think_q4_ld(0) == 0 and qdk.think_q4_ld(1) == 64 and qdk.think_q4_ld(128) == 64
    assert qdk.think_q4_ld(129) == 128 and qdk.think_q4_ld(-1) == -1
    assert qdk.think_q4_groups_bytes(2, 8, 131072, 51) == 2 * 8 * 1024 * 52 * 8
    f = lib.think_quantize_keys_q4
    # (k_pruned, ldk, B, Hkv, N, T, codes, ldq, groups, stream)
    assert f(FAKE, 256, 1, 2, 200, 10, FAKE, 64, FAKE, None) == qdk.THINK_ERR_INVALID_ARG     # ldq < q4_ld(200)
    assert f(FAKE, 256, 1, 2, 200, 10, FAKE, 160, FAKE, None) == qdk.THINK_ERR_INVALID_ARG    # not a multiple of 64
    assert f(FAKE, 100, 1, 2, 200, 10, FAKE, 128, FAKE, None) == qdk.THINK_ERR_INVALID_ARG    # ldk < N
    assert f(FAKE, 260, 1, 2, 200, 10, FAKE, 128, FAKE, None) == qdk.THINK_ERR_ALIGNMENT      # 520 B pitch
    assert f(FAKE, 256, 1, 2, 200, 129, FAKE, 128, FAKE, None) == qdk.THINK_ERR_INVALID_ARG   # T > 128
    assert f(None, 256, 1, 2, 200, 10, FAKE, 128, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 256, 1, 2, 0, 10, FAKE, 0, FAKE, None) == qdk.THINK_OK                     # N == 0
    s = I64x3(128 * 64 * 2, 128 * 64, 128)
    g = lib.think_pruned_decode_attn_q4
    ws = qdk.think_decode_workspace_size(1, 4, 2, 200)
    def call(**kw):
        a = dict(q=FAKE, codes=FAKE, ldq=128, groups=FAKE, v=FAKE, vs=s, idx=FAKE, B=1, Hq=4, Hkv=2,
                 N=200, d=128, T=10, scale=0.088, out=FAKE, ws=FAKE, wsb=ws)
        a.update(kw)
        return g(*a.values(), None)
    assert call(ldq=64) == qdk.THINK_ERR_INVALID_ARG
    assert call(d=64) == qdk.THINK_ERR_UNSUPPORTED
    assert call(Hq=12) == qdk.THINK_ERR_UNSUPPORTED          # G = 6
    assert call(N=0) == qdk.THINK_ERR_INVALID_ARG
    assert call(wsb=ws - 16) == qdk.THINK_ERR_WORKSPACE
    assert call(codes=MISALIGNED) == qdk.THINK_ERR_ALIGNMENT
    assert call(scale=float("nan")) == qdk.THINK_ERR_INVALID_ARG
    assert call(B=0) == qdk.THINK_OK


def test_adaptive_validation():
    assert qdk.think_ragged_rows(2, 8, 51) == 2 * 8 * 64 and qdk.think_ragged_rows(1, 1, 129) == -1
    f = lib.think_select_adaptive
    # (scores, B, Hkv, d, tau, T_min, T_max, Th, rowoff, idx, stream)
    assert f(FAKE, 1, 2, 128, 1.5, 1, 64, FAKE, FAKE, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 128, float("nan"), 1, 64, FAKE, FAKE, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 128, 0.5, 8, 4, FAKE, FAKE, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 128, 0.5, 0, 4, FAKE, FAKE, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 1, 2, 96, 0.5, 1, 4, FAKE, FAKE, FAKE, None) == qdk.THINK_ERR_UNSUPPORTED
    assert f(FAKE, 1, 2, 128, 0.5, 1, 4, None, FAKE, FAKE, None) == qdk.THINK_ERR_INVALID_ARG
    assert f(FAKE, 0, 2, 128, 0.5, 1, 4, FAKE, FAKE, FAKE, None) == qdk.THINK_OK
    s = I64x3(128 * 64, 128 * 64, 128)
    g = lib.think_compact_keys_ragged
    assert g(FAKE, s, 1, 2, 64, 128, 1, FAKE, None, FAKE, 10, FAKE, 64, None) == qdk.THINK_ERR_INVALID_ARG
    assert g(FAKE, s, 1, 2, 64, 128, 1, FAKE, FAKE, FAKE, 129, FAKE, 64, None) == qdk.THINK_ERR_INVALID_ARG
    p = lib.think_prune_adaptive
    sws = qdk.think_score_workspace_size(1, 4, 2, 64)
    # (q_win, k, strides, B, Hq, Hkv, N, S, d, dtype, tau, T_min, T_max, scores, Th, rowoff, idx, kp, ldk,
    #  ws, ws_bytes, stream)
    pa = lambda **kw: (lambda a: p(a["q"], a["k"], s, a["B"], 4, 2, 64, 8, a["d"], 1, a["tau"], a["tmin"], a["tmax"],
                                   FAKE, a["Th"], FAKE, FAKE, FAKE, 64, FAKE, a["wsb"], None))(
        dict(dict(q=FAKE, k=FAKE, B=1, d=128, tau=0.5, tmin=1, tmax=32, Th=FAKE, wsb=sws), **kw))
    assert pa(tau=1.5) == qdk.THINK_ERR_INVALID_ARG
    assert pa(tmin=8, tmax=4) == qdk.THINK_ERR_INVALID_ARG
    assert pa(tmax=129) == qdk.THINK_ERR_INVALID_ARG
    assert pa(d=96) == qdk.THINK_ERR_UNSUPPORTED
    assert pa(Th=None) == qdk.THINK_ERR_INVALID_ARG
    assert pa(Th=ctypes.c_void_p(0x10002)) == qdk.THINK_ERR_ALIGNMENT
    assert pa(k=MISALIGNED) == qdk.THINK_ERR_ALIGNMENT
    assert pa(wsb=sws - 8) == qdk.THINK_ERR_WORKSPACE
    assert pa(B=0, wsb=0) == qdk.THINK_OK
    h = lib.think_pruned_decode_attn_ragged
    vs = I64x3(128 * 64 * 2, 128 * 64, 128)
    ws = qdk.think_decode_workspace_size(1, 4, 2, 64)
    assert h(FAKE, FAKE, 64, FAKE, vs, FAKE, FAKE, FAKE, 0, 1, 4, 2, 64, 128, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_INVALID_ARG
    assert h(FAKE, FAKE, 64, FAKE, vs, FAKE, None, FAKE, 32, 1, 4, 2, 64, 128, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_INVALID_ARG
    assert h(FAKE, FAKE, 64, FAKE, vs, FAKE, FAKE, FAKE, 32, 1, 4, 2, 64, 128, 0.1, FAKE, FAKE, ws - 8, None) == qdk.THINK_ERR_WORKSPACE
    assert h(FAKE, FAKE, 64, FAKE, vs, FAKE, FAKE, FAKE, 32, 0, 4, 2, 64, 128, 0.1, FAKE, FAKE, 0, None) == qdk.THINK_OK


def test_eviction_validation():
    st = I64x3(128 * 64, 128 * 64, 128)
    f = lib.think_token_mass
    ws = qdk.think_token_mass_workspace_size(1, 4, 2, 64, 8)
    assert ws > 256 and qdk.think_token_mass_workspace_size(1, 4, 3, 64, 8) == 0
    # (q_win, k, strides, B, Hq, Hkv, N, S, d, dtype, scale, mass, ws, ws_bytes, stream)
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 0, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_UNSUPPORTED   # fp32
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 64, 1, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_UNSUPPORTED    # d
    assert f(FAKE, FAKE, st, 1, 16, 2, 64, 128, 128, 1, 0.1, FAKE, FAKE, 1 << 30, None) == qdk.THINK_ERR_UNSUPPORTED  # G*S > 512
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 0, 128, 1, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_INVALID_ARG    # S = 0
    assert f(FAKE, FAKE, st, 1, 4, 2, 64, 8, 128, 1, 0.1, FAKE, FAKE, ws - 8, None) == qdk.THINK_ERR_WORKSPACE
    assert f(FAKE, MISALIGNED, st, 1, 4, 2, 64, 8, 128, 1, 0.1, FAKE, FAKE, ws, None) == qdk.THINK_ERR_ALIGNMENT
    assert f(FAKE, FAKE, st, 0, 4, 2, 64, 8, 128, 1, 0.1, FAKE, FAKE, 0, None) == qdk.THINK_OK
    g = lib.think_select_tokens
    sws = qdk.think_select_tokens_workspace_size(1, 2, 64)
    assert sws > 4 * 2 * 256 * 4 and qdk.think_select_tokens_workspace_size(1, 2, 0) == 0
    # (mass, B, Hkv, N, M, kept, ws, ws_bytes, stream)
    assert g(FAKE, 1, 2, 64, 0, FAKE, FAKE, sws, None) == qdk.THINK_ERR_INVALID_ARG
    assert g(FAKE, 1, 2, 64, 65, FAKE, FAKE, sws, None) == qdk.THINK_ERR_INVALID_ARG
    assert g(None, 1, 2, 64, 8, FAKE, FAKE, sws, None) == qdk.THINK_ERR_INVALID_ARG
    assert g(FAKE, 1, 2, 64, 8, FAKE, None, sws, None) == qdk.THINK_ERR_INVALID_ARG
    assert g(FAKE, 1, 2, 64, 8, FAKE, FAKE, sws - 4, None) == qdk.THINK_ERR_WORKSPACE
    assert g(FAKE, 1, 2, 64, 8, FAKE, MISALIGNED, sws, None) == qdk.THINK_ERR_ALIGNMENT
    assert g(FAKE, 0, 2, 64, 8, FAKE, None, 0, None) == qdk.THINK_OK
    h = lib.think_gather_tokens
    assert h(FAKE, st, 1, 2, 64, 96, 1, FAKE, 8, FAKE, None) == qdk.THINK_ERR_UNSUPPORTED
    assert h(FAKE, st, 1, 2, 64, 128, 1, FAKE, 8, MISALIGNED, None) == qdk.THINK_ERR_ALIGNMENT
    assert h(FAKE, st, 1, 2, 64, 128, 1, FAKE, 0, FAKE, None) == qdk.THINK_OK


def test_decode_validation():
    s = I64x3(128 * 64 * 2, 128 * 64, 128)
    f = lib.think_pruned_decode_attn
    args = lambda **kw: dict(dict(q=FAKE, kp=FAKE, ldk=64, v=FAKE, vs=s, idx=FAKE, B=1, Hq=4, Hkv=2,
                                   N=64, d=128, T=10, dt=1, scale=0.088, out=FAKE, ws=FAKE,
                                   wsb=1 << 20), **kw)
    call = lambda a: f(a["q"], a["kp"], a["ldk"], a["v"], a["vs"], a["idx"], a["B"], a["Hq"], a["Hkv"],
                       a["N"], a["d"], a["T"], a["dt"], a["scale"], a["out"], a["ws"], a["wsb"], None)
    assert call(args(N=0, ldk=0)) == qdk.THINK_ERR_INVALID_ARG          # attention over no keys
    assert call(args(Hq=6)) == qdk.THINK_ERR_UNSUPPORTED                 # group of 3
    assert call(args(Hq=32, Hkv=2)) == qdk.THINK_ERR_UNSUPPORTED         # group of 16
    assert call(args(T=0)) == qdk.THINK_ERR_INVALID_ARG
    assert call(args(d=64)) == qdk.THINK_ERR_UNSUPPORTED
    assert call(args(scale=float("inf"))) == qdk.THINK_ERR_INVALID_ARG
    assert call(args(q=MISALIGNED)) == qdk.THINK_ERR_ALIGNMENT
    assert call(args(wsb=64)) == qdk.THINK_ERR_WORKSPACE
    assert call(args(out=None)) == qdk.THINK_ERR_INVALID_ARG
    assert call(args(B=0)) == qdk.THINK_OK


def test_select_tokens_workspace_layout():
    # radix histograms [4][heads][256] + (M-th key, ties) per head + two counts
    # per chunk and head, int32, each part padded to 256 bytes; chunks of
    # 256 threads x kpt keys, kpt a multiple of 16 keeping chunks <= 1024
    def want(B, Hkv, N):
        heads = B * Hkv
        kpt = 16 * max(1, -(-N // (256 * 1024 * 16)))
        chunks = max(1, -(-N // (256 * kpt)))
        pad = lambda x: -(-x // 256) * 256
        return pad(4 * heads * 256 * 4) + pad(heads * 2 * 4) + heads * chunks * 2 * 4
    for B, Hkv, N in [(1, 1, 1), (1, 8, 131072), (4, 8, 32768), (1, 1, 4_194_304), (1, 1, 4_194_305),
                      (2, 3, 5_000_000), (1, 1, 2**31 - 1)]:
        assert qdk.think_select_tokens_workspace_size(B, Hkv, N) == want(B, Hkv, N), (B, Hkv, N)
    assert qdk.think_select_tokens_workspace_size(1, 1, 2**31) == 0


def _round_plan(heads, N):
    """The one-kernel prune's split plan restated: runs of L 64-token tiles per
    head and rounds of hpr heads (about 296 runs and at most 2560 tiles per
    round), L in 1..64 minimising rounds x ceil(runs per round / 296) x (L + 2),
    ties to the longer run.  Returns (L, runs per head, heads per round,
    rounds)."""
    cdiv = lambda a, b: -(-a // b)
    tph = max(1, cdiv(N, 64))
    heads = max(heads, 1)
    best = None
    for L in range(1, min(64, tph) + 1):
        R = cdiv(tph, L)
        hpr = min(max(296 // R, 1), heads)
        if hpr > 1 and hpr * tph > 2560:
            hpr = max(1, 2560 // tph)
        rounds = cdiv(heads, hpr)
        cost = rounds * cdiv(hpr * R, 296) * (L + 2)
        if best is None or cost <= best[0]:
            best = (cost, L, R, hpr, rounds)
    return best[1:]


def _wave_plans(heads, N):
    """The two-launch score pass's split plans restated: for W = 1..4 waves of
    148 x 3 resident blocks, the shortest runs whose count fits them.  Returns
    {W: runs per head}; the pass takes the fewest W filling >= 90% of the
    slots (else the best filled)."""
    cdiv = lambda a, b: -(-a // b)
    tph = max(1, cdiv(N, 64))
    plans = {}
    for w in range(1, 5):
        rph = max(1, 148 * 3 * w // max(heads, 1))
        st = min(max(cdiv(tph, rph), 1), tph)
        plans[w] = cdiv(tph, st)
    return plans


def test_score_workspace_follows_the_plans():
    # header 256 B + ready flags, head tickets (256-byte aligned) + group
    # tickets [heads][groups] + window-query energies [heads][G][128] fp64 +
    # run partials [heads][runs][128] + group sums [heads][groups][128]
    # (groups of 16 runs), for the plan with the most runs per head; pins the
    # plan rules on the CPU
    pad = lambda x: -(-x // 256) * 256
    for B, Hq, Hkv, N in [(1, 32, 8, 131072), (4, 32, 8, 32768), (1, 32, 32, 4096), (32, 32, 8, 8192),
                          (1, 1, 1, 512), (1, 8, 1, 1), (2, 16, 8, 0), (3, 24, 8, 100_000)]:
        heads, G = B * Hkv, Hq // Hkv
        R = max(_round_plan(heads, N)[1], max(_wave_plans(heads, N).values()))
        groups = -(-R // 16)
        want = (256 + 2 * pad(heads * 4) + pad(heads * groups * 4) + pad(heads * G * 128 * 8) +
                pad(heads * R * 128 * 8) + heads * groups * 128 * 8)
        assert qdk.think_score_workspace_size(B, Hq, Hkv, N, 128) == want, (B, Hq, Hkv, N)
    # long-context layer: one head per round, 293 runs of 7 tiles; GQA batch 4
    # at N = 32K: 4 heads per round, 74 runs of 7; the 32-batch sweep layer: 18
    # heads per round, 16 runs of 8; the MHA layer: one round of 32 heads
    assert _round_plan(8, 131072) == (7, 293, 1, 8)
    assert _round_plan(32, 32768) == (7, 74, 4, 8)
    assert _round_plan(256, 8192) == (8, 16, 18, 15)
    assert _round_plan(32, 4096) == (8, 8, 32, 1)
    # the two-launch pass on the long-context layer: one wave of 432 runs of 38 tiles
    assert _wave_plans(8, 131072)[1] == 54


def test_python_decode_checks_before_any_call():
    # The binding rejects a decode whose output is not a contiguous [B, Hq, d]
    # fp32 tensor, or whose tensors are not on the GPU, before it calls the
    # library (CPU tensors here: nothing reaches the C entry point).
    import torch
    B, Hq, Hkv, N, T, d = 1, 4, 2, 64, 10, 128
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16)
    kp = torch.zeros((B, Hkv, T, 64), dtype=torch.bfloat16)
    v = torch.zeros((B, Hkv, N, d), dtype=torch.bfloat16)
    idx = torch.zeros((B, Hkv, T), dtype=torch.int32)
    ws = torch.zeros(4096, dtype=torch.uint8)
    bad_outs = [torch.zeros((B, Hq, d), dtype=torch.float32),                 # host memory
                torch.zeros((B, Hq, 2 * d), dtype=torch.float32)[..., ::2],  # not contiguous
                torch.zeros((B, Hq + 1, d), dtype=torch.float32),            # wrong shape
                torch.zeros((B, Hq, d), dtype=torch.bfloat16)]               # wrong dtype
    for out in bad_outs:
        with pytest.raises(qdk.ThinkError):
            qdk.think_pruned_decode_attn(q, kp, 64, v, idx, out, ws)

"""fp64 CPU oracle of the ThinK decode-time path (query-driven key-channel pruning).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. The CUDA product path
(``query_driven_key_b200``) never imports it and shares no code with it.

Source: "ThinK: Thinner Key Cache by Query-Driven Pruning" (Xu et al., ICLR
2025), method section (rate each key channel's relevance to the query, sort,
prune the least relevant channels, run inference with the pruned cache) and
abstract (prune so that the loss in the attention weights stays minimal).

The arithmetic lives in ``think_oracle.c`` (plain fp64 loops); this module only
marshals numpy arrays into it, plus two small helpers that are written out in
Python because they are definitions, not kernels:

* ``attention_loss`` -- the attention-weight loss ||Q K^T - Q_S K_S^T||_F that
  the abstract says the pruning keeps small;
* ``bruteforce_best_subset`` -- the exhaustive minimiser of that loss over all
  channel subsets of a given size (tiny d only);
* ``oracle_append`` -- the growing cache: new tokens' keys compacted with the
  fixed kept channels and appended (a composition of ``oracle_compact``).

The 4-bit thinner cache (``oracle_quantize_q4`` / ``oracle_dequantize_q4``)
and the adaptive kept width (``oracle_select_adaptive``) are plain C in
``think_oracle.c``; ``oracle_decode_ragged`` composes the per-head oracle
calls for a kept width that differs between heads.  Token eviction
(``oracle_token_mass``, ``oracle_select_tokens``) is plain C too;
``oracle_evict_and_prune`` composes it with the prune.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, library routines, a hand-worked example).
"""
from __future__ import annotations

import ctypes
import itertools
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "think_oracle.c")
_LIB = os.path.join(_HERE, "libthink_oracle.so")

_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle's C source with gcc (fp64, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
             "-fPIC", "-shared", src, "-o", tmp, "-lm"],
            check=True,
        )
        os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: invalid argument (code {rc})")


class Oracle:
    """numpy front end of one compiled copy of ``think_oracle.c``."""

    def __init__(self, so_path: str):
        lib = ctypes.CDLL(so_path)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.oracle_score.argtypes = [P, P, I, I, I, I, I, I, P]
        lib.oracle_score_explicit.argtypes = [P, P, I, I, I, I, I, I, P]
        lib.oracle_select.argtypes = [P, I, I, I, I, P]
        lib.oracle_compact.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_decode.argtypes = [P, P, P, P, I, I, I, I, I, I, D, P]
        lib.oracle_dense_decode.argtypes = [P, P, P, I, I, I, I, I, D, P]
        lib.oracle_quantize_q4.argtypes = [P, I, I, I, I, I, P, P]
        lib.oracle_dequantize_q4.argtypes = [P, P, I, I, I, I, I, P]
        lib.oracle_select_adaptive.argtypes = [P, I, I, I, D, I, I, P, P, P, I]
        lib.oracle_token_mass.argtypes = [P, P, I, I, I, I, I, I, D, P]
        lib.oracle_select_tokens.argtypes = [P, I, I, I, I, P]
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        for f in ("oracle_score", "oracle_score_explicit", "oracle_select", "oracle_compact",
                  "oracle_decode", "oracle_dense_decode", "oracle_quantize_q4", "oracle_dequantize_q4",
                  "oracle_select_adaptive", "oracle_token_mass", "oracle_select_tokens"):
            getattr(lib, f).restype = I
        self.lib = lib

    def num_threads(self) -> int:
        return self.lib.oracle_num_threads()

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def score(self, q_win, k) -> np.ndarray:
        """q_win [B,Hq,S,d], k [B,Hkv,N,d] -> scores [B,Hkv,d] (fp64)."""
        q_win, k = _f64(q_win), _f64(k)
        B, Hq, S, d = q_win.shape
        Bk, Hkv, N, dk = k.shape
        if Bk != B or dk != d:
            raise ValueError("shape mismatch")
        out = np.zeros((B, Hkv, d), dtype=np.float64)
        _check(self.lib.oracle_score(_ptr(q_win), _ptr(k), B, Hq, Hkv, S, N, d, _ptr(out)),
               "oracle_score")
        return out

    def score_explicit(self, q_win, k) -> np.ndarray:
        """Same quantity from its definition (explicit S x N outer products)."""
        q_win, k = _f64(q_win), _f64(k)
        B, Hq, S, d = q_win.shape
        _, Hkv, N, _ = k.shape
        out = np.zeros((B, Hkv, d), dtype=np.float64)
        _check(self.lib.oracle_score_explicit(_ptr(q_win), _ptr(k), B, Hq, Hkv, S, N, d, _ptr(out)),
               "oracle_score_explicit")
        return out

    def select(self, scores, T: int) -> np.ndarray:
        """scores [B,Hkv,d] -> idx int32 [B,Hkv,T], the top-T channels in ascending order."""
        scores = _f64(scores)
        B, Hkv, d = scores.shape
        idx = np.zeros((B, Hkv, T), dtype=np.int32)
        _check(self.lib.oracle_select(_ptr(scores), B, Hkv, d, int(T), _ptr(idx)), "oracle_select")
        return idx

    def compact(self, k, idx) -> np.ndarray:
        """k [B,Hkv,N,d], idx [B,Hkv,T] -> K' [B,Hkv,N,T] (same values, fp64)."""
        k = _f64(k)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        B, Hkv, N, d = k.shape
        T = idx.shape[-1]
        kp = np.zeros((B, Hkv, N, T), dtype=np.float64)
        _check(self.lib.oracle_compact(_ptr(k), _ptr(idx), B, Hkv, N, d, T, _ptr(kp)),
               "oracle_compact")
        return kp

    def decode(self, q, kp, v, idx, scale: float | None = None) -> np.ndarray:
        """q [B,Hq,d], K' [B,Hkv,N,T], v [B,Hkv,N,d], idx [B,Hkv,T] -> out [B,Hq,d] (fp64)."""
        q, kp, v = _f64(q), _f64(kp), _f64(v)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        B, Hq, d = q.shape
        _, Hkv, N, T = kp.shape
        if scale is None:
            scale = default_scale(d)
        out = np.zeros((B, Hq, d), dtype=np.float64)
        _check(self.lib.oracle_decode(_ptr(q), _ptr(kp), _ptr(v), _ptr(idx), B, Hq, Hkv, N, d, T,
                                      float(scale), _ptr(out)), "oracle_decode")
        return out

    def dense_decode(self, q, k, v, scale: float | None = None) -> np.ndarray:
        """Dense decode attention over the unpruned cache: q [B,Hq,d], k/v [B,Hkv,N,d]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, d = q.shape
        _, Hkv, N, _ = k.shape
        if scale is None:
            scale = default_scale(d)
        out = np.zeros((B, Hq, d), dtype=np.float64)
        _check(self.lib.oracle_dense_decode(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, N, d,
                                            float(scale), _ptr(out)), "oracle_dense_decode")
        return out

    def quantize_q4(self, kp, group: int = 128):
        """K' [B,Hkv,N,T] (bf16 values) -> codes uint8 [B,Hkv,N,T] (0..15) and group
        parameters fp32 [B,Hkv,ceil(N/group),T,2] = (scale, min)."""
        kp = _f64(kp)
        B, Hkv, N, T = kp.shape
        ng = -(-N // group)
        codes = np.zeros((B, Hkv, N, T), dtype=np.uint8)
        gs = np.zeros((B, Hkv, ng, T, 2), dtype=np.float32)
        _check(self.lib.oracle_quantize_q4(_ptr(kp), B, Hkv, N, T, group, _ptr(codes), _ptr(gs)),
               "oracle_quantize_q4")
        return codes, gs

    def dequantize_q4(self, codes, gs, group: int = 128) -> np.ndarray:
        """codes [B,Hkv,N,T], group parameters -> dequantised K' (bf16 values, fp64)."""
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        gs = np.ascontiguousarray(gs, dtype=np.float32)
        B, Hkv, N, T = codes.shape
        out = np.zeros((B, Hkv, N, T), dtype=np.float64)
        _check(self.lib.oracle_dequantize_q4(_ptr(codes), _ptr(gs), B, Hkv, N, T, group, _ptr(out)),
               "oracle_dequantize_q4")
        return out

    def select_adaptive(self, scores, tau: float, T_min: int, T_max: int):
        """scores [B,Hkv,d] -> (T_h [B,Hkv], off [B*Hkv+1], idx [total]) of the adaptive rule."""
        scores = _f64(scores)
        B, Hkv, d = scores.shape
        Th = np.zeros(B * Hkv, dtype=np.int32)
        off = np.zeros(B * Hkv + 1, dtype=np.int32)
        idx = np.zeros(max(1, B * Hkv * T_max), dtype=np.int32)
        rows = self.lib.oracle_select_adaptive(_ptr(scores), B, Hkv, d, float(tau), int(T_min), int(T_max),
                                               _ptr(Th), _ptr(off), _ptr(idx), idx.size)
        _check(min(rows, 0), "oracle_select_adaptive")
        return Th.reshape(B, Hkv), off, idx[:rows].copy()

    def token_mass(self, q_win, k, scale: float | None = None) -> np.ndarray:
        """q_win [B,Hq,S,d], k [B,Hkv,N,d] -> observation-window attention mass [B,Hkv,N]."""
        q_win, k = _f64(q_win), _f64(k)
        B, Hq, S, d = q_win.shape
        _, Hkv, N, _ = k.shape
        scale = default_scale(d) if scale is None else scale
        mass = np.zeros((B, Hkv, N), dtype=np.float64)
        _check(self.lib.oracle_token_mass(_ptr(q_win), _ptr(k), B, Hq, Hkv, S, N, d, float(scale), _ptr(mass)),
               "oracle_token_mass")
        return mass

    def select_tokens(self, mass, M: int) -> np.ndarray:
        """mass [B,Hkv,N] -> the M kept tokens per head [B,Hkv,M] (ascending)."""
        mass = _f64(mass)
        B, Hkv, N = mass.shape
        kept = np.zeros((B, Hkv, M), dtype=np.int32)
        _check(self.lib.oracle_select_tokens(_ptr(mass), B, Hkv, N, M, _ptr(kept)), "oracle_select_tokens")
        return kept

    def prune(self, q_win, k, T: int):
        """The whole prune step: scores, kept channels, thinner key cache."""
        scores = self.score(q_win, k)
        idx = self.select(scores, T)
        return scores, idx, self.compact(k, idx)


def default_oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default_oracle().num_threads()


def set_num_threads(n: int) -> None:
    default_oracle().set_num_threads(n)


def default_scale(d: int) -> float:
    """Softmax temperature 1/sqrt(d) of the full head width (reading: the pruned
    dot product keeps the unpruned model's scale)."""
    return 1.0 / float(np.sqrt(d))


def t_from_lambda(d: int, lam: float) -> int:
    """Kept channels T for pruning ratio lambda: (1 - lambda) * d rounded half up,
    clamped to [1, d]."""
    t = int(np.floor((1.0 - lam) * d + 0.5))
    return max(1, min(d, t))


def oracle_score(q_win, k):
    return default_oracle().score(q_win, k)


def oracle_score_explicit(q_win, k):
    return default_oracle().score_explicit(q_win, k)


def oracle_select(scores, T):
    return default_oracle().select(scores, T)


def oracle_compact(k, idx):
    return default_oracle().compact(k, idx)


def oracle_decode(q, kp, v, idx, scale=None):
    return default_oracle().decode(q, kp, v, idx, scale)


def oracle_dense_decode(q, k, v, scale=None):
    return default_oracle().dense_decode(q, k, v, scale)


def oracle_prune(q_win, k, T):
    return default_oracle().prune(q_win, k, T)


def oracle_append(kp, k_new, idx):
    """Growing cache: after the prune, the keys of new tokens are compacted with
    each head's kept channels (fixed at prune time) and appended along N:
    [K' | compact(k_new, idx)].  The ThinK pages only say that inference runs
    with the pruned cache; the new tokens' keys are read here the same way as
    the cached ones.  kp [B,Hkv,N,T], k_new [B,Hkv,n,d] -> [B,Hkv,N+n,T]."""
    return np.concatenate([_f64(kp), oracle_compact(k_new, idx)], axis=2)


def oracle_quantize_q4(kp, group: int = 128):
    return default_oracle().quantize_q4(kp, group)


def oracle_dequantize_q4(codes, gs, group: int = 128):
    return default_oracle().dequantize_q4(codes, gs, group)


def oracle_select_adaptive(scores, tau, T_min, T_max):
    return default_oracle().select_adaptive(scores, tau, T_min, T_max)


def oracle_decode_ragged(q, k, v, Th, off, idx, scale=None):
    """Decode with a kept width per head: each (b, h_kv) attends with its own
    kept channels idx[off_h : off_h + T_h] (oracle_compact and oracle_decode
    per head).  q [B,Hq,d], k, v [B,Hkv,N,d] -> out [B,Hq,d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for h in range(Hkv):
            bh = b * Hkv + h
            ih = np.asarray(idx[off[bh]:off[bh] + Th[b, h]], dtype=np.int32)[None, None, :]
            kp = oracle_compact(k[b:b + 1, h:h + 1], ih)
            out[b:b + 1, h * G:(h + 1) * G] = oracle_decode(q[b:b + 1, h * G:(h + 1) * G], kp,
                                                             v[b:b + 1, h:h + 1], ih, scale)
    return out


def oracle_token_mass(q_win, k, scale=None):
    return default_oracle().token_mass(q_win, k, scale)


def oracle_select_tokens(mass, M):
    return default_oracle().select_tokens(mass, M)


def oracle_gather_tokens(x, kept):
    """x [B,Hkv,N,d], kept [B,Hkv,M] -> x[b,h,kept[b,h],:] [B,Hkv,M,d] (numpy gather)."""
    x = _f64(x)
    return np.take_along_axis(x, np.asarray(kept)[..., None].astype(np.int64), axis=2)


def oracle_evict_and_prune(q_win, k, M, T):
    """Token eviction then channel pruning: kept tokens by window attention
    mass, then oracle_prune on the kept tokens' keys.  Returns (kept, scores,
    idx, K' over the kept tokens)."""
    kept = oracle_select_tokens(oracle_token_mass(q_win, k), M)
    scores, idx, kp = oracle_prune(q_win, oracle_gather_tokens(k, kept), T)
    return kept, scores, idx, kp


def attention_loss(q_win_head, k_head, keep) -> float:
    """||Q K^T - Q_S K_S^T||_F for one head: Q [S,d], K [N,d], keep = channel list.

    The abstract's objective: pruning should lose as little of the attention
    weights Q K^T as possible."""
    Q = _f64(q_win_head)
    K = _f64(k_head)
    keep = list(keep)
    full = Q @ K.T
    part = Q[:, keep] @ K[:, keep].T
    return float(np.linalg.norm(full - part, "fro"))


def bruteforce_best_subset(q_win_head, k_head, T: int):
    """Exhaustive search over all C(d, T) channel subsets of the attention loss.

    Returns (best_loss, list of every subset, as sorted tuples, that reaches it
    within 1e-12 relative)."""
    Q = _f64(q_win_head)
    K = _f64(k_head)
    d = Q.shape[1]
    results = []
    for keep in itertools.combinations(range(d), T):
        results.append((attention_loss(Q, K, keep), keep))
    best = min(r[0] for r in results)
    tol = 1e-12 * max(1.0, abs(best))
    return best, [keep for loss, keep in results if loss <= best + tol]

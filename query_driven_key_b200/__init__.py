"""Python binding of libthink.so, the C-ABI CUDA library of the ThinK decode path.

"ThinK: Thinner Key Cache by Query-Driven Pruning": score every key channel
against the observation-window queries, keep the top-T channels per KV head,
compact K into a thinner cache, and run decode attention with it.

Argument marshalling only: every function passes device pointers, sizes and
strides of torch tensors to the C entry point of the same name; every step of
the computation runs in the library's CUDA kernels. There is no CPU fallback:
importing this package raises if ``libthink.so`` cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# THINK_DEBUG_LIB=1 loads the debug build (index checks at the global stores,
# reported as THINK_DEVICE_OOB in the device status word) instead.
LIB_PATH = os.path.join(_PKG, "libthink_debug.so" if os.environ.get("THINK_DEBUG_LIB") == "1" else "libthink.so")

THINK_OK = 0
THINK_ERR_INVALID_ARG = 1
THINK_ERR_UNSUPPORTED = 2
THINK_ERR_WORKSPACE = 3
THINK_ERR_CUDA = 4
THINK_ERR_ALIGNMENT = 5
THINK_F32 = 0
THINK_BF16 = 1
THINK_DEVICE_TIMEOUT_FULL = 0x1
THINK_DEVICE_TIMEOUT_EMPTY = 0x2
THINK_DEVICE_TIMEOUT_READY = 0x4
THINK_DEVICE_TIMEOUT_BARRIER = 0x8
THINK_DEVICE_OOB = 0x10

EXPORTED = (
    "think_status_string", "think_t_from_lambda", "think_pruned_ld",
    "think_score_workspace_size", "think_score_channels", "think_select_channels",
    "think_compact_keys", "think_append_keys", "think_prune", "think_decode_workspace_size",
    "think_pruned_decode_attn",
    "think_workspace_init", "think_read_device_status", "think_noalloc_scratch_bytes",
    "think_pruned_decode_attn_noalloc", "think_noalloc_read_device_status", "think_q4_ld", "think_q4_groups_bytes",
    "think_quantize_keys_q4", "think_pruned_decode_attn_q4", "think_ragged_rows", "think_select_adaptive",
    "think_compact_keys_ragged", "think_prune_adaptive", "think_pruned_decode_attn_ragged",
    "think_token_mass_workspace_size",
    "think_token_mass", "think_select_tokens_workspace_size", "think_select_tokens", "think_gather_tokens",
)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libthink.so not found at {LIB_PATH}; build it with "
            "`python query_driven_key_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ, D, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                           ctypes.c_double, ctypes.c_float)
    I64P = ctypes.POINTER(ctypes.c_int64)
    lib.think_status_string.argtypes = [I]
    lib.think_status_string.restype = ctypes.c_char_p
    lib.think_t_from_lambda.argtypes = [I, D]
    lib.think_t_from_lambda.restype = I
    lib.think_pruned_ld.argtypes = [I64, I]
    lib.think_pruned_ld.restype = I64
    lib.think_score_workspace_size.argtypes = [I, I, I, I64, I]
    lib.think_score_workspace_size.restype = SZ
    lib.think_score_channels.argtypes = [P, P, I64P, I, I, I, I64, I, I, I, P, P, SZ, P]
    lib.think_score_channels.restype = I
    lib.think_select_channels.argtypes = [P, I, I, I, I, P, P]
    lib.think_select_channels.restype = I
    lib.think_compact_keys.argtypes = [P, I64P, I, I, I64, I, I, P, I, P, I64, P]
    lib.think_compact_keys.restype = I
    lib.think_prune.argtypes = [P, P, I64P, I, I, I, I64, I, I, I, I, P, P, P, I64, P, SZ, P]
    lib.think_prune.restype = I
    lib.think_append_keys.argtypes = [P, I64P, I, I, I64, I, I, P, I, P, I64, I64, P]
    lib.think_append_keys.restype = I
    lib.think_q4_ld.argtypes = [I64]
    lib.think_q4_ld.restype = I64
    lib.think_q4_groups_bytes.argtypes = [I, I, I64, I]
    lib.think_q4_groups_bytes.restype = SZ
    lib.think_quantize_keys_q4.argtypes = [P, I64, I, I, I64, I, P, I64, P, P]
    lib.think_quantize_keys_q4.restype = I
    lib.think_pruned_decode_attn_q4.argtypes = [P, P, I64, P, P, I64P, P, I, I, I, I64, I, I, F, P, P, SZ, P]
    lib.think_pruned_decode_attn_q4.restype = I
    lib.think_ragged_rows.argtypes = [I, I, I]
    lib.think_ragged_rows.restype = I64
    lib.think_select_adaptive.argtypes = [P, I, I, I, D, I, I, P, P, P, P]
    lib.think_prune_adaptive.argtypes = [P, P, I64P, I, I, I, I64, I, I, I, D, I, I, P, P, P, P, P, I64, P, SZ, P]
    lib.think_prune_adaptive.restype = I
    lib.think_select_adaptive.restype = I
    lib.think_compact_keys_ragged.argtypes = [P, I64P, I, I, I64, I, I, P, P, P, I, P, I64, P]
    lib.think_compact_keys_ragged.restype = I
    lib.think_pruned_decode_attn_ragged.argtypes = [P, P, I64, P, I64P, P, P, P, I, I, I, I, I64, I, F, P, P, SZ, P]
    lib.think_pruned_decode_attn_ragged.restype = I
    lib.think_token_mass_workspace_size.argtypes = [I, I, I, I64, I]
    lib.think_token_mass_workspace_size.restype = SZ
    lib.think_token_mass.argtypes = [P, P, I64P, I, I, I, I64, I, I, I, F, P, P, SZ, P]
    lib.think_token_mass.restype = I
    lib.think_select_tokens.argtypes = [P, I, I, I64, I, P, P, SZ, P]
    lib.think_select_tokens.restype = I
    lib.think_select_tokens_workspace_size.argtypes = [I, I, I64]
    lib.think_select_tokens_workspace_size.restype = SZ
    lib.think_gather_tokens.argtypes = [P, I64P, I, I, I64, I, I, P, I, P, P]
    lib.think_gather_tokens.restype = I
    lib.think_decode_workspace_size.argtypes = [I, I, I, I64, I, I]
    lib.think_decode_workspace_size.restype = SZ
    lib.think_pruned_decode_attn.argtypes = [P, P, I64, P, I64P, P, I, I, I, I64, I, I, I, F, P,
                                             P, SZ, P]
    lib.think_pruned_decode_attn.restype = I
    lib.think_noalloc_scratch_bytes.argtypes = []
    lib.think_noalloc_scratch_bytes.restype = SZ
    lib.think_pruned_decode_attn_noalloc.argtypes = [P, P, I64, P, I64P, P, I, I, I, I64, I, I, I, F,
                                                     P, P]
    lib.think_pruned_decode_attn_noalloc.restype = I
    lib.think_workspace_init.argtypes = [P, SZ, P]
    lib.think_workspace_init.restype = I
    lib.think_read_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), P]
    lib.think_read_device_status.restype = I
    lib.think_noalloc_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
    lib.think_noalloc_read_device_status.restype = I
    return lib


lib = _load()


class ThinkError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {lib.think_status_string(code).decode()}")


def _check(code: int, where: str) -> None:
    if code != THINK_OK:
        raise ThinkError(code, where)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return THINK_BF16
    if t.dtype == torch.float32:
        return THINK_F32
    raise ThinkError(THINK_ERR_INVALID_ARG, f"dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else ctypes.c_void_p(t.data_ptr() or 0)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_raw_stream = torch._C._cuda_getCurrentRawStream  # device index -> current stream handle


def _strides3(t: torch.Tensor):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ThinkError(THINK_ERR_INVALID_ARG, "expected a [B,H,N,d] tensor with contiguous channels")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def think_t_from_lambda(d: int, lam: float) -> int:
    return lib.think_t_from_lambda(int(d), float(lam))


def think_pruned_ld(N: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return lib.think_pruned_ld(int(N), THINK_BF16 if dtype == torch.bfloat16 else THINK_F32)


def think_score_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int = 128) -> int:
    return lib.think_score_workspace_size(B, Hq, Hkv, N, d)


def think_decode_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int = 128,
                                dtype: torch.dtype = torch.bfloat16) -> int:
    return lib.think_decode_workspace_size(B, Hq, Hkv, N, d,
                                           THINK_BF16 if dtype == torch.bfloat16 else THINK_F32)


def think_score_channels(q_win: torch.Tensor, k: torch.Tensor, scores: torch.Tensor,
                         workspace: torch.Tensor, stream=None) -> None:
    """q_win [B,Hq,S_obs,d] (contiguous), k [B,Hkv,N,d] -> scores [B,Hkv,d] fp64."""
    B, Hq, S, d = q_win.shape
    _, Hkv, N, _ = k.shape
    if not q_win.is_contiguous() or scores.dtype != torch.float64:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_score_channels")
    _check(lib.think_score_channels(_ptr(q_win), _ptr(k), _strides3(k), B, Hq, Hkv, N, S, d,
                                    _dtype(k), _ptr(scores), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "think_score_channels")


def think_select_channels(scores: torch.Tensor, T: int, idx: torch.Tensor, stream=None) -> None:
    """scores [B,Hkv,d] fp64 -> idx [B,Hkv,T] int32 (ascending kept channels)."""
    B, Hkv, d = scores.shape
    if scores.dtype != torch.float64 or idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_select_channels")
    _check(lib.think_select_channels(_ptr(scores), B, Hkv, d, int(T), _ptr(idx), _stream(stream)),
           "think_select_channels")


def think_compact_keys(k: torch.Tensor, idx: torch.Tensor, k_pruned: torch.Tensor, ldk: int,
                       stream=None) -> None:
    """k [B,Hkv,N,d], idx [B,Hkv,T] -> k_pruned, element (b,h,t,n) at ((b*Hkv+h)*T+t)*ldk+n."""
    B, Hkv, N, d = k.shape
    T = idx.shape[-1]
    if idx.dtype != torch.int32 or k_pruned.dtype != k.dtype:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_compact_keys")
    _check(lib.think_compact_keys(_ptr(k), _strides3(k), B, Hkv, N, d, _dtype(k), _ptr(idx), T,
                                  _ptr(k_pruned), int(ldk), _stream(stream)), "think_compact_keys")


def think_append_keys(k_new: torch.Tensor, idx: torch.Tensor, k_pruned: torch.Tensor, ldk: int,
                      n_at: int, stream=None) -> None:
    """k_new [B,Hkv,n,d] -> K' columns [n_at, n_at + n) of every kept channel."""
    B, Hkv, n, d = k_new.shape
    T = idx.shape[-1]
    if idx.dtype != torch.int32 or k_pruned.dtype != k_new.dtype:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_append_keys")
    _check(lib.think_append_keys(_ptr(k_new), _strides3(k_new), B, Hkv, n, d, _dtype(k_new),
                                 _ptr(idx), T, _ptr(k_pruned), int(ldk), int(n_at), _stream(stream)),
           "think_append_keys")


def think_prune(q_win: torch.Tensor, k: torch.Tensor, T: int, scores: torch.Tensor,
                idx: torch.Tensor, k_pruned: torch.Tensor, ldk: int, workspace: torch.Tensor,
                stream=None) -> None:
    """Scores + top-T selection (one launch) then compaction (one launch)."""
    B, Hq, S, d = q_win.shape
    _, Hkv, N, _ = k.shape
    if (not q_win.is_contiguous() or scores.dtype != torch.float64 or idx.dtype != torch.int32
            or k_pruned.dtype != k.dtype):
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_prune")
    _check(lib.think_prune(_ptr(q_win), _ptr(k), _strides3(k), B, Hq, Hkv, N, S, d, _dtype(k),
                           int(T), _ptr(scores), _ptr(idx), _ptr(k_pruned), int(ldk),
                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream)), "think_prune")


def think_pruned_decode_attn(q: torch.Tensor, k_pruned: torch.Tensor, ldk: int, v: torch.Tensor,
                             idx: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                             scale: float | None = None, N: int | None = None,
                             stream=None) -> None:
    """q [B,Hq,d], thinner K (pitch ldk), v [B,Hkv,N,d], idx [B,Hkv,T] -> out [B,Hq,d] fp32."""
    B, Hq, d = q.shape
    _, Hkv, Nv, _ = v.shape
    N = Nv if N is None else N
    T = idx.shape[-1]
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if not q.is_contiguous() or out.dtype != torch.float32 or idx.dtype != torch.int32 \
            or not out.is_contiguous() or tuple(out.shape) != (B, Hq, d) \
            or not (q.is_cuda and k_pruned.is_cuda and v.is_cuda and idx.is_cuda and out.is_cuda):
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_pruned_decode_attn")
    _check(lib.think_pruned_decode_attn(_ptr(q), _ptr(k_pruned), int(ldk), _ptr(v), _strides3(v),
                                        _ptr(idx), B, Hq, Hkv, N, d, T, _dtype(q), float(scale),
                                        _ptr(out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "think_pruned_decode_attn")


def think_pruned_decode_attn_noalloc(q: torch.Tensor, k_pruned: torch.Tensor, ldk: int,
                                     v: torch.Tensor, idx: torch.Tensor, out: torch.Tensor,
                                     scale: float | None = None, N: int | None = None,
                                     stream=None) -> None:
    """think_pruned_decode_attn with the library's built-in scratch instead of a
    caller workspace (for callers that may not allocate device memory)."""
    B, Hq, d = q.shape
    _, Hkv, Nv, _ = v.shape
    N = Nv if N is None else N
    T = idx.shape[-1]
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if not q.is_contiguous() or out.dtype != torch.float32 or idx.dtype != torch.int32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_pruned_decode_attn_noalloc")
    _check(lib.think_pruned_decode_attn_noalloc(_ptr(q), _ptr(k_pruned), int(ldk), _ptr(v),
                                                _strides3(v), _ptr(idx), B, Hq, Hkv, N, d, T,
                                                _dtype(q), float(scale), _ptr(out), _stream(stream)),
           "think_pruned_decode_attn_noalloc")


def think_q4_ld(N: int) -> int:
    return lib.think_q4_ld(int(N))


def think_q4_groups_bytes(B: int, Hkv: int, N: int, T: int) -> int:
    return lib.think_q4_groups_bytes(B, Hkv, int(N), T)


def think_quantize_keys_q4(k_pruned: torch.Tensor, ldk: int, N: int, codes: torch.Tensor, ldq: int,
                           groups: torch.Tensor, stream=None) -> None:
    """bf16 K' [B,Hkv,T,ldk] -> codes [B,Hkv,T,ldq] uint8 and groups (scale, mn) fp32."""
    B, Hkv, T, _ = k_pruned.shape
    if k_pruned.dtype != torch.bfloat16 or codes.dtype != torch.uint8 or groups.dtype != torch.float32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_quantize_keys_q4")
    _check(lib.think_quantize_keys_q4(_ptr(k_pruned), int(ldk), B, Hkv, int(N), T, _ptr(codes), int(ldq),
                                      _ptr(groups), _stream(stream)), "think_quantize_keys_q4")


def think_pruned_decode_attn_q4(q: torch.Tensor, codes: torch.Tensor, ldq: int, groups: torch.Tensor,
                                v: torch.Tensor, idx: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                                N: int, scale: float | None = None, stream=None) -> None:
    """Decode attention over the 4-bit thinner cache (keys = dequantised codes)."""
    B, Hq, d = q.shape
    _, Hkv, _, _ = v.shape
    T = idx.shape[-1]
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if (not q.is_contiguous() or q.dtype != torch.bfloat16 or v.dtype != torch.bfloat16
            or out.dtype != torch.float32 or idx.dtype != torch.int32):
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_pruned_decode_attn_q4")
    _check(lib.think_pruned_decode_attn_q4(_ptr(q), _ptr(codes), int(ldq), _ptr(groups), _ptr(v), _strides3(v),
                                           _ptr(idx), B, Hq, Hkv, int(N), d, T, float(scale), _ptr(out),
                                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "think_pruned_decode_attn_q4")


def think_ragged_rows(B: int, Hkv: int, T_max: int) -> int:
    return lib.think_ragged_rows(B, Hkv, T_max)


def think_select_adaptive(scores: torch.Tensor, tau: float, T_min: int, T_max: int, Th: torch.Tensor,
                          rowoff: torch.Tensor, idx: torch.Tensor, stream=None) -> None:
    """scores [B,Hkv,d] fp64 -> Th [B*Hkv], rowoff [B*Hkv+1], idx [rows] (int32, ragged layout)."""
    B, Hkv, d = scores.shape
    _check(lib.think_select_adaptive(_ptr(scores), B, Hkv, d, float(tau), int(T_min), int(T_max), _ptr(Th),
                                     _ptr(rowoff), _ptr(idx), _stream(stream)), "think_select_adaptive")


def think_prune_adaptive(q_win: torch.Tensor, k: torch.Tensor, tau: float, T_min: int, T_max: int,
                         scores: torch.Tensor, Th: torch.Tensor, rowoff: torch.Tensor, idx: torch.Tensor,
                         k_pruned: torch.Tensor, ldk: int, workspace: torch.Tensor, stream=None) -> None:
    """Scores, adaptive selection and ragged compaction (three launches): the
    outputs of think_score_channels + think_select_adaptive +
    think_compact_keys_ragged."""
    B, Hq, S, d = q_win.shape
    _, Hkv, N, _ = k.shape
    if not q_win.is_contiguous() or scores.dtype != torch.float64 or k_pruned.dtype != k.dtype:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_prune_adaptive")
    _check(lib.think_prune_adaptive(_ptr(q_win), _ptr(k), _strides3(k), B, Hq, Hkv, N, S, d, _dtype(k), float(tau),
                                    int(T_min), int(T_max), _ptr(scores), _ptr(Th), _ptr(rowoff), _ptr(idx),
                                    _ptr(k_pruned), int(ldk), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "think_prune_adaptive")


def think_compact_keys_ragged(k: torch.Tensor, idx: torch.Tensor, Th: torch.Tensor, rowoff: torch.Tensor,
                              T_max: int, k_pruned: torch.Tensor, ldk: int, stream=None) -> None:
    B, Hkv, N, d = k.shape
    _check(lib.think_compact_keys_ragged(_ptr(k), _strides3(k), B, Hkv, N, d, _dtype(k), _ptr(idx), _ptr(Th),
                                         _ptr(rowoff), int(T_max), _ptr(k_pruned), int(ldk), _stream(stream)),
           "think_compact_keys_ragged")


def think_pruned_decode_attn_ragged(q: torch.Tensor, k_pruned: torch.Tensor, ldk: int, v: torch.Tensor,
                                    idx: torch.Tensor, Th: torch.Tensor, rowoff: torch.Tensor, T_max: int,
                                    out: torch.Tensor, workspace: torch.Tensor, N: int | None = None,
                                    scale: float | None = None, stream=None) -> None:
    B, Hq, d = q.shape
    _, Hkv, Nv, _ = v.shape
    N = Nv if N is None else N
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if not q.is_contiguous() or out.dtype != torch.float32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_pruned_decode_attn_ragged")
    _check(lib.think_pruned_decode_attn_ragged(_ptr(q), _ptr(k_pruned), int(ldk), _ptr(v), _strides3(v), _ptr(idx),
                                               _ptr(Th), _ptr(rowoff), int(T_max), B, Hq, Hkv, int(N), d,
                                               float(scale), _ptr(out), _ptr(workspace),
                                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "think_pruned_decode_attn_ragged")


class AdaptiveCache:
    """Device buffers of one layer pruned with a kept width per head (ragged
    thinner K).  Allocates with torch on construction, then only calls the C
    entry points: prune = scores, adaptive selection, ragged compaction
    (think_prune_adaptive)."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, tau: float, T_min: int, T_max: int, d: int = 128,
                 dtype: torch.dtype = torch.bfloat16, device="cuda"):
        self.B, self.Hq, self.Hkv, self.N, self.d, self.dtype = B, Hq, Hkv, N, d, dtype
        self.tau, self.T_min, self.T_max = tau, T_min, T_max
        self.ldk = think_pruned_ld(N, dtype)
        rows = think_ragged_rows(B, Hkv, T_max)
        self.scores = torch.empty((B, Hkv, d), dtype=torch.float64, device=device)
        self.Th = torch.empty(B * Hkv, dtype=torch.int32, device=device)
        self.rowoff = torch.empty(B * Hkv + 1, dtype=torch.int32, device=device)
        self.idx = torch.empty(rows, dtype=torch.int32, device=device)
        self.k_pruned = torch.empty((rows, self.ldk), dtype=dtype, device=device)
        self.score_ws = torch.zeros(max(256, think_score_workspace_size(B, Hq, Hkv, N, d)),
                                    dtype=torch.uint8, device=device)
        self.decode_ws = torch.zeros(max(256, think_decode_workspace_size(B, Hq, Hkv, N, d, dtype)),
                                     dtype=torch.uint8, device=device)

    def prune(self, q_win, k, stream=None):
        think_prune_adaptive(q_win, k, self.tau, self.T_min, self.T_max, self.scores, self.Th, self.rowoff,
                             self.idx, self.k_pruned, self.ldk, self.score_ws, stream)

    def prune_stepwise(self, q_win, k, stream=None):
        """The same prune through the three separate entry points."""
        think_score_channels(q_win, k, self.scores, self.score_ws, stream)
        think_select_adaptive(self.scores, self.tau, self.T_min, self.T_max, self.Th, self.rowoff, self.idx,
                              stream)
        think_compact_keys_ragged(k, self.idx, self.Th, self.rowoff, self.T_max, self.k_pruned, self.ldk, stream)

    def decode(self, q, v, out, scale=None, stream=None):
        think_pruned_decode_attn_ragged(q, self.k_pruned, self.ldk, v, self.idx, self.Th, self.rowoff, self.T_max,
                                        out, self.decode_ws, N=self.N, scale=scale, stream=stream)


def think_token_mass_workspace_size(B: int, Hq: int, Hkv: int, N: int, S_obs: int) -> int:
    return lib.think_token_mass_workspace_size(B, Hq, Hkv, int(N), S_obs)


def think_token_mass(q_win: torch.Tensor, k: torch.Tensor, mass: torch.Tensor, workspace: torch.Tensor,
                     scale: float | None = None, stream=None) -> None:
    """q_win [B,Hq,S,d], k [B,Hkv,N,d] (bf16) -> mass [B,Hkv,N] fp32 (window attention mass)."""
    B, Hq, S, d = q_win.shape
    _, Hkv, N, _ = k.shape
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if not q_win.is_contiguous() or mass.dtype != torch.float32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_token_mass")
    _check(lib.think_token_mass(_ptr(q_win), _ptr(k), _strides3(k), B, Hq, Hkv, N, S, d, _dtype(k), float(scale),
                                _ptr(mass), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)), "think_token_mass")


def think_select_tokens_workspace_size(B: int, Hkv: int, N: int) -> int:
    return int(lib.think_select_tokens_workspace_size(B, Hkv, N))


def think_select_tokens(mass: torch.Tensor, M: int, kept: torch.Tensor, workspace: torch.Tensor,
                        stream=None) -> None:
    """mass [B,Hkv,N] fp32 -> kept [B,Hkv,M] int32 (largest mass, ties to the lower index, ascending)."""
    B, Hkv, N = mass.shape
    if not mass.is_contiguous() or mass.dtype != torch.float32 or kept.dtype != torch.int32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_select_tokens")
    _check(lib.think_select_tokens(_ptr(mass), B, Hkv, N, int(M), _ptr(kept), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "think_select_tokens")


def think_gather_tokens(x: torch.Tensor, kept: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """x [B,Hkv,N,d], kept [B,Hkv,M] -> out [B,Hkv,M,d] (contiguous)."""
    B, Hkv, N, d = x.shape
    M = kept.shape[-1]
    if not out.is_contiguous() or out.dtype != x.dtype or kept.dtype != torch.int32:
        raise ThinkError(THINK_ERR_INVALID_ARG, "think_gather_tokens")
    _check(lib.think_gather_tokens(_ptr(x), _strides3(x), B, Hkv, N, d, _dtype(x), _ptr(kept), int(M), _ptr(out),
                                   _stream(stream)), "think_gather_tokens")


class EvictedCache:
    """Token eviction then channel pruning of one layer: keep the M tokens of
    largest window attention mass per head, gather their K and V rows, prune
    the channels of the kept keys (a PrunedCache over M tokens).  Allocates
    with torch on construction, then only calls the C entry points."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, S_obs: int, M: int, T: int, d: int = 128,
                 dtype: torch.dtype = torch.bfloat16, device="cuda"):
        self.B, self.Hq, self.Hkv, self.N, self.M, self.T, self.d = B, Hq, Hkv, N, M, T, d
        self.mass = torch.empty((B, Hkv, N), dtype=torch.float32, device=device)
        self.kept = torch.empty((B, Hkv, M), dtype=torch.int32, device=device)
        self.k_kept = torch.empty((B, Hkv, M, d), dtype=dtype, device=device)
        self.v_kept = torch.empty((B, Hkv, M, d), dtype=dtype, device=device)
        self.mass_ws = torch.zeros(max(256, think_token_mass_workspace_size(B, Hq, Hkv, N, S_obs)),
                                   dtype=torch.uint8, device=device)
        self.select_ws = torch.zeros(max(256, think_select_tokens_workspace_size(B, Hkv, N)),
                                     dtype=torch.uint8, device=device)
        self.pruned = PrunedCache(B, Hq, Hkv, M, T, d, dtype=dtype, device=device)

    def prune(self, q_win, k, v, stream=None):
        think_token_mass(q_win, k, self.mass, self.mass_ws, stream=stream)
        think_select_tokens(self.mass, self.M, self.kept, self.select_ws, stream)
        think_gather_tokens(k, self.kept, self.k_kept, stream)
        think_gather_tokens(v, self.kept, self.v_kept, stream)
        self.pruned.prune(q_win, self.k_kept, stream)

    def decode(self, q, out, scale=None, stream=None):
        self.pruned.decode(q, self.v_kept, out, scale=scale, stream=stream)


def think_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(lib.think_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "think_workspace_init")


def think_read_device_status(workspace: torch.Tensor, stream=None) -> int:
    st = ctypes.c_uint32(0)
    _check(lib.think_read_device_status(_ptr(workspace), ctypes.byref(st), _stream(stream)),
           "think_read_device_status")
    return st.value


def think_noalloc_read_device_status(stream=None) -> int:
    """Status word of the last no-allocation decode on the current device
    (synchronises the stream)."""
    st = ctypes.c_uint32(0)
    _check(lib.think_noalloc_read_device_status(ctypes.byref(st), _stream(stream)),
           "think_noalloc_read_device_status")
    return st.value


class PrunedCache:
    """Device buffers of one pruned layer: kept channels, thinner K, workspaces.

    A convenience holder for callers of the functions above; it allocates with
    torch on construction and then only calls the C entry points.  ``N`` is
    the cache length at prune time, ``capacity`` (>= N) the longest the cache
    may grow to by ``append``; ``n`` is the current length."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, T: int, d: int = 128,
                 dtype: torch.dtype = torch.bfloat16, device="cuda", capacity: int | None = None):
        self.B, self.Hq, self.Hkv, self.N, self.T, self.d, self.dtype = B, Hq, Hkv, N, T, d, dtype
        self.capacity = N if capacity is None else max(N, capacity)
        self.n = N
        self.ldk = think_pruned_ld(self.capacity, dtype)
        self.scores = torch.empty((B, Hkv, d), dtype=torch.float64, device=device)
        self.idx = torch.empty((B, Hkv, T), dtype=torch.int32, device=device)
        self.k_pruned = torch.empty((B, Hkv, T, self.ldk), dtype=dtype, device=device)
        self.score_ws = torch.zeros(max(256, think_score_workspace_size(B, Hq, Hkv, N, d)),
                                    dtype=torch.uint8, device=device)
        self.decode_ws = torch.zeros(
            max(256, think_decode_workspace_size(B, Hq, Hkv, self.capacity, d, dtype)),
            dtype=torch.uint8, device=device)

    def prune(self, q_win, k, stream=None):
        think_prune(q_win, k, self.T, self.scores, self.idx, self.k_pruned, self.ldk,
                    self.score_ws, stream)
        self.n = self.N

    def append(self, k_new, stream=None):
        """Append the keys of k_new.shape[2] new tokens (compacted with the kept channels)."""
        think_append_keys(k_new, self.idx, self.k_pruned, self.ldk, self.n, stream)
        self.n += k_new.shape[2]

    def prune_stepwise(self, q_win, k, stream=None):
        """The same prune through the three separate entry points."""
        think_score_channels(q_win, k, self.scores, self.score_ws, stream)
        think_select_channels(self.scores, self.T, self.idx, stream)
        think_compact_keys(k, self.idx, self.k_pruned, self.ldk, stream)
        self.n = self.N

    def quantize_q4(self, stream=None):
        """Build the 4-bit thinner cache (codes, groups) from the current K' (bf16)."""
        if not hasattr(self, "codes"):
            self.ldq = think_q4_ld(self.capacity)
            self.codes = torch.zeros((self.B, self.Hkv, self.T, self.ldq), dtype=torch.uint8,
                                     device=self.k_pruned.device)
            T2 = (self.T + 1) // 2 * 2
            self.groups = torch.zeros((self.B, self.Hkv, self.ldq // 64, T2, 2), dtype=torch.float32,
                                      device=self.k_pruned.device)
        think_quantize_keys_q4(self.k_pruned, self.ldk, self.n, self.codes, self.ldq, self.groups, stream)

    def decode_q4(self, q, v, out, scale=None, stream=None):
        """Attend over the current n tokens with the 4-bit thinner cache."""
        think_pruned_decode_attn_q4(q, self.codes, self.ldq, self.groups, v, self.idx, out, self.decode_ws,
                                    N=self.n, scale=scale, stream=stream)

    def decode(self, q, v, out, scale=None, stream=None):
        """Attend over the current n tokens (v holds at least n token rows).

        Decode steps are short (a few microseconds on the device for short
        caches), so the host path matters: the arguments that do not change
        between steps (this cache's buffers, V's address, shape and strides,
        the scale, the shapes of q and out) are checked and marshalled on the
        first call, and later calls with the same V tensor and scale only check
        q and out against them and pass their addresses."""
        f = getattr(self, "_dfast", None)
        if f is not None and v is f[0] and scale == f[1] and v.data_ptr() == f[2] and v.shape == f[3] \
                and q.shape == f[4] and out.shape == f[4] and q.dtype == self.dtype \
                and out.dtype == torch.float32 and q.is_contiguous() and out.is_contiguous() \
                and q.is_cuda and out.is_cuda:
            rc = lib.think_pruned_decode_attn(
                q.data_ptr(), f[5], f[6], f[2], f[7], f[8], self.B, self.Hq, self.Hkv, self.n, self.d, self.T,
                f[9], f[10], out.data_ptr(), f[11], f[12],
                _raw_stream(f[13]) if stream is None else stream.cuda_stream)
            if rc != THINK_OK:
                raise ThinkError(rc, "think_pruned_decode_attn")
            return
        think_pruned_decode_attn(q, self.k_pruned, self.ldk, v, self.idx, out, self.decode_ws,
                                 scale=scale, N=self.n, stream=stream)
        d = q.shape[-1]
        self._dfast = (v, scale, v.data_ptr(), v.shape, q.shape, self.k_pruned.data_ptr(), int(self.ldk),
                       _strides3(v), self.idx.data_ptr(), _dtype(q),
                       float(1.0 / float(d) ** 0.5 if scale is None else scale),
                       self.decode_ws.data_ptr(), self.decode_ws.numel(), self.k_pruned.device.index)

"""ctypes binding of the C ABI in include/attn.h.

Argument marshalling only: tensors are turned into device pointers and sizes,
the status code is turned into an exception. Every step of the computation runs
in the CUDA library; there is no fallback path. If the library has not been
built, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

# HASB_DEBUG=1 loads the index-checking debug build (-DATTN_DEBUG) instead
_SO_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libattn_sm100_debug.so" if os.environ.get("HASB_DEBUG") == "1" else "libattn_sm100.so")
_LIB = None

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4
ATTN_ERR_SCRATCH_LIMIT = 5

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_CHUNK = 2

NORM_NONE = 0
NORM_HEAD = 1
NORM_INNER = 2

ROPE_NONE = 0
ROPE_INTERLEAVED = 1
ROPE_SPLIT = 2

DTYPE_CODES = {torch.bfloat16: 0, torch.float16: 1}

# name -> (restype, argtypes) of every exported function
_SIGNATURES = {
    "attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 +
                 [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_fwd_host": (ctypes.c_int, [ctypes.c_void_p] * 10 + [ctypes.c_int] * 6 +
                      [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_host_chunks": (ctypes.c_int, [ctypes.c_int] * 4 + [ctypes.c_void_p]),
    "attn_qk_prologue": (ctypes.c_int, [ctypes.c_void_p] * 8 + [ctypes.c_int] * 7 +
                         [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_stream_update": (ctypes.c_int, [ctypes.c_void_p] * 10 + [ctypes.c_int] * 7 +
                           [ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_fwd_cache": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 +
                       [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_splitkv_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 5),
    "attn_fwd_splitkv": (ctypes.c_int, [ctypes.c_void_p] * 6 + [ctypes.c_size_t] + [ctypes.c_int] * 7 +
                         [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                          ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]),
    "attn_fwd_splitkv_static": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 +
                                [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]),
    "attn_fwd_window": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 +
                        [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                         ctypes.c_void_p]),
    "attn_fp8_cast": (ctypes.c_int, [ctypes.c_void_p] * 2 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]),
    "attn_fp8_cast_vt": (ctypes.c_int, [ctypes.c_void_p] * 2 + [ctypes.c_int] * 6 + [ctypes.c_void_p]),
    "attn_fwd_fp8": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 +
                     [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_fp8_quantize_tokens": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p]),
    "attn_fp8_quantize_vt": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p]),
    "attn_fwd_fp8_scaled": (ctypes.c_int, [ctypes.c_void_p] * 8 + [ctypes.c_int] * 9 +
                            [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "attn_rope_after_cache": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 2 + [ctypes.c_void_p] +
                              [ctypes.c_int] * 9 + [ctypes.c_void_p]),
    "attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "attn_debug_fault_site": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]),
    "attn_debug_build": (ctypes.c_int, []),
    "attn_device_fault": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]),
    "attn_set_wait_timeout_ns": (ctypes.c_int, [ctypes.c_ulonglong]),
    "attn_selftest_mma": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p]),
    "attn_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_ulonglong, ctypes.c_void_p]),
    "attn_selftest_exp2": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def library_path() -> str:
    return _SO_PATH


def lib() -> ctypes.CDLL:
    """The loaded C library (loaded on first use)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_SO_PATH):
            raise RuntimeError(
                f"CUDA library {_SO_PATH} is missing; build it with "
                "`python -m head_attention_streaming_b200.build`")
        L = ctypes.CDLL(_SO_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    try:
        return lib().attn_status_string(int(status)).decode()
    except Exception:  # library missing: still format the error
        return "unknown"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: float | None = None,
             causal: int = MASK_NONE, kv_offset: int = 0, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Fused attention forward through ``attn_fwd`` of the C ABI.

    q: [B, Lq, Hq, d]; k, v: [B, Lk, Hkv, d]; CUDA, contiguous, bf16 or fp16.
    causal: 0 none, 1 causal (key j <= kv_offset + i), 2 streaming chunk
    (key j < kv_offset + Lq). Returns ``(out, lse)`` with out [B, Lq, Hq, d]
    in q's dtype and lse [B, Hq, Lq] float32 (None if return_lse is False and
    no lse buffer was given).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in DTYPE_CODES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype, bf16 or fp16")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    B, Lq, Hq, d = q.shape
    Bk, Lk, Hkv, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("batch and head_dim of q and k/v must match")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor shaped and typed like q")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    elif lse is not None and (lse.shape != (B, Hq, Lq) or lse.dtype != torch.float32
                              or not lse.is_contiguous() or not lse.is_cuda):
        raise ValueError("lse must be a contiguous float32 CUDA tensor [B, Hq, Lq]")
    st = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Lq, Lk, Hq, Hkv, d,
                        float(scale), int(causal), int(kv_offset), DTYPE_CODES[q.dtype],
                        _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")
    return out, lse


def _check_f32(name, t, numel, device):
    if t is None:
        return
    if (not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() or t.numel() != numel
            or t.device != device):
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of {numel} elements")


def qk_prologue(q: torch.Tensor, k: torch.Tensor | None = None, *, norm_scope: int = NORM_NONE,
                eps: float = 1e-6, gamma_q: torch.Tensor | None = None,
                gamma_k: torch.Tensor | None = None, rope_style: int = ROPE_NONE,
                angles_q: torch.Tensor | None = None, angles_k: torch.Tensor | None = None,
                out_q: torch.Tensor | None = None, out_k: torch.Tensor | None = None,
                stream=None):
    """Q/K RMSNorm then RoPE through ``attn_qk_prologue`` of the C ABI.

    q: [B, Lq, Hq, d], k: [B, Lk, Hkv, d] or None (CUDA, contiguous, bf16/fp16).
    gamma_*: float32 [d] (head scope) or [H*d] (inner scope), None = ones.
    angles_*: float32 [L, d] (the expanded rope_freqs table), required iff
    rope_style != ROPE_NONE. ``out_q`` / ``out_k`` may be the inputs (in place);
    by default new tensors. Returns ``(q_out, k_out)``.
    """
    tensors = [("q", q)] + ([("k", k)] if k is not None else [])
    for name, t in tensors:
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype not in DTYPE_CODES:
            raise ValueError(f"{name} must be a contiguous 4-D bf16/fp16 CUDA tensor")
    B, Lq, Hq, d = q.shape
    Lk, Hkv = 0, 0
    if k is not None:
        if k.dtype != q.dtype or k.shape[0] != B or k.shape[3] != d:
            raise ValueError("k must share q's dtype, batch and head_dim")
        Lk, Hkv = k.shape[1], k.shape[2]
    wq = d if norm_scope == NORM_HEAD else Hq * d
    wk = d if norm_scope == NORM_HEAD else Hkv * d
    _check_f32("gamma_q", gamma_q, wq, q.device)
    _check_f32("gamma_k", gamma_k, wk, q.device)
    _check_f32("angles_q", angles_q, Lq * d, q.device)
    _check_f32("angles_k", angles_k, Lk * d, q.device)
    if out_q is None:
        out_q = torch.empty_like(q)
    if k is not None and out_k is None:
        out_k = torch.empty_like(k)
    for name, o, ref in (("out_q", out_q, q), ("out_k", out_k, k)):
        if ref is not None and (o.shape != ref.shape or o.dtype != ref.dtype or not o.is_cuda
                                or not o.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor shaped and typed like its input")
    st = lib().attn_qk_prologue(_ptr(q), _ptr(out_q), _ptr(k), _ptr(out_k if k is not None else None),
                                _ptr(gamma_q), _ptr(gamma_k), _ptr(angles_q), _ptr(angles_k),
                                B, Lq, Lk, Hq, Hkv, d, int(norm_scope), float(eps), int(rope_style),
                                DTYPE_CODES[q.dtype], _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_qk_prologue")
    return out_q, (out_k if k is not None else None)


def stream_update(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  slot: int, *, q: torch.Tensor | None = None, q_out: torch.Tensor | None = None,
                  norm_scope: int = NORM_NONE, eps: float = 1e-6, gamma_q=None, gamma_k=None,
                  rope_style: int = ROPE_NONE, angles_q=None, angles_k=None, stream=None):
    """Write the chunk's K (normalised and rotated) and V into cache slots
    ``slot .. slot + L - 1`` and, when ``q`` is given, the query prologue,
    through ``attn_stream_update`` of the C ABI. Returns ``q_out`` (or None).

    k, v: [B, L, Hkv, d]; k_cache, v_cache: [B, S, Hkv, d]; q: [B, L, Hq, d].
    """
    for name, t in (("k", k), ("v", v), ("k_cache", k_cache), ("v_cache", v_cache)) + \
            ((("q", q),) if q is not None else ()):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype not in DTYPE_CODES:
            raise ValueError(f"{name} must be a contiguous 4-D bf16/fp16 CUDA tensor")
    B, L, Hkv, d = k.shape
    if v.shape != k.shape or k_cache.shape != v_cache.shape or k_cache.shape[0] != B or \
            k_cache.shape[2:] != (Hkv, d) or len({t.dtype for t in (k, v, k_cache, v_cache)}) != 1:
        raise ValueError("k, v and the caches must agree in batch, heads, head_dim and dtype")
    S = k_cache.shape[1]
    Hq = 0
    if q is not None:
        if q.dtype != k.dtype or q.shape[0] != B or q.shape[1] != L or q.shape[3] != d:
            raise ValueError("q must be [B, L, Hq, d] in k's dtype")
        Hq = q.shape[2]
        if q_out is None:
            q_out = torch.empty_like(q)
    wq = d if norm_scope == NORM_HEAD else Hq * d
    wk = d if norm_scope == NORM_HEAD else Hkv * d
    _check_f32("gamma_q", gamma_q, wq, k.device)
    _check_f32("gamma_k", gamma_k, wk, k.device)
    _check_f32("angles_q", angles_q, L * d, k.device)
    _check_f32("angles_k", angles_k, L * d, k.device)
    st = lib().attn_stream_update(_ptr(q), _ptr(q_out), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(gamma_q), _ptr(gamma_k), _ptr(angles_q), _ptr(angles_k), B, L, S,
                                  int(slot), Hq, Hkv, d, int(norm_scope), float(eps), int(rope_style),
                                  DTYPE_CODES[k.dtype], _stream_handle(stream, k.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_stream_update")
    return q_out


def attn_fwd_cache(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, Lk: int, *,
                   scale: float | None = None, causal: int = MASK_NONE, kv_offset: int = 0,
                   out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                   return_lse: bool = True, stream=None):
    """``attn_fwd`` over the first ``Lk`` tokens of [B, S, Hkv, d] caches
    (``attn_fwd_cache`` of the C ABI). Returns ``(out, lse)``."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in DTYPE_CODES or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("q and the caches must share one dtype, bf16 or fp16")
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    B, Lq, Hq, d = q.shape
    S, Hkv = k_cache.shape[1], k_cache.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_cache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, Lq, int(Lk),
                              S, Hq, Hkv, d, float(scale), int(causal), int(kv_offset),
                              DTYPE_CODES[q.dtype], _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_cache")
    return out, lse


def splitkv_workspace_bytes(B: int, Lq: int, Hq: int, d: int, n_splits: int) -> int:
    """Bytes of the float32 workspace attn_fwd_splitkv needs for n_splits ranges."""
    return int(lib().attn_splitkv_workspace_bytes(B, Lq, Hq, d, n_splits))


def attn_fwd_splitkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_splits: int = 0,
                     scale: float | None = None, causal: int = MASK_NONE, kv_offset: int = 0,
                     workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Key-split attention forward through ``attn_fwd_splitkv`` of the C ABI
    (masks 0, 1, 2). ``workspace`` (float32, CUDA) is allocated here when not
    given, sized for the split count the library chooses. Returns
    ``(out, lse, splits_used)``.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in DTYPE_CODES or k.dtype != q.dtype or v.dtype != q.dtype or k.shape != v.shape:
        raise ValueError("q, k, v must share one dtype (bf16/fp16); k and v one shape")
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    used = ctypes.c_int(0)
    args = (B, Lq, Lk, Hq, Hkv, d, float(scale), int(causal), int(kv_offset), DTYPE_CODES[q.dtype])
    if workspace is None:
        # the largest split count the library could choose: one per 128-key tile, at most 32
        tiles = (Lk + 127) // 128
        cap = n_splits if n_splits > 0 else min(tiles, 32)
        workspace = torch.empty(max(1, splitkv_workspace_bytes(B, Lq, Hq, d, max(1, cap)) // 4),
                                dtype=torch.float32, device=q.device)
    elif not workspace.is_cuda or workspace.dtype != torch.float32 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous float32 CUDA tensor")
    st = lib().attn_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(workspace),
                                workspace.numel() * 4, int(n_splits), *args[:9], args[9],
                                ctypes.byref(used), _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_splitkv")
    return out, lse, used.value


def attn_fwd_splitkv_static(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_splits: int = 0,
                            scale: float | None = None, causal: int = MASK_NONE, kv_offset: int = 0,
                            out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                            return_lse: bool = True, stream=None):
    """Key-split attention through ``attn_fwd_splitkv_static``: the library's
    own scratch, no workspace, nothing allocated by the call (``out`` and
    ``lse`` are allocated here only when not given). Returns ``(out, lse, splits_used)``."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in DTYPE_CODES or k.dtype != q.dtype or v.dtype != q.dtype or k.shape != v.shape:
        raise ValueError("q, k, v must share one dtype (bf16/fp16); k and v one shape")
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    used = ctypes.c_int(0)
    st = lib().attn_fwd_splitkv_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), int(n_splits),
                                       B, Lq, Lk, Hq, Hkv, d, float(scale), int(causal), int(kv_offset),
                                       DTYPE_CODES[q.dtype], ctypes.byref(used),
                                       _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_splitkv_static")
    return out, lse, used.value


def attn_fwd_window(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, window=(-1, -1),
                    scale: float | None = None, kv_offset: int = 0, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Sliding-window attention through ``attn_fwd_window`` of the C ABI: row i
    (key position kv_offset + i) sees keys within ``window = (left, right)`` of
    it, -1 = unbounded on that side. Returns ``(out, lse)``."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in DTYPE_CODES or k.dtype != q.dtype or v.dtype != q.dtype or k.shape != v.shape:
        raise ValueError("q, k, v must share one dtype (bf16/fp16); k and v one shape")
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    left, right = window
    st = lib().attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Lq, Lk, Hq, Hkv, d,
                               float(scale), int(left), int(right), int(kv_offset), DTYPE_CODES[q.dtype],
                               _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_window")
    return out, lse


E4M3 = torch.float8_e4m3fn


def _check_cuda(name, t, dim):
    if not t.is_cuda or not t.is_contiguous() or t.dim() != dim:
        raise ValueError(f"{name} must be a contiguous {dim}-D CUDA tensor")


def fp8_cast(x: torch.Tensor, *, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """e4m3 copy of a 16-bit tensor (round to nearest even, saturated at +-448)
    through ``attn_fp8_cast``; x.numel() must be a multiple of 8."""
    _check_cuda("x", x, x.dim())
    if x.dtype not in DTYPE_CODES:
        raise ValueError("x must be bf16 or fp16")
    if out is None:
        out = torch.empty(x.shape, dtype=E4M3, device=x.device)
    elif out.dtype != E4M3 or out.numel() != x.numel() or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous float8_e4m3fn CUDA tensor with x's size")
    st = lib().attn_fp8_cast(_ptr(x), _ptr(out), x.numel(), DTYPE_CODES[x.dtype],
                             _stream_handle(stream, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fp8_cast")
    return out


def fp8_cast_vt(v: torch.Tensor, *, pitch: int | None = None, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """V [B, Lk, Hkv, d] (16-bit) to e4m3 V^T [B, Hkv, d, pitch] through
    ``attn_fp8_cast_vt``; pitch defaults to Lk rounded up to 16. Bytes at keys
    >= Lk of a row are left as they were."""
    _check_cuda("v", v, 4)
    if v.dtype not in DTYPE_CODES:
        raise ValueError("v must be bf16 or fp16")
    B, Lk, Hkv, d = v.shape
    if pitch is None:
        pitch = (Lk + 15) // 16 * 16
    if out is None:
        out = torch.empty((B, Hkv, d, pitch), dtype=E4M3, device=v.device)
    elif (out.dtype != E4M3 or tuple(out.shape) != (B, Hkv, d, pitch) or not out.is_contiguous()
          or not out.is_cuda):
        raise ValueError("out must be a contiguous float8_e4m3fn CUDA tensor [B, Hkv, d, pitch]")
    st = lib().attn_fp8_cast_vt(_ptr(v), _ptr(out), B, Lk, Hkv, d, int(pitch), DTYPE_CODES[v.dtype],
                                _stream_handle(stream, v.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fp8_cast_vt")
    return out


def attn_fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, vt8: torch.Tensor, *, scale: float | None = None,
                 causal: int = MASK_NONE, kv_offset: int = 0, out: torch.Tensor | None = None,
                 lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Attention on e4m3 operands through ``attn_fwd_fp8``: q8 [B, Lq, Hq, d],
    k8 [B, Lk, Hkv, d], vt8 [B, Hkv, d, pitch] (``fp8_cast_vt``), all
    float8_e4m3fn. Returns ``(out, lse)``, out bf16 [B, Lq, Hq, d]."""
    for name, t in (("q8", q8), ("k8", k8), ("vt8", vt8)):
        _check_cuda(name, t, 4)
        if t.dtype != E4M3:
            raise ValueError(f"{name} must be float8_e4m3fn")
    B, Lq, Hq, d = q8.shape
    Bk, Lk, Hkv, dk = k8.shape
    if Bk != B or dk != d or tuple(vt8.shape[:3]) != (B, Hkv, d):
        raise ValueError("q8, k8, vt8 shapes disagree")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Lq, Hq, d), dtype=torch.bfloat16, device=q8.device)
    elif (out.dtype != torch.bfloat16 or tuple(out.shape) != (B, Lq, Hq, d) or not out.is_contiguous()
          or not out.is_cuda):
        raise ValueError("out must be a contiguous bf16 CUDA tensor [B, Lq, Hq, d]")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q8.device)
    st = lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(out), _ptr(lse), B, Lq, Lk,
                            vt8.shape[3], Hq, Hkv, d, float(scale), int(causal), int(kv_offset),
                            _stream_handle(stream, q8.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return out, lse


def fp8_quantize_tokens(x: torch.Tensor, *, s_pitch: int | None = None, out: torch.Tensor | None = None,
                        scales: torch.Tensor | None = None, stream=None):
    """Per-token scaled e4m3 codes of x [B, L, H, d] through
    ``attn_fp8_quantize_tokens``. Returns (codes [B, L, H, d] float8_e4m3fn,
    scales [B, H, s_pitch] float32; s_pitch defaults to L rounded up to 4)."""
    _check_cuda("x", x, 4)
    if x.dtype not in DTYPE_CODES:
        raise ValueError("x must be bf16 or fp16")
    B, L, H, d = x.shape
    if s_pitch is None:
        s_pitch = (L + 3) // 4 * 4
    if out is None:
        out = torch.empty(x.shape, dtype=E4M3, device=x.device)
    elif out.dtype != E4M3 or out.shape != x.shape or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous float8_e4m3fn CUDA tensor shaped like x")
    if scales is None:
        scales = torch.empty((B, H, s_pitch), dtype=torch.float32, device=x.device)
    elif (scales.dtype != torch.float32 or tuple(scales.shape) != (B, H, s_pitch)
          or not scales.is_contiguous() or not scales.is_cuda):
        raise ValueError("scales must be a contiguous float32 CUDA tensor [B, H, s_pitch]")
    st = lib().attn_fp8_quantize_tokens(_ptr(x), _ptr(out), _ptr(scales), B, L, H, d, int(s_pitch),
                                        DTYPE_CODES[x.dtype], _stream_handle(stream, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fp8_quantize_tokens")
    return out, scales


def fp8_quantize_vt(v: torch.Tensor, *, pitch: int | None = None, out: torch.Tensor | None = None,
                    scales: torch.Tensor | None = None, stream=None):
    """Per-channel scaled e4m3 codes of V [B, Lk, Hkv, d], transposed to
    [B, Hkv, d, pitch], through ``attn_fp8_quantize_vt``. Returns (codes,
    scales [B, Hkv, d] float32)."""
    _check_cuda("v", v, 4)
    if v.dtype not in DTYPE_CODES:
        raise ValueError("v must be bf16 or fp16")
    B, Lk, Hkv, d = v.shape
    if pitch is None:
        pitch = (Lk + 15) // 16 * 16
    if out is None:
        out = torch.empty((B, Hkv, d, pitch), dtype=E4M3, device=v.device)
    elif (out.dtype != E4M3 or tuple(out.shape) != (B, Hkv, d, pitch) or not out.is_contiguous()
          or not out.is_cuda):
        raise ValueError("out must be a contiguous float8_e4m3fn CUDA tensor [B, Hkv, d, pitch]")
    if scales is None:
        scales = torch.empty((B, Hkv, d), dtype=torch.float32, device=v.device)
    elif (scales.dtype != torch.float32 or tuple(scales.shape) != (B, Hkv, d) or not scales.is_contiguous()
          or not scales.is_cuda):
        raise ValueError("scales must be a contiguous float32 CUDA tensor [B, Hkv, d]")
    st = lib().attn_fp8_quantize_vt(_ptr(v), _ptr(out), _ptr(scales), B, Lk, Hkv, d, int(pitch),
                                    DTYPE_CODES[v.dtype], _stream_handle(stream, v.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fp8_quantize_vt")
    return out, scales


def attn_fwd_fp8_scaled(q8: torch.Tensor, sq: torch.Tensor, k8: torch.Tensor, sk: torch.Tensor,
                        vt8: torch.Tensor, sv: torch.Tensor | None = None, *, scale: float | None = None,
                        causal: int = MASK_NONE, kv_offset: int = 0, out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Per-token scaled FP8 attention through ``attn_fwd_fp8_scaled``: codes
    and scales as ``fp8_quantize_tokens`` (Q, K) and ``fp8_quantize_vt`` (V;
    sv None: V cast without scales by ``fp8_cast_vt``). Returns ``(out, lse)``."""
    for name, t in (("q8", q8), ("k8", k8), ("vt8", vt8)):
        _check_cuda(name, t, 4)
        if t.dtype != E4M3:
            raise ValueError(f"{name} must be float8_e4m3fn")
    B, Lq, Hq, d = q8.shape
    Bk, Lk, Hkv, dk = k8.shape
    if Bk != B or dk != d or tuple(vt8.shape[:3]) != (B, Hkv, d):
        raise ValueError("q8, k8, vt8 shapes disagree")
    for name, t, lead in (("sq", sq, (B, Hq)), ("sk", sk, (B, Hkv))):
        _check_cuda(name, t, 3)
        if t.dtype != torch.float32 or tuple(t.shape[:2]) != lead:
            raise ValueError(f"{name} must be float32 [{lead[0]}, {lead[1]}, pitch]")
    if sv is not None:
        _check_cuda("sv", sv, 3)
        if sv.dtype != torch.float32 or tuple(sv.shape) != (B, Hkv, d):
            raise ValueError("sv must be float32 [B, Hkv, d]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Lq, Hq, d), dtype=torch.bfloat16, device=q8.device)
    elif (out.dtype != torch.bfloat16 or tuple(out.shape) != (B, Lq, Hq, d) or not out.is_contiguous()
          or not out.is_cuda):
        raise ValueError("out must be a contiguous bf16 CUDA tensor [B, Lq, Hq, d]")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q8.device)
    st = lib().attn_fwd_fp8_scaled(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(out),
                                   _ptr(lse), B, Lq, Lk, vt8.shape[3], sq.shape[2], sk.shape[2], Hq, Hkv, d,
                                   float(scale), int(causal), int(kv_offset), _stream_handle(stream, q8.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8_scaled")
    return out, lse


def rope_after_cache(q: torch.Tensor, k_cache: torch.Tensor, Lk: int, angles: torch.Tensor, *,
                     rope_style: int, q_row0: int = 0, k_rows: torch.Tensor | None = None,
                     q_out: torch.Tensor | None = None, k_rot: torch.Tensor | None = None, stream=None):
    """After-cache RoPE through ``attn_rope_after_cache``: q [B, Lq, Hq, d]
    rotated with angle rows q_row0.., and the first ``Lk`` slots of k_cache
    [B, S, Hkv, d] rotated into the same slots of k_rot with angle rows
    ``k_rows`` (int32 [Lk] on the device; None: the slot index). Returns
    ``(q_out, k_rot)``."""
    _check_cuda("q", q, 4)
    _check_cuda("k_cache", k_cache, 4)
    if q.dtype not in DTYPE_CODES or k_cache.dtype != q.dtype:
        raise ValueError("q and k_cache must share one dtype, bf16 or fp16")
    if not angles.is_cuda or angles.dtype != torch.float32 or not angles.is_contiguous() or angles.dim() != 2:
        raise ValueError("angles must be a contiguous float32 CUDA tensor [rows, d]")
    B, Lq, Hq, d = q.shape
    S, Hkv = k_cache.shape[1], k_cache.shape[2]
    if k_rows is not None and (not k_rows.is_cuda or k_rows.dtype != torch.int32
                               or not k_rows.is_contiguous() or k_rows.numel() < Lk):
        raise ValueError("k_rows must be a contiguous int32 CUDA tensor of at least Lk entries")
    if q_out is None:
        q_out = torch.empty_like(q)
    if k_rot is None:
        k_rot = torch.empty_like(k_cache)
    elif k_rot.shape != k_cache.shape or k_rot.dtype != k_cache.dtype or not k_rot.is_contiguous():
        raise ValueError("k_rot must be a contiguous tensor shaped and typed like k_cache")
    st = lib().attn_rope_after_cache(_ptr(q), _ptr(q_out), _ptr(k_cache), _ptr(k_rot), _ptr(angles),
                                     angles.shape[0], int(q_row0), _ptr(k_rows), B, Lq, int(Lk), S, Hq,
                                     Hkv, d, int(rope_style), DTYPE_CODES[q.dtype],
                                     _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_rope_after_cache")
    return q_out, k_rot


def attn_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev, *,
                  scale: float | None = None, causal: int = MASK_NONE, kv_offset: int = 0,
                  stream=None) -> None:
    """Queue host->device copies of q, k, v, the forward, and device->host copies of
    o (and lse) on ``stream`` through ``attn_fwd_host`` of the C ABI.

    Host tensors should be pinned CPU tensors; device tensors are the caller's
    staging buffers of the same shapes. Returns once queued.
    """
    B, Lq, Hq, d = q_host.shape
    _, Lk, Hkv, _ = k_host.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    for t in (q_host, k_host, v_host, o_host):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host operands must be contiguous CPU tensors")
    for t in (q_dev, k_dev, v_dev, o_dev):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("device buffers must be contiguous CUDA tensors")
    if q_host.dtype not in DTYPE_CODES:
        raise ValueError("dtype must be bf16 or fp16")
    st = lib().attn_fwd_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host), _ptr(lse_host),
                             _ptr(q_dev), _ptr(k_dev), _ptr(v_dev), _ptr(o_dev), _ptr(lse_dev),
                             B, Lq, Lk, Hq, Hkv, d, float(scale), int(causal), int(kv_offset),
                             DTYPE_CODES[q_host.dtype], _stream_handle(stream, q_dev.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_host")


def host_chunks(B: int, Lq: int, Hq: int, d: int) -> list[tuple[int, int, int, int]]:
    """The chunk plan of ``attn_fwd_host`` for these sizes: one (b0, nb, r0, n)
    per chunk, rows [r0, r0 + n) of batches [b0, b0 + nb)."""
    plan = (ctypes.c_int * 64)()
    n = lib().attn_host_chunks(int(B), int(Lq), int(Hq), int(d), plan)
    if n < 0:
        raise AttnError(-n, "attn_host_chunks")
    return [tuple(plan[4 * c:4 * c + 4]) for c in range(n)]


def device_fault(clear: bool = True) -> int:
    """Synchronize the device and return (and optionally clear) the fault bits."""
    bits = ctypes.c_uint(0)
    st = lib().attn_device_fault(ctypes.byref(bits), 1 if clear else 0)
    if st not in (ATTN_OK, ATTN_ERR_TIMEOUT):
        raise AttnError(st, "attn_device_fault")
    return int(bits.value)


def debug_fault_site(clear: bool = True) -> int:
    """Synchronize the device and return (optionally clearing) the site number
    of the first failed index check of the debug build (0: none; always 0 in
    the release build)."""
    site = ctypes.c_uint(0)
    st = lib().attn_debug_fault_site(ctypes.byref(site), 1 if clear else 0)
    if st != ATTN_OK:
        raise AttnError(st, "attn_debug_fault_site")
    return int(site.value)


def is_debug_build() -> bool:
    return bool(lib().attn_debug_build())


def set_wait_timeout_ns(ns: int) -> None:
    lib().attn_set_wait_timeout_ns(int(ns))


def selftest_mma(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """One 128x128 tile through the tensor-core path: returns (S, O) float32."""
    s_out = torch.empty((128, 128), dtype=torch.float32, device=q.device)
    o_out = torch.empty((128, 128), dtype=torch.float32, device=q.device)
    st = lib().attn_selftest_mma(_ptr(q), _ptr(k), _ptr(v), _ptr(s_out), _ptr(o_out),
                                 DTYPE_CODES[q.dtype], _stream_handle(None, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_mma")
    return s_out, o_out


def selftest_wait_timeout(timeout_ns: int, device=None) -> int:
    """Status of a launch whose only wait can never complete (expect ATTN_ERR_TIMEOUT)."""
    return int(lib().attn_selftest_wait_timeout(int(timeout_ns), _stream_handle(None, device)))


def selftest_exp2(x: torch.Tensor) -> torch.Tensor:
    """2^x through the kernel's FMA-pipe exponential (float32 CUDA tensor)."""
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    st = lib().attn_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream_handle(None, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_exp2")
    return y

"""Exact attention forward for B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI in ``include/fa_b200.h``.  It only
marshals arguments (device pointers, sizes, the current CUDA stream) and, when
the caller passes none, allocates the output, LSE and split-KV workspace with
torch; every step of the computation runs in the library's CUDA kernels.

There is no fallback: if ``libfa_b200.so`` is missing or fails to load, the
first call raises.  Build it with ``python -m
exact_attention_forward_flash_b200.build`` (or ``__graft_entry__.build()``).

Entry points (same names as the C ABI):

* ``fa_fwd(q, k, v, ...)`` -- dense [B, S, H, D];
* ``fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, ...)``
  -- packed [total, H, D] with cu_seqlens ("mgoin/tml-fa4" contract);
* ``fa_fwd_splitkv(q, k, v, ...)`` -- dense, keys split and merged by LSE.

Each returns ``(out, lse)``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_b200.so")

FA_OK = 0
_DTYPES = {torch.bfloat16: 0, torch.float16: 1}

_lib = None


class FAError(RuntimeError):
    """A library call returned a non-OK status."""

    def __init__(self, status: int, name: str, message: str):
        super().__init__(f"{name}: {message}")
        self.status = status
        self.name = name


class FaMods(ctypes.Structure):
    """Mirror of fa_mods (include/fa_b200.h)."""
    _fields_ = [("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("softcap", ctypes.c_float)]


def _mods(window, softcap):
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    return FaMods(wl, wr, float(softcap or 0.0))


def load_library(path: Optional[str] = None):
    """Load the shared library (raises if it is absent)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library not built: {path} is missing "
            "(run python -m exact_attention_forward_flash_b200.build)")
    lib = ctypes.CDLL(path)
    P, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                           i32, f32, P, P, i32, P]
    lib.fa_fwd.restype = i32
    lib.fa_fwd_varlen.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32,
                                  i32, i32, i32, i32, i32, i32, f32, P, i32, P]
    lib.fa_fwd_varlen.restype = i32
    lib.fa_splitkv_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.fa_splitkv_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_splitkv_default_splits.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.fa_splitkv_default_splits.restype = i32
    lib.fa_fwd_splitkv.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32,
                                   i32, i32, i32, f32, P, P, i32, i32, P,
                                   ctypes.c_size_t, P]
    lib.fa_fwd_splitkv.restype = i32
    lib.fa_fwd_splitkv_static.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32,
                                          i32, i32, i32, f32, P, P, i32, i32, P]
    lib.fa_fwd_splitkv_static.restype = i32
    M = ctypes.POINTER(FaMods)
    lib.fa_fwd_ex.argtypes = lib.fa_fwd.argtypes[:-1] + [M, P]
    lib.fa_fwd_ex.restype = i32
    lib.fa_fwd_varlen_ex.argtypes = lib.fa_fwd_varlen.argtypes[:-1] + [M, P]
    lib.fa_fwd_varlen_ex.restype = i32
    lib.fa_fwd_splitkv_ex.argtypes = lib.fa_fwd_splitkv.argtypes[:-1] + [M, P]
    lib.fa_fwd_splitkv_ex.restype = i32
    lib.fa_fwd_shard_partial.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                         i32, f32, P, P, P, i32, M, i32, P, ctypes.c_size_t, P]
    lib.fa_fwd_shard_partial.restype = i32
    lib.fa_combine_partials.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P]
    lib.fa_combine_partials.restype = i32
    lib.fa_watchdog_selftest.argtypes = [ctypes.c_ulonglong, P]
    lib.fa_watchdog_selftest.restype = i32
    lib.fa_selftest_exp2_fma.argtypes = [P, P, ctypes.c_longlong, P]
    lib.fa_selftest_exp2_fma.restype = i32
    lib.fa_check_device_error.argtypes = [ctypes.POINTER(i32), i32]
    lib.fa_check_device_error.restype = i32
    lib.fa_status_string.argtypes = [i32]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_error_message.argtypes = []
    lib.fa_last_error_message.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_version.restype = ctypes.c_char_p
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int):
    if status != FA_OK:
        lib = load_library()
        raise FAError(status, lib.fa_status_string(status).decode(),
                      lib.fa_last_error_message().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _dtype(q: torch.Tensor, name: str = "q") -> int:
    if q.dtype not in _DTYPES:
        raise TypeError(f"{name} must be bf16 or fp16, got {q.dtype}")
    return _DTYPES[q.dtype]


def _need_args(q, items):
    """One pass over a call's tensors.  Each (tensor, elements, dtype, name)
    must hold exactly `elements` elements (the library sees only pointers, so
    a smaller buffer would be read or written out of bounds on the device),
    lie on q's device, be contiguous and have `dtype`; None for elements or
    dtype skips that check.  q's device must be a CUDA device and the current
    one, since the library launches on the current device."""
    dev = q.get_device()
    for t, n, dt, name in items:
        if t is None:
            continue
        if n is not None and t.numel() != n:
            raise ValueError(f"{name} holds {t.numel()} elements; this call needs {n}")
        if t.get_device() != dev:
            raise ValueError(f"{name} is on {t.device}, not on {q.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dt is not None and t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
    if dev < 0:
        raise ValueError("all tensors must be CUDA tensors")
    if dev != torch.cuda.current_device():
        raise ValueError(f"the tensors are on cuda:{dev} but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _dense_shapes(q, k, v):
    qs, ks = q.shape, k.shape
    if len(qs) != 4 or len(ks) != 4 or ks[0] != qs[0] or ks[3] != qs[3] or v.shape != ks:
        raise ValueError("q [B,Sq,Hq,D] and k, v [B,Sk,Hkv,D] shapes disagree")


def _qkv(q, k, v):
    t = q.dtype
    return (q, None, t, "q"), (k, None, t, "k"), (v, None, t, "v")


def fa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
           causal: bool = False, softmax_scale: Optional[float] = None,
           seqused_k: Optional[torch.Tensor] = None,
           rel_bias: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None,
           window: Optional[Tuple[int, int]] = None, softcap: float = 0.0,
           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Dense forward: q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] -> (out, lse [B,Hq,Sq]).

    ``window=(left, right)`` and ``softcap`` are the fa_mods modifiers."""
    lib = load_library()
    _dtype(q)
    _dense_shapes(q, k, v)
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    R = 0 if rel_bias is None else int(rel_bias.shape[-1])
    _need_args(q, _qkv(q, k, v) + (
        (out, q.numel(), q.dtype, "out"), (lse, B * Hq * Sq, torch.float32, "lse"),
        (seqused_k, B, torch.int32, "seqused_k"),
        (rel_bias, B * Sq * Hq * R, q.dtype, "rel_bias")))
    m = _mods(window, softcap)
    _check(lib.fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq,
                         Sk, Hq, Hkv, D, _dtype(q), int(bool(causal)),
                         float(softmax_scale or 0.0), _ptr(seqused_k),
                         _ptr(rel_bias), R, ctypes.byref(m), _stream(stream)))
    return out, lse


def fa_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                  max_seqlen_q: int, max_seqlen_k: int, *,
                  seqused_k: Optional[torch.Tensor] = None,
                  causal: bool = False, softmax_scale: Optional[float] = None,
                  rel_bias: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None,
                  window: Optional[Tuple[int, int]] = None, softcap: float = 0.0,
                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Varlen forward: q [total_q,Hq,D], k/v [total_k,Hkv,D] ->
    (out [total_q,Hq,D], lse [Hq,total_q])."""
    lib = load_library()
    _dtype(q)
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or k.shape[2] != q.shape[2]:
        raise ValueError("q [total_q,Hq,D] and k, v [total_k,Hkv,D] shapes disagree")
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    B = int(cu_seqlens_q.shape[0]) - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    R = 0 if rel_bias is None else int(rel_bias.shape[-1])
    _need_args(q, _qkv(q, k, v) + (
        (out, q.numel(), q.dtype, "out"), (lse, Hq * total_q, torch.float32, "lse"),
        (cu_seqlens_q, B + 1, torch.int32, "cu_seqlens_q"),
        (cu_seqlens_k, B + 1, torch.int32, "cu_seqlens_k"),
        (seqused_k, B, torch.int32, "seqused_k"),
        (rel_bias, total_q * Hq * R, q.dtype, "rel_bias")))
    m = _mods(window, softcap)
    _check(lib.fa_fwd_varlen_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
        _ptr(cu_seqlens_k), _ptr(seqused_k), B, int(max_seqlen_q),
        int(max_seqlen_k), total_q, total_k, Hq, Hkv, D, _dtype(q),
        int(bool(causal)), float(softmax_scale or 0.0), _ptr(rel_bias), R,
        ctypes.byref(m), _stream(stream)))
    return out, lse


def splitkv_default_splits(B, Sq, Sk, Hq, Hkv, D, num_sms=0) -> int:
    return int(load_library().fa_splitkv_default_splits(B, Sq, Sk, Hq, Hkv, D, num_sms))


def splitkv_workspace_bytes(B, Sq, Hq, D, num_splits) -> int:
    return int(load_library().fa_splitkv_workspace_bytes(B, Sq, Hq, D, num_splits))


def fa_fwd_splitkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                   num_splits: int = 0, causal: bool = False,
                   softmax_scale: Optional[float] = None,
                   seqused_k: Optional[torch.Tensor] = None,
                   rel_bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None,
                   lse: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   window: Optional[Tuple[int, int]] = None, softcap: float = 0.0,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV dense forward (decode); returns (out, lse [B,Hq,Sq])."""
    lib = load_library()
    _dtype(q)
    _dense_shapes(q, k, v)
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    ns = num_splits
    if ns <= 0:
        ns = splitkv_default_splits(B, Sq, Sk, Hq, Hkv, D,
                                    torch.cuda.get_device_properties(q.device).multi_processor_count)
    need = splitkv_workspace_bytes(B, Sq, Hq, D, ns)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    R = 0 if rel_bias is None else int(rel_bias.shape[-1])
    _need_args(q, _qkv(q, k, v) + (
        (out, q.numel(), q.dtype, "out"), (lse, B * Hq * Sq, torch.float32, "lse"),
        (seqused_k, B, torch.int32, "seqused_k"),
        (rel_bias, B * Sq * Hq * R, q.dtype, "rel_bias"), (workspace, None, None, "workspace")))
    m = _mods(window, softcap)
    _check(lib.fa_fwd_splitkv_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv,
        D, _dtype(q), int(bool(causal)), float(softmax_scale or 0.0),
        _ptr(seqused_k), _ptr(rel_bias), R, int(ns), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(m),
        _stream(stream)))
    return out, lse


def fa_fwd_shard_partial(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                         k_after: Optional[torch.Tensor] = None,
                         causal: bool = False, softmax_scale: Optional[float] = None,
                         seqused_k: Optional[torch.Tensor] = None,
                         rel_bias: Optional[torch.Tensor] = None,
                         window: Optional[Tuple[int, int]] = None, softcap: float = 0.0,
                         num_splits: int = 1,
                         o_part: Optional[torch.Tensor] = None,
                         lse_part: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Normalised fp32 partial of one key shard: q [B,Sq,Hq,D] (all query
    rows), k/v [B,Sk,Hkv,D] (this shard's keys), k_after int32 [B] (keys of
    each sequence after the shard).  Returns (o_part [B*Sq*Hq, D] fp32,
    lse_part [B*Sq*Hq] fp32), packed (token, head) rows."""
    lib = load_library()
    _dtype(q)
    _dense_shapes(q, k, v)
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    rows = B * Sq * Hq
    if o_part is None:
        o_part = torch.empty((rows, D), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((rows,), dtype=torch.float32, device=q.device)
    ns = num_splits
    if ns <= 0:
        ns = splitkv_default_splits(B, Sq, max(Sk, 1), Hq, Hkv, D,
                                    torch.cuda.get_device_properties(q.device).multi_processor_count)
    if workspace is None and ns > 1:
        workspace = torch.empty(max(splitkv_workspace_bytes(B, Sq, Hq, D, ns), 16),
                                dtype=torch.uint8, device=q.device)
    R = 0 if rel_bias is None else int(rel_bias.shape[-1])
    _need_args(q, _qkv(q, k, v) + (
        (o_part, rows * D, torch.float32, "o_part"), (lse_part, rows, torch.float32, "lse_part"),
        (seqused_k, B, torch.int32, "seqused_k"), (k_after, B, torch.int32, "k_after"),
        (rel_bias, B * Sq * Hq * R, q.dtype, "rel_bias"), (workspace, None, None, "workspace")))
    m = _mods(window, softcap)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fa_fwd_shard_partial(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, Sq, Sk, Hq, Hkv, D,
        _dtype(q), int(bool(causal)), float(softmax_scale or 0.0), _ptr(seqused_k),
        _ptr(k_after), _ptr(rel_bias), R, ctypes.byref(m), int(ns), _ptr(workspace),
        ws_bytes, _stream(stream)))
    return o_part, lse_part


def fa_combine_partials(o_parts: torch.Tensor, lse_parts: torch.Tensor, B: int, Sq: int,
                        Hq: int, *, dtype: torch.dtype = torch.bfloat16,
                        out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge stacked partials o_parts [n, B*Sq*Hq, D] / lse_parts [n, B*Sq*Hq]
    into (out [B,Sq,Hq,D] of `dtype`, lse [B,Hq,Sq])."""
    lib = load_library()
    n, rows, D = o_parts.shape
    if rows != B * Sq * Hq or tuple(lse_parts.shape) != (n, rows):
        raise ValueError("o_parts must be [n, B*Sq*Hq, D] and lse_parts [n, B*Sq*Hq]")
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=o_parts.device)
    _dtype(out, "out")
    _need_args(o_parts, (
        (o_parts, None, torch.float32, "o_parts"), (lse_parts, None, torch.float32, "lse_parts"),
        (out, rows * D, out.dtype, "out"), (lse, rows, torch.float32, "lse")))
    _check(lib.fa_combine_partials(_ptr(o_parts), _ptr(lse_parts), n, B, Sq, Hq, D,
                                   _dtype(out), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def fa_fwd_splitkv_static(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                          num_splits: int = 0, causal: bool = False,
                          softmax_scale: Optional[float] = None,
                          seqused_k: Optional[torch.Tensor] = None,
                          rel_bias: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None,
                          stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV dense forward whose partials go to the library's own static
    scratch (no workspace); for callers that must not allocate device memory.
    Pass ``out`` and ``lse`` to keep this call free of allocations too."""
    lib = load_library()
    _dtype(q)
    _dense_shapes(q, k, v)
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    R = 0 if rel_bias is None else int(rel_bias.shape[-1])
    _need_args(q, _qkv(q, k, v) + (
        (out, q.numel(), q.dtype, "out"), (lse, B * Hq * Sq, torch.float32, "lse"),
        (seqused_k, B, torch.int32, "seqused_k"),
        (rel_bias, B * Sq * Hq * R, q.dtype, "rel_bias")))
    _check(lib.fa_fwd_splitkv_static(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv,
        D, _dtype(q), int(bool(causal)), float(softmax_scale or 0.0),
        _ptr(seqused_k), _ptr(rel_bias), R, int(num_splits), _stream(stream)))
    return out, lse


FA_ERR_DEVICE_TIMEOUT, FA_ERR_DEVICE_INPUT = 5, 6
DEVICE_TIMEOUT, DEVICE_INPUT = 1, 2   # bits of the device error word


def check_device_error(clear: bool = True) -> int:
    """Synchronise and return the kernels' device error word: 0 = none, bit 1
    (DEVICE_TIMEOUT) a wait gave up, bit 2 (DEVICE_INPUT) a sequence broke
    the cu_seqlens / seqused_k contract and was skipped."""
    code = ctypes.c_int(0)
    st = load_library().fa_check_device_error(ctypes.byref(code), int(clear))
    if st not in (FA_OK, FA_ERR_DEVICE_TIMEOUT, FA_ERR_DEVICE_INPUT):
        _check(st)
    return int(code.value)


def selftest_exp2_fma(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x through the softmax's FMA-pipe exponential (a device self-test of
    that routine); x is a contiguous float32 CUDA tensor."""
    lib = load_library()
    y = torch.empty_like(x)
    _need_args(x, ((x, None, torch.float32, "x"), (y, x.numel(), torch.float32, "y")))
    _check(lib.fa_selftest_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def watchdog_selftest(timeout_s: float = 0.05, stream=None) -> None:
    """Enqueue the watchdog self-test (a bounded wait that must time out)."""
    _check(load_library().fa_watchdog_selftest(int(timeout_s * 1e9), _stream(stream)))


def version() -> str:
    return load_library().fa_version().decode()


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)

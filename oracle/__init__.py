"""CPU fp64 reference for the exact attention forward (test infrastructure).

This package is the oracle the CUDA path is checked against.  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product library never does.  It shares no code with the CUDA path.

The arithmetic lives in ``fa_oracle.c`` (plain C, double precision, OpenMP over
rows); this module only marshals arrays into it.  It follows the pages:

* "mgoin/tml-fa4", argument contract: varlen layout, cu_seqlens, the distance
  d = i + (k_len_b - q_len_b) - j and the rel_bias term for 0 <= d < rel_extent,
  and the causal meaning of d (d == 0 is the query's own key).
* "flashrt/fa4-cute-runtime": (out, lse) results; ``seqused_k`` as the valid
  K/V length of a padded buffer.
* "FlashAttention-4 backend for Blackwell #1235": combining key-range splits
  through the LSE.
* "mgoin/tml-fa4" lists mask/score modifiers without defining them; the
  sliding window and soft-cap here are the plainest readings (see
  ``fa_oracle.c``).

Layouts: dense q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D], out like q, lse
[B, Hq, Sq]; varlen q [total_q, Hq, D], k/v [total_k, Hkv, D], lse
[Hq, total_q].  Inputs may be torch tensors of any float dtype or numpy
arrays; they are widened to float32 (exact for bf16/fp16 values) and every
operation is carried out in double.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_fa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile fa_oracle.c into a shared object beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O3", "-fopenmp", "-shared", "-fPIC", "-std=c11",
            "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        lib.fa_oracle_forward.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32,
                                          i32, ctypes.c_double, P, i32, i32,
                                          i32, P, P, i32, i32, i32,
                                          ctypes.c_double]
        lib.fa_oracle_forward.restype = i32
        lib.fa_oracle_rows.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32,
                                       i32, ctypes.c_double, P, i32, P, P, P,
                                       ctypes.c_long, P, P, i32, i32, i32,
                                       ctypes.c_double]
        lib.fa_oracle_rows.restype = i32
        lib.fa_oracle_lse_combine.argtypes = [P, P, i32, ctypes.c_long, i32,
                                              P, P]
        lib.fa_oracle_lse_combine.restype = None
        lib.fa_oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses by default."""
    return int(_load().fa_oracle_num_threads())


def _f32(x) -> np.ndarray:
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _i32(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a) -> Optional[int]:
    return None if a is None else a.ctypes.data


def _default_scale(D: int, softmax_scale) -> float:
    # reading of the pages: no scale given means 1/sqrt(head_dim)
    return 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)


def _as_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, rel_bias):
    """Dense [B,S,H,D] inputs become the packed form with cu = b*S."""
    dense = q.ndim == 4
    if dense:
        B, Sq, Hq, D = q.shape
        Bk, Sk, Hkv, Dk = k.shape
        if Bk != B or Dk != D or v.shape != k.shape:
            raise ValueError("dense q/k/v shapes disagree")
        cu_q = np.arange(B + 1, dtype=np.int32) * Sq
        cu_k = np.arange(B + 1, dtype=np.int32) * Sk
        q = q.reshape(B * Sq, Hq, D)
        k = k.reshape(B * Sk, Hkv, D)
        v = v.reshape(B * Sk, Hkv, D)
        if rel_bias is not None:
            rel_bias = rel_bias.reshape(B * Sq, Hq, -1)
    else:
        if cu_seqlens_q is None or cu_seqlens_k is None:
            raise ValueError("varlen inputs need cu_seqlens_q and cu_seqlens_k")
        cu_q, cu_k = _i32(cu_seqlens_q), _i32(cu_seqlens_k)
        B = cu_q.shape[0] - 1
    return dense, q, k, v, cu_q, cu_k, B, rel_bias


def attention(q, k, v, *, cu_seqlens_q=None, cu_seqlens_k=None,
              seqused_k=None, causal: bool = False, softmax_scale=None,
              rel_bias=None, kv_range=None, window=(-1, -1), softcap: float = 0.0,
              nthreads: int = 0):
    """Exact attention of every row; returns (out, lse) as float64 arrays.

    ``kv_range=(lo, hi)`` restricts every sequence to its keys [lo, hi) and
    returns that split's partial (O normalised over the range, and its LSE).
    ``window=(left, right)`` masks keys more than ``left`` before / ``right``
    after the row's diagonal (negative: no bound); ``softcap > 0`` maps each
    scaled score s to softcap * tanh(s / softcap) before the bias.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    rel_bias = _f32(rel_bias)
    dense, q, k, v, cu_q, cu_k, B, rel_bias = _as_varlen(
        q, k, v, cu_seqlens_q, cu_seqlens_k, rel_bias)
    total_q, Hq, D = q.shape
    Hkv = k.shape[1]
    R = 0 if rel_bias is None else rel_bias.shape[-1]
    su = _i32(seqused_k)
    lo, hi = (0, 2**31 - 1) if kv_range is None else kv_range
    out = np.zeros((total_q, Hq, D), dtype=np.float64)
    lse = np.zeros((Hq, total_q), dtype=np.float64)
    rc = _load().fa_oracle_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_q), _ptr(cu_k), _ptr(su), B, Hq,
        Hkv, D, int(bool(causal)), _default_scale(D, softmax_scale),
        _ptr(rel_bias), R, int(lo), int(hi), _ptr(out), _ptr(lse), nthreads,
        int(window[0]), int(window[1]), float(softcap))
    if rc:
        raise ValueError(f"oracle rejected the problem (code {rc})")
    if dense:
        Sq = total_q // max(B, 1) if B else 0
        out = out.reshape(B, Sq, Hq, D)
        lse = lse.reshape(Hq, B, Sq).transpose(1, 0, 2).copy()
    return out, lse


def attention_rows(q, k, v, rows, *, cu_seqlens_q=None, cu_seqlens_k=None,
                   seqused_k=None, causal: bool = False, softmax_scale=None,
                   rel_bias=None, window=(-1, -1), softcap: float = 0.0,
                   nthreads: int = 0):
    """Exact attention of chosen rows only.

    ``rows`` is an int array [n, 3] of (b, h, i): batch, query head and query
    position within the sequence.  Returns out [n, D] and lse [n] (float64).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    rel_bias = _f32(rel_bias)
    _, q, k, v, cu_q, cu_k, B, rel_bias = _as_varlen(
        q, k, v, cu_seqlens_q, cu_seqlens_k, rel_bias)
    _, Hq, D = q.shape
    Hkv = k.shape[1]
    R = 0 if rel_bias is None else rel_bias.shape[-1]
    su = _i32(seqused_k)
    rows = _i32(rows).reshape(-1, 3)
    rb = np.ascontiguousarray(rows[:, 0])
    rh = np.ascontiguousarray(rows[:, 1])
    ri = np.ascontiguousarray(rows[:, 2])
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().fa_oracle_rows(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_q), _ptr(cu_k), _ptr(su), B, Hq,
        Hkv, D, int(bool(causal)), _default_scale(D, softmax_scale),
        _ptr(rel_bias), R, _ptr(rb), _ptr(rh), _ptr(ri), n, _ptr(out),
        _ptr(lse), nthreads, int(window[0]), int(window[1]), float(softcap))
    if rc:
        raise ValueError(f"oracle rejected the rows (code {rc})")
    return out, lse


def lse_combine(o_parts, lse_parts):
    """Merge key-range partials: o_parts [S, n, D], lse_parts [S, n]."""
    o_parts = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    lse_parts = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    S, n, D = o_parts.shape
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    _load().fa_oracle_lse_combine(_ptr(o_parts), _ptr(lse_parts), S, n, D,
                                  _ptr(out), _ptr(lse))
    return out, lse

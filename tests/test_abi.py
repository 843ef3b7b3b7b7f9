"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every entry point that include/fa_b200.h
declares, and reject malformed arguments with a status before it touches the
device -- never by falling back to another computation.
"""
import ctypes
import os
import re

import pytest

import exact_attention_forward_flash_b200 as fa
from exact_attention_forward_flash_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_b200.h")

FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_WORKSPACE = 0, 1, 2, 3, 4

# a 16-byte aligned address that the library never dereferences in these
# tests (every call below fails validation first)
A = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10008)


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_entry_point(lib):
    names = _declared()
    assert {"fa_fwd", "fa_fwd_varlen", "fa_fwd_splitkv"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        fa.load_library(str(tmp_path / "nope.so"))


def _fwd(lib, q=A, k=A, v=A, out=A, lse=A, B=1, Sq=16, Sk=16, Hq=4, Hkv=2, D=128,
         dt=0, causal=0, scale=0.0, su=None, rb=None, R=0):
    return lib.fa_fwd(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, causal, scale,
                      su, rb, R, None)


def test_validation_statuses(lib):
    # head dims: multiples of 8 from 16 to 256
    assert _fwd(lib, D=8) == FA_ERR_UNSUPPORTED
    assert _fwd(lib, D=100) == FA_ERR_UNSUPPORTED
    assert _fwd(lib, D=264) == FA_ERR_UNSUPPORTED
    assert _fwd(lib, D=12) == FA_ERR_UNSUPPORTED
    assert _fwd(lib, Hq=6, Hkv=4) == FA_ERR_INVALID
    assert _fwd(lib, dt=7) == FA_ERR_INVALID
    assert _fwd(lib, q=None) == FA_ERR_INVALID
    assert _fwd(lib, k=None) == FA_ERR_INVALID
    assert _fwd(lib, q=MIS) == FA_ERR_INVALID
    assert _fwd(lib, out=MIS) == FA_ERR_INVALID
    assert _fwd(lib, rb=A, R=100) == FA_ERR_INVALID      # rel_extent % 128
    assert _fwd(lib, rb=A, R=0) == FA_ERR_INVALID
    assert _fwd(lib, rb=MIS, R=128) == FA_ERR_INVALID
    assert _fwd(lib, scale=float("nan")) == FA_ERR_INVALID
    import exact_attention_forward_flash_b200 as fa
    for bad in (float("nan"), -1.0, float("inf")):
        m = fa.FaMods(-1, -1, bad)
        r = lib.fa_fwd_ex(A, A, A, A, A, 1, 16, 16, 4, 2, 128, 0, 0, 0.0, None, None, 0,
                          ctypes.byref(m), None)
        assert r == FA_ERR_INVALID, bad
    assert _fwd(lib, Sq=-1) == FA_ERR_INVALID
    assert _fwd(lib, B=-1) == FA_ERR_INVALID
    msg = lib.fa_last_error_message().decode()
    assert msg, "a failed call leaves a message"


def test_empty_problems_are_no_ops(lib):
    # nothing to compute: success without touching the device
    assert _fwd(lib, B=0) == FA_OK
    assert _fwd(lib, Sq=0) == FA_OK


def test_varlen_validation(lib):
    P = None
    r = lib.fa_fwd_varlen(A, A, A, A, A, None, None, None, 2, 8, 8, 16, 16, 4, 2,
                          128, 0, 0, 0.0, None, 0, None)
    assert r == FA_ERR_INVALID  # cu_seqlens missing
    r = lib.fa_fwd_varlen(A, A, A, A, A, A, A, P, 2, 8, 8, 16, 16, 4, 2, 100, 0, 0,
                          0.0, None, 0, None)
    assert r == FA_ERR_UNSUPPORTED


def test_splitkv_host_logic(lib):
    ws = lib.fa_splitkv_workspace_bytes
    assert ws(8, 1, 32, 128, 37) >= 37 * 8 * 32 * 129 * 4
    assert ws(8, 1, 32, 128, 37) % 256 == 0
    assert ws(0, 1, 32, 128, 4) == 0
    ds = lib.fa_splitkv_default_splits
    # 8 x 8 (batch, K/V head) units of one tile each on 148 SMs: split for
    # about 16 units per SM, every split at least 8 key tiles long
    ns = ds(8, 1, 131072, 32, 8, 128, 148)
    assert 16 <= ns <= 256
    assert ds(8, 1, 2048, 32, 8, 128, 148) <= 2            # short keys
    assert ds(64, 1024, 4096, 32, 32, 128, 148) == 1        # already many units
    # a short call (8 units of 8 key tiles on 148 SMs): splits of 2 tiles
    assert ds(1, 128, 1024, 8, 1, 64, 148) == 4
    r = lib.fa_fwd_splitkv(A, A, A, A, A, 1, 1, 16, 4, 2, 128, 0, 0, 0.0, None,
                           None, 0, -1, A, 1 << 20, None)
    assert r == FA_ERR_INVALID


def test_status_strings(lib):
    for s, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID"), (2, "FA_ERR_UNSUPPORTED"),
                    (3, "FA_ERR_CUDA"), (4, "FA_ERR_WORKSPACE"), (5, "FA_ERR_DEVICE_TIMEOUT")]:
        assert lib.fa_status_string(s).decode() == name


def test_watchdog_selftest_validates_its_limit(lib):
    # out of [1 ms, 1 s]: rejected before anything is enqueued
    assert lib.fa_watchdog_selftest(10, None) == FA_ERR_INVALID
    assert lib.fa_watchdog_selftest(5_000_000_000, None) == FA_ERR_INVALID


def test_shard_partial_and_combine_validation(lib):
    # shard partial: the same argument checks as the split-KV entry point
    sp = lib.fa_fwd_shard_partial
    args = lambda D=128, lse=A, ns=1: (A, A, A, A, lse, 1, 1, 16, 4, 2, D, 0, 0, 0.0,  # noqa: E731
                                       None, None, None, 0, None, ns, None, 0, None)
    assert sp(*args(D=100)) == FA_ERR_UNSUPPORTED
    assert sp(*args(lse=None)) == FA_ERR_INVALID
    assert sp(*args(ns=-1)) == FA_ERR_INVALID
    # combine: part count, head dim, dtype and alignment are checked first
    cp = lib.fa_combine_partials
    assert cp(A, A, 0, 1, 1, 4, 128, 0, A, A, None) == FA_ERR_INVALID
    assert cp(A, A, 2, 1, 1, 4, 100, 0, A, A, None) == FA_ERR_UNSUPPORTED
    assert cp(A, A, 2, 1, 1, 4, 128, 7, A, A, None) == FA_ERR_INVALID
    assert cp(MIS, A, 2, 1, 1, 4, 128, 0, A, A, None) == FA_ERR_INVALID
    assert cp(A, A, 2, 1, 1, 4, 128, 0, None, A, None) == FA_ERR_INVALID
    assert cp(A, A, 2, 0, 1, 4, 128, 0, A, A, None) == FA_OK  # no rows: nothing to do


def test_default_splits_properties(lib):
    ds = lib.fa_splitkv_default_splits
    rng = __import__("random").Random(5)
    for _ in range(500):
        B, Sq = rng.randint(1, 64), rng.choice([1, 1, 4, 37, 128, 1024])
        Hkv = rng.choice([1, 2, 4, 8, 32])
        Hq = Hkv * rng.choice([1, 2, 4, 8])
        D = rng.choice([16, 64, 72, 128, 256])
        Sk = rng.randint(1, 300000)
        ns = ds(B, Sq, Sk, Hq, Hkv, D, 148)
        bn = 64 if D > 128 else 128
        assert 1 <= ns <= 256
        assert ns <= max(1, -(-Sk // (2 * bn)))  # every split holds at least two key tiles


# ---------------------------------------------------------------------------
# the Python binding's own checks (CPU tensors: every check below fires before
# anything reaches the library, and a well-formed call on CPU tensors is an
# error, never a CPU computation)
# ---------------------------------------------------------------------------
import torch  # noqa: E402

BF = torch.bfloat16


def _dense(B=2, Sq=5, Sk=7, Hq=4, Hkv=2, D=64, dtype=BF):
    return (torch.zeros(B, Sq, Hq, D, dtype=dtype), torch.zeros(B, Sk, Hkv, D, dtype=dtype),
            torch.zeros(B, Sk, Hkv, D, dtype=dtype))


def _raises(exc, match, fn, *a, **kw):
    with pytest.raises(exc, match=match):
        fn(*a, **kw)


@pytest.mark.parametrize("call", ["fa_fwd", "fa_fwd_splitkv", "fa_fwd_splitkv_static"])
def test_binding_rejects_buffers_of_the_wrong_extent(lib, call):
    fn = getattr(fa, call)
    kw = {"num_splits": 2} if call != "fa_fwd" else {}
    q, k, v = _dense()
    _raises(ValueError, "out holds", fn, q, k, v, out=torch.zeros(2, 5, 4, 63, dtype=BF), **kw)
    _raises(ValueError, "lse holds", fn, q, k, v, lse=torch.zeros(2, 4, 4), **kw)
    _raises(TypeError, "lse must be", fn, q, k, v, lse=torch.zeros(2, 4, 5, dtype=BF), **kw)
    _raises(ValueError, "seqused_k holds", fn, q, k, v,
            seqused_k=torch.zeros(3, dtype=torch.int32), **kw)
    _raises(TypeError, "seqused_k must be", fn, q, k, v,
            seqused_k=torch.zeros(2, dtype=torch.int64), **kw)
    # rel_bias covers every (token, head): [B*Sq, Hq, R] or [B, Sq, Hq, R]
    _raises(ValueError, "rel_bias holds", fn, q, k, v,
            rel_bias=torch.zeros(2 * 5, 3, 128, dtype=BF), **kw)
    _raises(TypeError, "rel_bias must be", fn, q, k, v,
            rel_bias=torch.zeros(2, 5, 4, 128, dtype=torch.float16), **kw)
    _raises(ValueError, "shapes disagree", fn, q, k, v[:, :6].contiguous(), **kw)
    _raises(ValueError, "shapes disagree", fn, q, k[..., :32].contiguous(),
            v[..., :32].contiguous(), **kw)
    _raises(TypeError, "k must be", fn, q, k.half(), v, **kw)
    _raises(ValueError, "contiguous", fn, q, k, v, out=torch.zeros(2, 4, 5, 64, dtype=BF)
            .transpose(1, 2), **kw)
    # everything well formed, but on the CPU: an error, not a fallback
    _raises(ValueError, "CUDA tensors", fn, q, k, v,
            rel_bias=torch.zeros(2, 5, 4, 128, dtype=BF),
            seqused_k=torch.full((2,), 7, dtype=torch.int32), **kw)


def test_binding_varlen_extents(lib):
    q = torch.zeros(9, 4, 64, dtype=BF)
    k = torch.zeros(11, 2, 64, dtype=BF)
    cu_q = torch.tensor([0, 4, 9], dtype=torch.int32)
    cu_k = torch.tensor([0, 5, 11], dtype=torch.int32)
    f = fa.fa_fwd_varlen
    _raises(ValueError, "cu_seqlens_k holds", f, q, k, k, cu_q, cu_k[:2], 5, 6)
    _raises(TypeError, "cu_seqlens_q must be", f, q, k, k, cu_q.long(), cu_k, 5, 6)
    _raises(ValueError, "lse holds", f, q, k, k, cu_q, cu_k, 5, 6, lse=torch.zeros(4, 8))
    _raises(ValueError, "rel_bias holds", f, q, k, k, cu_q, cu_k, 5, 6,
            rel_bias=torch.zeros(8, 4, 128, dtype=BF))
    _raises(ValueError, "shapes disagree", f, q, k, k[:10].contiguous(), cu_q, cu_k, 5, 6)
    _raises(ValueError, "shapes disagree", f, q.view(9, 4, 64, 1), k, k, cu_q, cu_k, 5, 6)
    _raises(ValueError, "CUDA tensors", f, q, k, k, cu_q, cu_k, 5, 6,
            rel_bias=torch.zeros(9, 4, 128, dtype=BF))


def test_binding_shard_partial_and_combine_extents(lib):
    q, k, v = _dense()
    f = fa.fa_fwd_shard_partial
    _raises(ValueError, "k_after holds", f, q, k, v, k_after=torch.zeros(1, dtype=torch.int32))
    _raises(ValueError, "o_part holds", f, q, k, v, o_part=torch.zeros(40, 63))
    _raises(TypeError, "lse_part must be", f, q, k, v, lse_part=torch.zeros(40, dtype=BF))
    _raises(ValueError, "CUDA tensors", f, q, k, v, k_after=torch.zeros(2, dtype=torch.int32))
    o_parts, l_parts = torch.zeros(3, 40, 64), torch.zeros(3, 40)
    c = fa.fa_combine_partials
    _raises(ValueError, "out holds", c, o_parts, l_parts, 2, 5, 4,
            out=torch.zeros(2, 5, 4, 32, dtype=BF))
    _raises(TypeError, "lse must be", c, o_parts, l_parts, 2, 5, 4,
            lse=torch.zeros(2, 4, 5, dtype=BF))
    _raises(TypeError, "bf16 or fp16", c, o_parts, l_parts, 2, 5, 4, dtype=torch.float32)
    _raises(ValueError, "CUDA tensors", c, o_parts, l_parts, 2, 5, 4)


def _kind_of_c(param: str) -> str:
    """Kind of one C parameter as the header spells it."""
    p = " ".join(param.split())
    if "*" in p:
        return "ptr"
    base = " ".join(w for w in p.split()[:-1] if w != "const")
    # size_t and unsigned long long are both 64-bit unsigned here (LP64),
    # and ctypes makes c_size_t and c_ulonglong one type
    return {"int": "i32", "fa_dtype": "i32", "fa_status": "i32", "float": "f32",
            "size_t": "u64", "unsigned long long": "u64", "long long": "i64"}[base]


def _kind_of_ctypes(t) -> str:
    if t in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(t, type(ctypes.POINTER(ctypes.c_int))):
        return "ptr"
    assert ctypes.sizeof(t) in (4, 8)
    return {ctypes.c_int: "i32", ctypes.c_float: "f32", ctypes.c_size_t: "u64",
            ctypes.c_ulonglong: "u64", ctypes.c_longlong: "i64"}[t]


def test_binding_signatures_match_the_header(lib):
    """Every entry point the header declares has ctypes argtypes in the
    binding with the same number of parameters of the same kinds, so that a
    change on one side cannot silently shift the arguments of the other."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    protos = {m.group(1): m.group(2) for m in
              re.finditer(r"\b(fa_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S)}
    assert len(protos) >= 16
    for name, params in protos.items():
        params = " ".join(params.split())
        want = [] if params in ("", "void") else [_kind_of_c(x) for x in params.split(",")]
        got = getattr(lib, name).argtypes
        assert got is not None, f"{name}: the binding declares no argtypes"
        assert [_kind_of_ctypes(t) for t in got] == want, name

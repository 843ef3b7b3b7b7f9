"""What the Python binding hands the library (CPU, no GPU).

A recording stand-in for the library receives every compute call, with CPU
tensors made to report device 0.  This checks that the workload shapes the
tests and the benchmark use pass the binding's own checks, that each wrapper
passes as many arguments as the entry point's ctypes signature declares, and
that sizes, the dtype code and the bias extent land in their places.
"""
import types

import pytest
import torch

import fa_inputs
import exact_attention_forward_flash_b200 as fa
from exact_attention_forward_flash_b200 import build as fa_build


@pytest.fixture()
def rec(monkeypatch):
    fa_build.build()
    real = fa.load_library()
    calls = []

    class Recorder:
        def __getattr__(self, name):
            fn = getattr(real, name)
            if name in ("fa_splitkv_default_splits", "fa_splitkv_workspace_bytes",
                        "fa_status_string", "fa_last_error_message"):
                return fn

            def record(*args):
                assert len(args) == len(fn.argtypes), (name, len(args), len(fn.argtypes))
                calls.append((name, args))
                return 0
            return record

    monkeypatch.setattr(fa, "load_library", lambda *a, **k: Recorder())
    monkeypatch.setattr(torch.Tensor, "get_device", lambda self: 0)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda d: types.SimpleNamespace(multi_processor_count=148))
    monkeypatch.setattr(fa, "_stream", lambda s: None)
    return calls


def _ptr(a):
    return a.value if a is not None else None


def test_dense_call_marshalling(rec):
    p = fa_inputs.random_dense(1, 2, 37, 90, 8, 2, 72, dtype=torch.float16, causal=True,
                               seqused=[70, 90], bias_extent=128)
    out, lse = fa.fa_fwd(p.q, p.k, p.v, causal=True, softmax_scale=0.25, seqused_k=p.seqused_k,
                         rel_bias=p.rel_bias, window=(40, 3), softcap=7.5)
    name, a = rec[-1]
    assert name == "fa_fwd_ex"
    assert [_ptr(x) for x in a[:5]] == [t.data_ptr() for t in (p.q, p.k, p.v, out, lse)]
    assert a[5:12] == (2, 37, 90, 8, 2, 72, 1)              # B Sq Sk Hq Hkv D, fp16
    assert a[12] == 1 and a[13] == 0.25                        # causal, scale
    assert _ptr(a[14]) == p.seqused_k.data_ptr() and _ptr(a[15]) == p.rel_bias.data_ptr()
    assert a[16] == 128                                        # rel_extent
    assert out.shape == p.q.shape and lse.shape == (2, 8, 37) and lse.dtype == torch.float32


def test_varlen_and_splitkv_marshalling(rec):
    v = fa_inputs.random_varlen(2, [130, 1, 77], [130, 5, 200], Hq=8, Hkv=2, D=128, causal=True,
                                bias_extent=256)
    out, lse = fa.fa_fwd_varlen(v.q, v.k, v.v, v.cu_seqlens_q, v.cu_seqlens_k, 130, 200,
                                causal=True, rel_bias=v.rel_bias)
    name, a = rec[-1]
    assert name == "fa_fwd_varlen_ex"
    assert a[8:16] == (3, 130, 200, 208, 335, 8, 2, 128)   # B maxq maxk total_q total_k Hq Hkv D
    assert a[16] == 0 and a[20] == 256                       # bf16, rel_extent
    assert lse.shape == (8, 208)
    p = fa_inputs.random_dense(3, 2, 1, 3000, 8, 2, 128)
    fa.fa_fwd_splitkv(p.q, p.k, p.v, num_splits=5)
    name, a = rec[-1]
    assert name == "fa_fwd_splitkv_ex" and a[5:11] == (2, 1, 3000, 8, 2, 128)
    assert a[17] == 5                                          # num_splits
    assert a[19] == max(fa.splitkv_workspace_bytes(2, 1, 8, 128, 5), 16)  # workspace bytes
    fa.fa_fwd_splitkv(p.q, p.k, p.v)                         # default split count
    assert rec[-1][1][17] == fa.splitkv_default_splits(2, 1, 3000, 8, 2, 128, 148)


def test_shard_partial_and_combine_marshalling(rec):
    p = fa_inputs.random_dense(4, 2, 5, 300, 4, 2, 64, causal=True, bias_extent=128)
    ka = torch.tensor([100, 0], dtype=torch.int32)
    o, l = fa.fa_fwd_shard_partial(p.q, p.k, p.v, k_after=ka, causal=True, rel_bias=p.rel_bias)
    name, a = rec[-1]
    assert name == "fa_fwd_shard_partial"
    assert a[5:12] == (2, 5, 300, 4, 2, 64, 0)
    assert o.shape == (40, 64) and l.shape == (40,)
    out, lse = fa.fa_combine_partials(torch.stack([o, o]), torch.stack([l, l]), 2, 5, 4,
                                      dtype=torch.float16)
    name, a = rec[-1]
    assert name == "fa_combine_partials" and a[2:8] == (2, 2, 5, 4, 64, 1)
    assert out.shape == (2, 5, 4, 64) and out.dtype == torch.float16 and lse.shape == (2, 4, 5)


@pytest.mark.parametrize("name", [w for w in fa_inputs.WORKLOADS if w != "video_dit_20480"])
def test_named_workloads_pass_the_checks_as_the_benchmark_calls_them(rec, name):
    p = fa_inputs.make(name, decode_sk=2048) if name == "decode_splitkv" else fa_inputs.make(name)
    out = torch.empty_like(p.q)
    lse = (torch.empty((p.B, p.Hq, p.q.shape[1])) if p.layout == "dense"
           else torch.empty((p.Hq, p.q.shape[0])))
    kw = dict(causal=p.causal, softmax_scale=p.softmax_scale, seqused_k=p.seqused_k,
              rel_bias=p.rel_bias, out=out, lse=lse, window=p.window, softcap=p.softcap)
    if p.splitkv:
        fa.fa_fwd_splitkv(p.q, p.k, p.v, num_splits=4, **kw)
    elif p.layout == "dense":
        fa.fa_fwd(p.q, p.k, p.v, **kw)
    else:
        fa.fa_fwd_varlen(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.max_seqlen_q,
                         p.max_seqlen_k, **kw)
    assert len(rec) == 1

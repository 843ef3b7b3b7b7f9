"""The allocation-free split-KV entry point (fa_fwd_splitkv_static).

Some callers cannot call cudaMalloc (their device memory belongs to a host
framework's allocator or a pool fixed at start-up, or they may not allocate
after initialisation), so they cannot hand fa_fwd_splitkv a workspace.  The
static entry point keeps its split partials in a fixed-size array inside the
library instead.  These tests call it through the C ABI and check its output
on two calls in a row against fa_fwd_splitkv's (same kernels, caller
workspace; bit for bit) and against the CPU fp64 oracle within the parity
gates the other tests use; that an empty call before a real one leaves the
real one correct (the scratch address is that of the current device); and
that an oversized problem is refused.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import fa_inputs
import oracle
import exact_attention_forward_flash_b200 as fa
from parity_util import compare

pytestmark = pytest.mark.gpu

SCRATCH = 16 * 1024 * 1024  # FA_SPLITKV_STATIC_SCRATCH_BYTES


def _static_call(lib, q, k, v, out, lse, num_splits, causal=False, seqused=None):
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.fa_fwd_splitkv_static(
        P(q), P(k), P(v), P(out), P(lse), B, Sq, Sk, Hq, Hkv, D,
        0 if q.dtype == torch.bfloat16 else 1, int(causal), 0.0, P(seqused), None, 0,
        num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("D,ns", [(128, 0), (128, 9), (256, 5), (72, 4), (40, 0)])
def test_static_matches_workspace_entry_twice(D, ns):
    lib = fa.load_library()
    probs = [fa_inputs.random_dense(500 + D + s, 4, 2, 3000, 16, 4, D, causal=True)
             for s in range(2)]
    for p in probs:  # two calls in a row, each checked against the workspace entry
        g = p.to("cuda")
        ref_o, ref_l = fa.fa_fwd_splitkv(g.q, g.k, g.v, num_splits=ns, causal=True)
        out = torch.full_like(g.q, float("nan"))
        lse = torch.full((4, 16, 2), float("nan"), device="cuda")
        st = _static_call(lib, g.q, g.k, g.v, out, lse, ns, causal=True)
        assert st == 0, lib.fa_last_error_message().decode()
        torch.cuda.synchronize()
        compare(out, lse, ref_o.float().cpu().numpy(), ref_l.cpu().numpy(),
                what=f"static D={D} ns={ns}")
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
        # and against the oracle, which shares nothing with either entry point
        ro, rl = oracle.attention(p.q, p.k, p.v, causal=True)
        compare(out, lse, ro, rl, what=f"static D={D} ns={ns} vs oracle")


def test_empty_call_before_a_real_one():
    # an empty problem (no query rows, then no keys) goes first on this
    # device; the real call after it must get this device's scratch
    lib = fa.load_library()
    p = fa_inputs.random_dense(777, 2, 3, 2000, 8, 2, 128)
    g = p.to("cuda")
    empty_q = torch.empty((0, 3, 8, 128), dtype=torch.bfloat16, device="cuda")
    assert _static_call(lib, empty_q, g.k[:0], g.v[:0], empty_q, torch.empty(0, device="cuda"),
                        0) == 0
    no_k = g.k[:, :0].contiguous()
    o0 = torch.full_like(g.q, float("nan"))
    l0 = torch.full((2, 8, 3), float("nan"), device="cuda")
    assert _static_call(lib, g.q, no_k, no_k, o0, l0, 0) == 0
    torch.cuda.synchronize()
    assert (o0 == 0).all() and torch.isneginf(l0).all()
    out = torch.full_like(g.q, float("nan"))
    lse = torch.full((2, 8, 3), float("nan"), device="cuda")
    assert _static_call(lib, g.q, g.k, g.v, out, lse, 0) == 0, lib.fa_last_error_message().decode()
    torch.cuda.synchronize()
    ro, rl = oracle.attention(p.q, p.k, p.v)
    compare(out, lse, ro, rl, what="static after empty calls")


def test_static_refuses_partials_beyond_its_scratch():
    lib = fa.load_library()
    # 64 x 64 x 32 rows x (128 + 1) fp32 x 16 splits = 33.8 MB > 16 MiB
    B, Sq, Sk, Hq, Hkv, D, ns = 64, 64, 4096, 32, 32, 128, 16
    need = fa.splitkv_workspace_bytes(B, Sq, Hq, D, ns)
    assert need > SCRATCH
    q = torch.zeros((B, Sq, Hq, D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Sk, Hkv, D), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 7.0)
    lse = torch.zeros((B, Hq, Sq), device="cuda")
    st = _static_call(lib, q, k, k, out, lse, ns)
    assert st == 4  # FA_ERR_WORKSPACE
    assert "static scratch" in lib.fa_last_error_message().decode()
    torch.cuda.synchronize()
    assert (out == 7.0).all()

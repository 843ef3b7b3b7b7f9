"""Device-side checks of the input contract ("mgoin/tml-fa4", argument contract).

cu_seqlens and seqused_k live on the device, so the host cannot check them
without a synchronisation.  The kernels check each sequence where they read
it: cu_seqlens nondecreasing within [0, total] and ending at the totals, no q
length above max_seqlen_q, seqused_k within [0, the sequence's keys].  A
sequence that breaks the contract is skipped (its rows of out and lse keep
their contents), the others are computed, and the device error word carries
code 2 until fa_check_device_error clears it.  Every case here keeps every
index the kernels use inside the buffers: the broken sequences are never read.
After each case a correct call on the same context must match the oracle.
"""
import numpy as np
import pytest
import torch

import fa_inputs
import oracle
import exact_attention_forward_flash_b200 as fa
from parity_util import compare

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


@pytest.fixture(autouse=True)
def _clean_word():
    fa.load_library()
    assert fa.check_device_error(clear=True) == 0
    yield
    assert fa.check_device_error(clear=True) == 0


def _varlen_call(g, cu_q, cu_k, max_q, causal, seqused=None):
    out = torch.full_like(g.q, SENTINEL)
    lse = torch.full((g.Hq, g.q.shape[0]), SENTINEL, dtype=torch.float32, device="cuda")
    fa.fa_fwd_varlen(g.q, g.k, g.v, cu_q, cu_k, max_q, max_q, seqused_k=seqused, causal=causal,
                     rel_bias=g.rel_bias, out=out, lse=lse)
    return out, lse


def _check_sequence(p, out, lse, b, causal):
    """Sequence b of the varlen problem p against the oracle."""
    cq, ck = p.cu_seqlens_q.tolist(), p.cu_seqlens_k.tolist()
    q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
    rb = None if p.rel_bias is None else p.rel_bias[q0:q1].unsqueeze(0)
    ro, rl = oracle.attention(p.q[q0:q1].unsqueeze(0), p.k[k0:k1].unsqueeze(0),
                              p.v[k0:k1].unsqueeze(0), causal=causal, rel_bias=rb)
    compare(out[q0:q1].unsqueeze(0), lse[:, q0:q1].unsqueeze(0), ro, rl, what=f"sequence {b}")


def _untouched(out, lse, q0, q1):
    return bool((out[q0:q1] == SENTINEL).all()) and bool((lse[:, q0:q1] == SENTINEL).all())


def _then_a_correct_call(p, causal):
    g = p.to("cuda")
    out, lse = fa.fa_fwd_varlen(g.q, g.k, g.v, g.cu_seqlens_q, g.cu_seqlens_k, p.max_seqlen_q,
                                p.max_seqlen_k, causal=causal, rel_bias=g.rel_bias)
    assert fa.check_device_error() == 0
    ro, rl = oracle.attention(p.q, p.k, p.v, cu_seqlens_q=p.cu_seqlens_q,
                              cu_seqlens_k=p.cu_seqlens_k, causal=causal, rel_bias=p.rel_bias)
    compare(out, lse, ro, rl, what="correct call after the contract error")


@pytest.mark.parametrize("causal", [False, True])
def test_sequence_longer_than_max_seqlen_q(causal):
    # lengths 100 and 300, max_seqlen_q passed as 200: the second sequence is
    # in bounds (cu_seqlens is right) but longer than the launch was sized for
    p = fa_inputs.random_varlen(3000, [100, 300], [100, 300], Hq=8, Hkv=2, D=128, causal=causal,
                                bias_extent=128)
    g = p.to("cuda")
    out, lse = _varlen_call(g, g.cu_seqlens_q, g.cu_seqlens_k, 200, causal)
    assert fa.check_device_error(clear=False) == fa.DEVICE_INPUT
    assert fa.check_device_error(clear=True) == fa.DEVICE_INPUT
    _check_sequence(p, out, lse, 0, causal)
    assert _untouched(out, lse, 100, 400)
    _then_a_correct_call(p, causal)


def test_decreasing_cu_seqlens_k_and_wrong_total():
    # cu_seqlens_k = [0, 300, 250]: sequence 1 ends before it starts, and the
    # last entry is not total_k; sequence 0 is intact
    p = fa_inputs.random_varlen(3001, [100, 300], [300, 0], Hq=4, Hkv=4, D=64, causal=False)
    g = p.to("cuda")
    bad_k = torch.tensor([0, 300, 250], dtype=torch.int32, device="cuda")
    out, lse = _varlen_call(g, g.cu_seqlens_q, bad_k, 300, False)
    assert fa.check_device_error(clear=True) == fa.DEVICE_INPUT
    _check_sequence(p, out, lse, 0, False)
    assert _untouched(out, lse, 100, 400)
    _then_a_correct_call(p, False)


def test_cu_seqlens_q_not_ending_at_total_q():
    # cu_seqlens_q = [0, 100, 390] with total_q = 400: the last sequence breaks
    # the contract (the last entry must be the total); the first is computed
    p = fa_inputs.random_varlen(3002, [100, 300], [120, 300], Hq=8, Hkv=8, D=128, causal=True)
    g = p.to("cuda")
    bad_q = torch.tensor([0, 100, 390], dtype=torch.int32, device="cuda")
    out, lse = _varlen_call(g, bad_q, g.cu_seqlens_k, 300, True)
    assert fa.check_device_error(clear=True) == fa.DEVICE_INPUT
    _check_sequence(p, out, lse, 0, True)
    assert _untouched(out, lse, 100, 400)
    _then_a_correct_call(p, True)


def test_seqused_k_beyond_the_keys_dense():
    # seqused_k = [Sk + 1, 500]: batch entry 0 is out of bounds, entry 1 fine
    p = fa_inputs.random_dense(3003, 2, 130, 600, 4, 2, 128, causal=True, seqused=[601, 500],
                               pad_value=1e4)
    g = p.to("cuda")
    out = torch.full_like(g.q, SENTINEL)
    lse = torch.full((2, 4, 130), SENTINEL, dtype=torch.float32, device="cuda")
    fa.fa_fwd(g.q, g.k, g.v, causal=True, seqused_k=g.seqused_k, out=out, lse=lse)
    assert fa.check_device_error(clear=True) == fa.DEVICE_INPUT
    assert (out[0] == SENTINEL).all() and (lse[0] == SENTINEL).all()
    ro, rl = oracle.attention(p.q[1:], p.k[1:], p.v[1:], causal=True,
                              seqused_k=np.array([500], np.int32))
    compare(out[1:], lse[1:], ro, rl, what="entry 1")
    # negative seqused_k is refused the same way
    g.seqused_k.copy_(torch.tensor([-1, 500], dtype=torch.int32))
    out.fill_(SENTINEL)
    fa.fa_fwd(g.q, g.k, g.v, causal=True, seqused_k=g.seqused_k, out=out, lse=lse)
    assert fa.check_device_error(clear=True) == fa.DEVICE_INPUT
    assert (out[0] == SENTINEL).all()
    # a correct call on the same context
    g.seqused_k.copy_(torch.tensor([600, 500], dtype=torch.int32))
    o2, l2 = fa.fa_fwd(g.q, g.k, g.v, causal=True, seqused_k=g.seqused_k)
    assert fa.check_device_error() == 0
    ro, rl = oracle.attention(p.q, p.k, p.v, causal=True, seqused_k=np.array([600, 500], np.int32))
    compare(o2, l2, ro, rl, what="correct seqused_k")


def test_status_of_the_check_call():
    # the C call returns FA_ERR_DEVICE_INPUT for code 2
    import ctypes
    p = fa_inputs.random_varlen(3004, [50], [50], Hq=4, Hkv=4, D=64)
    g = p.to("cuda")
    _varlen_call(g, g.cu_seqlens_q, g.cu_seqlens_k, 10, False)
    code = ctypes.c_int(0)
    st = fa.load_library().fa_check_device_error(ctypes.byref(code), 1)
    assert st == fa.FA_ERR_DEVICE_INPUT and code.value == fa.DEVICE_INPUT

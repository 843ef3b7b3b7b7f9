"""Host-side argument fuzzing of the dense and varlen entry points (CPU).

Random argument tuples go to the library; a model of the argument rules
stated in include/fa_b200.h predicts the status: the first rule broken decides
it (FA_ERR_INVALID for a malformed argument, FA_ERR_UNSUPPORTED for a
well-formed one the library does not serve), and a well-formed empty problem
succeeds without touching a device.  Calls the model predicts to be
well-formed and non-empty are not made: they would go on to the device.
"""
import ctypes
import math

import pytest
from hypothesis import given, settings, strategies as st

import exact_attention_forward_flash_b200 as fa
from exact_attention_forward_flash_b200 import build as fa_build

OK, INVALID, UNSUPPORTED = 0, 1, 2
A = 0x10000          # 16-byte aligned, never dereferenced
MIS = 0x10008


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def served(D):
    return D % 8 == 0 and 16 <= D <= 256


def model(dt, B, Sq, Sk, Hq, Hkv, D, scale, softcap, ptrs, rb, R):
    """Predicted status of a dense call, rules in the order the header lists
    them; None when the call is well formed and has work to do."""
    q, k, v, out = ptrs
    if dt not in (0, 1):
        return INVALID
    if B < 0 or Hq <= 0 or Hkv <= 0 or D <= 0:
        return INVALID
    if Hq % Hkv:
        return INVALID
    if not served(D):
        return UNSUPPORTED
    if Sq < 0 or Sk < 0:
        return INVALID
    if rb is not None:
        if R <= 0 or R % 128:
            return INVALID
        if rb % 16:
            return INVALID
        if B * Sq * Hq * R * 2 >= 64 << 30:
            return UNSUPPORTED
    if not math.isfinite(scale):
        return INVALID
    if not math.isfinite(softcap) or softcap < 0:
        return INVALID
    tq, tk = B * Sq, B * Sk
    if tq > 0x7fffffff or tk > 0x7fffffff or tq * Hq > 1 << 40:
        return UNSUPPORTED
    if tq > 0:
        if q is None or out is None or q % 16 or out % 16:
            return INVALID
        if tk > 0 and (k is None or v is None or k % 16 or v % 16):
            return INVALID
        return None
    return OK


ptr = st.sampled_from([A, MIS, None])
# sizes up to 2^30: B*Sq*Hq*rel_extent reaches 2^74
size = st.one_of(st.integers(-3, 40), st.sampled_from([0, 1 << 16, 1 << 20, 1 << 30]))


@settings(max_examples=600, deadline=None, derandomize=True)
@given(dt=st.sampled_from([0, 1, 2, -1]), B=size, Sq=size, Sk=size,
       Hq=st.integers(-1, 64), Hkv=st.integers(-1, 16),
       D=st.one_of(st.sampled_from([16, 64, 72, 128, 256]), st.integers(-8, 300)),
       scale=st.sampled_from([0.0, 0.125, -1.0, math.nan, math.inf]),
       softcap=st.sampled_from([0.0, 5.0, -1.0, math.nan, math.inf]),
       q=ptr, k=ptr, v=ptr, out=ptr,
       rb=st.sampled_from([None, A, MIS]), R=st.sampled_from([0, 64, 128, 256, 200, -128]))
def test_dense_status_matches_the_argument_rules(lib, dt, B, Sq, Sk, Hq, Hkv, D, scale,
                                                  softcap, q, k, v, out, rb, R):
    want = model(dt, B, Sq, Sk, Hq, Hkv, D, scale, softcap, (q, k, v, out), rb, R)
    if want is None:
        return
    m = fa.FaMods(-1, -1, softcap)
    P = lambda a: None if a is None else ctypes.c_void_p(a)
    got = lib.fa_fwd_ex(P(q), P(k), P(v), P(out), P(A), B, Sq, Sk, Hq, Hkv, D, dt, 0, scale,
                        None, P(rb), R, ctypes.byref(m), None)
    assert got == want, (got, want)
    if got != OK:
        assert lib.fa_last_error_message().decode()


@settings(max_examples=300, deadline=None, derandomize=True)
@given(B=st.integers(-2, 6), total_q=st.integers(-2, 50), total_k=st.integers(-2, 50),
       max_q=st.integers(-2, 50), D=st.sampled_from([64, 100, 128, 8]),
       cu=st.sampled_from([A, None]))
def test_varlen_status_matches_the_argument_rules(lib, B, total_q, total_k, max_q, D, cu):
    if B < 0:
        want = INVALID
    elif not served(D):
        want = UNSUPPORTED
    elif total_q < 0 or total_k < 0 or max_q < 0:
        want = INVALID
    elif B > 0 and cu is None:
        want = INVALID
    elif total_q == 0 or B == 0:
        want = OK
    else:
        return  # well formed with work: would reach the device
    P = lambda a: None if a is None else ctypes.c_void_p(a)
    got = lib.fa_fwd_varlen(P(A), P(A), P(A), P(A), P(A), P(cu), P(cu), None, B, max_q, max_q,
                            total_q, total_k, 4, 2, D, 0, 0, 0.0, None, 0, None)
    assert got == want, (got, want)


def test_rel_bias_size_rule_at_overflowing_sizes(lib):
    # B*Sq*Hq*rel_extent far beyond 2^63: the size rule must still answer
    # (the product is taken in 128 bits), before the soft-cap rule
    m = fa.FaMods(-1, -1, -1.0)   # softcap < 0: the later rule that answers instead
    P = ctypes.c_void_p
    got = lib.fa_fwd_ex(P(A), P(A), P(A), P(A), P(A), 1 << 30, 1 << 30, 0, 1, 1, 16, 0, 0, 0.0,
                        None, P(A), 128, ctypes.byref(m), None)
    assert got == UNSUPPORTED

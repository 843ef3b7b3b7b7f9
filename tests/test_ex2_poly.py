"""The softmax's FMA-pipe exponential (ex2_poly2 in csrc/sm100_ptx.cuh).

Part of the softmax's exponentials run on the FMA pipe as 2^x = 2^round(x) *
p(x - round(x)) with a degree-3 polynomial p.  Its accuracy is pinned here on
its own, not only through the end-to-end parity:

* CPU: the Remez exchange in tests/ex2_poly_fit.py reproduces the four
  coefficients written in the kernel source, and the minimax relative error
  of p on [-1/2, 1/2] is 7.48e-5;
* CPU: the kernel's steps emulated in fp32 (round-to-nearest adds, fused
  multiply-adds, the exponent-field add) stay below 8e-5 over x in [-125, 8];
* GPU: the routine itself (fa_selftest_exp2_fma) against 2^x in fp64 over a
  dense sweep of [-125, 8]: relative error below 8e-5.
"""
import os
import re

import numpy as np
import pytest

import ex2_poly_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "exact_attention_forward_flash_b200", "csrc", "sm100_ptx.cuh")
BOUND = 8e-5


def kernel_coefficients():
    """c0..c3 as written in ex2_poly2 (Horner order in the source: c3, c2, c1, c0)."""
    src = open(PTX).read()
    body = src[src.index("void ex2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = []
    for m in re.finditer(r"f2\(([0-9.e+-]+)f,\s*\1f\)", body):
        v = float(m.group(1))
        if v not in (12582912.0, -12582912.0, -1.0) and v not in lits:
            lits.append(v)
    assert len(lits) == 4, lits
    c3, c2, c1, c0 = lits
    return np.array([c0, c1, c2, c3])


def test_remez_fit_reproduces_the_kernel_coefficients():
    c, err = ex2_poly_fit.remez()
    np.testing.assert_allclose(kernel_coefficients(), c, rtol=1e-12, atol=0)
    assert 7.4e-5 < err < 7.5e-5, err


def test_minimax_error_equioscillates():
    # the optimum: the weighted error reaches +-E at 5 alternating points
    c, err = ex2_poly_fit.remez()
    xs = np.linspace(-0.5, 0.5, 200001)
    e = ex2_poly_fit._error(c, xs)
    assert abs(e[0]) == pytest.approx(err, rel=1e-6)
    assert abs(e[-1]) == pytest.approx(err, rel=1e-6)
    peaks = np.sort(np.abs(e[np.r_[0, np.nonzero(np.diff(np.sign(np.diff(e))))[0] + 1, -1]]))
    assert len(peaks) == 5 and peaks[0] > 0.999 * err


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in
    fp64, one rounding of the sum to fp32."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulate(x):
    """The kernel's steps in fp32 arithmetic."""
    c0, c1, c2, c3 = (np.float32(v) for v in kernel_coefficients())
    xc = np.maximum(x.astype(np.float32), np.float32(-126))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = _fma32(j, np.full_like(j, -1), xc)
    q = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_fp32_emulation_within_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < BOUND, rel.max()


@pytest.mark.gpu
def test_device_routine_within_bound():
    import torch
    import exact_attention_forward_flash_b200 as fa
    x = torch.linspace(-125.0, 8.0, 4_000_001, dtype=torch.float32, device="cuda")
    # odd length: the last element takes the single-element path
    y = fa.selftest_exp2_fma(x)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    ref = np.exp2(xd)
    rel = np.abs(y.double().cpu().numpy() - ref) / ref
    assert rel.max() < BOUND, (rel.max(), xd[rel.argmax()])
    # and it matches the fp32 emulation of its own steps to the last bit on a
    # sample (the emulation is the written-out algorithm)
    sub = x[::1001].cpu().numpy()
    np.testing.assert_array_equal(y[::1001].cpu().numpy(), emulate(sub))
    # below the range: tiny, finite, non-negative (about 2^-126)
    z = fa.selftest_exp2_fma(torch.tensor([-126.5, -200.0, -1e30], device="cuda"))
    torch.cuda.synchronize()
    zz = z.double().cpu().numpy()
    assert np.isfinite(zz).all() and (zz >= 0).all() and (zz <= 2.0 ** -125).all()

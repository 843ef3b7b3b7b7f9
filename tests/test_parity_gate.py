"""The parity gate itself (CPU): an exactly rounded bf16/fp16 result always
passes, and an error beyond 1e-2 plus the type's half-ulp fails."""
import numpy as np
import pytest
import torch

from parity_util import compare


def test_exact_rounding_passes_where_half_ulp_exceeds_the_bare_bound():
    ref = np.array([[4.0 + 0.0156, -5.3, 0.5, 0.01]])
    for dt in (torch.bfloat16, torch.float16):
        out = torch.tensor(ref, dtype=torch.float64).to(dt)
        compare(out, None, ref, None, mean_abs=1.0, rel_rms=1.0, what=str(dt))


def test_error_beyond_the_bound_fails():
    ref = np.array([[0.5, 0.25]])
    out = torch.tensor(ref + np.array([[0.015, 0.0]]), dtype=torch.float32)
    with pytest.raises(AssertionError):
        compare(out, None, ref, None, mean_abs=1.0, rel_rms=1.0)

"""The comparison helpers' own arithmetic, on the CPU: bfloat16 ulps and the report of
O elements above the 1e-2 tolerance."""

import warnings

import numpy as np
import pytest
import torch

from gpu_helpers import O_TOL, BeyondOTol, bf16_ulp, report_beyond_o_tol


def _next_bf16_up(a):
    """The next bfloat16 above |a| (a itself a bfloat16 value), by its bit pattern."""
    bits = torch.tensor([abs(a)], dtype=torch.bfloat16).view(torch.int16).item()
    return torch.tensor([bits + 1], dtype=torch.int16).view(torch.bfloat16).item()


@pytest.mark.parametrize("a", [1.0, 1.5, 2.0, 3.99, 4.0, 0.0078125, 100.0, -5.25, 2.0 ** -120])
def test_ulp_is_the_spacing_of_bfloat16_values(a):
    v = torch.tensor([a], dtype=torch.bfloat16).item()
    assert bf16_ulp(v) == _next_bf16_up(v) - abs(v)


def test_report_lists_elements_above_the_tolerance_in_ulps():
    ref = np.array([0.5, 4.0, -6.0, 1.0])
    gpu = ref + np.array([0.009, 0.02, -0.03125, 0.0])
    with warnings.catch_warnings(record=True) as w:
        warnings.simplefilter("always")
        rows = report_beyond_o_tol(gpu, ref, "case")
    assert [r[0] for r in rows] == [(1,), (2,)]
    # ulp at 4 is 2^-5: 0.02 is 0.64 ulp; ulp at 6 is 2^-5: 0.03125 is 1 ulp
    assert rows[0][1] == 4.0 and rows[0][3] == pytest.approx(0.64)
    assert rows[1][1] == 6.0 and rows[1][3] == pytest.approx(1.0)
    assert len(w) == 1 and issubclass(w[0].category, BeyondOTol)
    assert "2 of 4" in str(w[0].message) and str(O_TOL) in str(w[0].message)


def test_report_is_silent_within_the_tolerance():
    ref = np.linspace(-3, 3, 50)
    with warnings.catch_warnings():
        warnings.simplefilter("error")
        assert report_beyond_o_tol(ref + 0.0099, ref) == []

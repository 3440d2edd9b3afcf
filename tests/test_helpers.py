"""The comparison helpers' own arithmetic, on the CPU: bfloat16 ulps and the report of
O elements above the 1e-2 tolerance."""

import warnings

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import inputs
from gpu_helpers import O_TOL, BeyondOTol, bf16_ulp, dq_edge_bound, f64, report_beyond_o_tol


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


def test_dq_edge_bound_covers_d_from_the_rounded_output():
    # dQ_r = scale * sum_c P_rc (dP_rc - D_r) K_c: with D_r taken from bf16(O) instead of
    # O, dQ_r moves by -scale * (D'_r - D_r) * sum_c P_rc K_c (the oracle's forward with
    # values K).  The bound must cover that shift on the causal edge rows.
    x = inputs.make_inputs(1, 1, 256, 64, causal=True, seed=3)
    q, k, v, do = (f64(t[0, 0]) for t in (x.q, x.k, x.v, x.dout))
    rows = np.array([0, 1, 2, 127, 128, 255])
    dq, delta = oracle.attention_backward_dq_rows(q[rows], do[rows], rows, k, v, x.scale, True)
    o, _ = oracle.attention_forward_rows(q[rows], rows, k, v, x.scale, True)
    pk, _ = oracle.attention_forward_rows(q[rows], rows, k, k, x.scale, True)
    pk_abs, _ = oracle.attention_forward_rows(q[rows], rows, k, np.abs(k), x.scale, True)
    o_b = torch.tensor(o).to(torch.bfloat16).double().numpy()
    d_shift = np.sum(do[rows] * o_b, axis=1) - np.sum(do[rows] * o, axis=1)
    dq_moved = dq - x.scale * d_shift[:, None] * pk
    bound = dq_edge_bound(do[rows], o_b, o, pk_abs, dq, x.scale, float(np.abs(v).max()))
    assert np.all(np.abs(dq_moved - dq) <= bound)
    # and the bound is not vacuous: it is below |dQ| on most elements of the longer rows
    assert np.mean(bound[3:] < np.abs(dq[3:])) > 0.5

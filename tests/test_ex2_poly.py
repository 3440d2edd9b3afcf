"""The softmax's exponential on the FMA pipe (ex2_poly / ex2_poly2 in csrc/sm100.cuh).

Part of the kernels' exponentials 2^x skip the special-function unit: x = n + f with
n = round(x) and |f| <= 1/2, 2^f from a degree-3 polynomial, n added to the exponent
field.  The polynomial is the minimax fit of 2^f on [-1/2, 1/2] for relative error.
These tests fit that polynomial here, by the Remez exchange algorithm, and check the
coefficients written in the kernel source against the fit; then the whole function,
simulated in float32 on the CPU, and (on a GPU) the kernels' own code against 2^x.
"""

import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SM100 = os.path.join(ROOT, "exact_io_aware_63_b200", "csrc", "sm100.cuh")
REL_BOUND = 7.5e-5  # the bound the kernels' comments state


def source_coefficients():
    """(C0..C3, rounding constant) of each of ex2_poly and ex2_poly2, read from the source."""
    text = open(SM100).read()
    out = []
    for fn in ("ex2_poly", "ex2_poly2"):
        body = re.search(r"\b" + fn + r"\(float x.*?\n}\n", text, flags=re.S).group(0)
        cs = [float(re.search(r"kC%d\s*=\s*([0-9.eE+-]+)f" % i, body).group(1)) for i in range(4)]
        rnd = float(re.search(r"kRound\s*=\s*([0-9.eE+-]+)f", body).group(1))
        out.append((cs, rnd))
    return out


def remez_relative(deg, a, b, iters=40):
    """Minimax polynomial (coefficients, lowest first) of degree `deg` for 2^x on [a, b]
    in relative error, by the Remez exchange: solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on a
    reference of deg + 2 points, move the reference to the extrema of the error, repeat."""
    n = deg + 2
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        cuts = np.concatenate(([0], np.nonzero(np.diff(np.sign(err)))[0] + 1, [len(grid)]))
        ext = [s + int(np.argmax(np.abs(err[s:e]))) for s, e in zip(cuts[:-1], cuts[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, abs(E)


def ex2_poly_f32(x, cs, rnd):
    """The kernels' function in float32 arithmetic: clamp, round by adding 1.5 * 2^23,
    remainder, Horner with fused multiply-adds (an exact float64 product and one
    rounding to float32), then n added to the exponent bits."""
    f32 = np.float32
    x = np.maximum(np.asarray(x, f32), f32(-126.0))
    t = (x + f32(rnd)).astype(f32)
    f = (x - (t - f32(rnd)).astype(f32)).astype(f32)
    c0, c1, c2, c3 = (f32(c) for c in cs)
    fma = lambda a, b, c: (a.astype(np.float64) * np.float64(b) + np.float64(c)).astype(f32)
    p = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(f32)


def test_both_forms_hold_the_same_constants():
    (c_a, r_a), (c_b, r_b) = source_coefficients()
    assert c_a == c_b and r_a == r_b == 1.5 * 2 ** 23


def test_coefficients_are_the_relative_minimax_fit():
    cs, _ = source_coefficients()[0]
    fit, E = remez_relative(3, -0.5, 0.5)
    # the fit's own error is the stated bound
    assert 7.4e-5 < E <= REL_BOUND
    # each coefficient is the float32 value nearest the fit (within one float32 step)
    for got, want in zip(cs, fit):
        step = np.spacing(np.float32(want))
        assert abs(np.float32(got) - np.float32(want)) <= step, (got, want)


def test_polynomial_relative_error_on_the_reduced_range():
    cs, _ = source_coefficients()[0]
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(np.array(cs, np.float64)[::-1], f)
    assert float(np.abs(p / 2.0 ** f - 1).max()) <= REL_BOUND


def test_whole_function_in_float32_against_two_to_the_x():
    cs, rnd = source_coefficients()[0]
    x = np.concatenate([np.linspace(-125.0, 0.0, 1_000_001),
                        # around the rounding boundaries n + 1/2 and at integers
                        np.arange(-125, 1) + 0.5, np.arange(-125, 1) - 0.5,
                        np.arange(-125, 1).astype(np.float64)])
    x = x.astype(np.float32)
    y = ex2_poly_f32(x, cs, rnd).astype(np.float64)
    want = 2.0 ** x.astype(np.float64)
    rel = np.abs(y / want - 1)
    # the polynomial's bound plus a few float32 roundings
    assert float(rel.max()) <= REL_BOUND + 4e-7
    # below the clamp the result is 2^-126 times a factor in [0.7, 1.42]: zero for a
    # bfloat16 probability
    y_low = ex2_poly_f32(np.array([-200.0, -127.0, -np.inf], np.float32), cs, rnd)
    assert np.all(np.abs(y_low.astype(np.float64)) < 2.0 ** -125)


@pytest.mark.gpu
@pytest.mark.parametrize("pair", [0, 1])
def test_kernel_code_against_two_to_the_x(cuda_device, pair):
    import torch
    from exact_io_aware_63_b200 import binding
    xs = np.concatenate([np.linspace(-125.0, 0.0, 1_000_001), np.arange(-125, 1) + 0.5,
                         np.arange(-125, 1) - 0.5, [-126.0, -200.0, -np.inf]]).astype(np.float32)
    x = torch.from_numpy(xs).to(cuda_device)
    y = torch.empty_like(x)
    assert binding.fa_selftest_ex2(x, y, x.numel(), pair) == 0
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    cs, rnd = source_coefficients()[0]
    # the device code gives the float32 simulation's values (within one float32 step:
    # the simulation's fused multiply-add is emulated in float64)
    main = xs >= -125.0
    sim = ex2_poly_f32(xs[main], cs, rnd)
    assert np.all(np.abs(got[main] - sim) <= np.spacing(sim)), float(np.abs(got[main] - sim).max())
    rel = np.abs(got[main].astype(np.float64) / 2.0 ** xs[main].astype(np.float64) - 1)
    assert float(rel.max()) <= REL_BOUND + 4e-7
    assert np.all(np.abs(got[~main].astype(np.float64)) < 2.0 ** -125)

"""Host checks of the FMA-pipe exp2 the kernels use for part of their
exponentials: the constants compiled into the kernels are the ones the fit
script derives, and the kernels' steps (clamp, 1.5*2^23 rounding shifter,
reduction, degree-3 Horner, exponent add) replayed in float32 stay within the
fit's error bound of 2^x over the whole argument range the kernels produce."""
import os
import re

import numpy as np

from exact_io_aware_99_b200 import fit_exp2

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_99_b200", "csrc", "sm100.cuh")


def header_coefficients():
    text = open(HDR).read()
    vals = {}
    for name in ("kC0", "kC1", "kC2", "kC3"):
        m = re.search(name + r"\s*=\s*([-0-9.eE+]+)f", text)
        assert m, name
        vals[name] = float(np.float32(m.group(1)))
    return [vals["kC0"], vals["kC1"], vals["kC2"], vals["kC3"]]


def test_header_constants_are_the_fitted_ones():
    assert header_coefficients() == fit_exp2.coefficients_f32()


def test_fit_is_minimax_quality():
    coef, err = fit_exp2.remez_relative()
    # degree-3 relative minimax of 2^f on [-1/2, 1/2]: equioscillation error
    # about 7.5e-5 (2^-13.7); far below the 2^-9 of the bf16 rounding P gets.
    assert err < 8e-5
    xs = np.linspace(-0.5, 0.5, 10001)
    rel = np.polynomial.polynomial.polyval(xs, coef) / np.exp2(xs) - 1
    # the error alternates in sign at DEGREE + 2 points (Chebyshev alternation)
    assert np.sum(np.abs(np.diff(np.sign(rel))) > 0) >= fit_exp2.DEGREE + 1


def test_emulated_kernel_steps_accuracy():
    x = np.linspace(-125.0, 8.0, 3_000_001, dtype=np.float32)
    y = fit_exp2.emulate_f32(x, header_coefficients())
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1.2e-4


def test_emulated_special_values():
    c = header_coefficients()
    y = fit_exp2.emulate_f32(np.array([0.0, 1.0, -1.0, 8.0, 0.5, -0.5], np.float32), c)
    np.testing.assert_allclose(y, [1, 2, 0.5, 256, 2 ** 0.5, 2 ** -0.5], rtol=1e-4)
    # clamp: -inf and very negative arguments give a tiny positive value
    # (the kernels zero masked entries separately)
    z = fit_exp2.emulate_f32(np.array([-np.inf, -1000.0, -126.0], np.float32), c)
    assert np.all(z > 0) and np.all(z < 2e-38)

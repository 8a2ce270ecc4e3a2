"""The FMA-pipe exponential of the forward kernel: its constants are the Remez
fit of io_aware_exact_35_b200/exp2_poly.py and its float32 model stays within
the fitted relative-error bound over the kernel's whole input range."""
import os
import re

import numpy as np

from io_aware_exact_35_b200 import exp2_poly

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "io_aware_exact_35_b200", "csrc", "sm100.cuh")


def header_coeffs():
    text = open(HDR).read()
    return [float(re.search(rf"kEx2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)]


def test_constants_match_the_fit():
    c, err = exp2_poly.remez_exp2()
    assert err < 8e-5
    hc = header_coeffs()
    for a, b in zip(hc, c):
        assert np.float32(a) == np.float32(b)


def test_float32_model_error_bound():
    c = np.array(header_coeffs())
    x = np.linspace(-125.0, 8.0, 1_000_003).astype(np.float32)
    y = exp2_poly.ex2_poly3_f32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
    # integer arguments (n exact, f = 0): only c0's error
    xi = np.arange(-125, 9).astype(np.float32)
    yi = exp2_poly.ex2_poly3_f32(xi, c).astype(np.float64)
    assert np.allclose(yi / np.exp2(xi), c[0], rtol=1e-7)


def test_underflow_is_clamped_not_wrapped():
    c = np.array(header_coeffs())
    y = exp2_poly.ex2_poly3_f32(np.array([-np.inf, -1e30, -126.0, -125.0], np.float32), c)
    assert np.all(y > 0) and np.all(y < 2.0 ** -124)

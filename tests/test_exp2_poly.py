"""The FMA-pipe exp2 of the kernels: its cubic, checked against 2^x on the CPU.

The constants are read from the CUDA header, the evaluation mirrors the kernel's
steps in float32 (round-to-nearest split, Horner, exponent add), and the result
must stay within the fitted bound everywhere the kernels use it.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "io_aware_exact_26_b200", "csrc", "sm100.cuh")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1))) for i in range(4)]


def exp2_fma(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    r = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - r).astype(np.float32)
    q = ((c3 * f + c2) * f + c1) * f + c0
    bits = q.astype(np.float32).view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_bound_over_the_kernel_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(exp2_fma(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4


def test_integers_and_halves():
    x = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_allclose(exp2_fma(x), np.exp2(x), rtol=1e-4)
    np.testing.assert_allclose(exp2_fma(x + 0.5), np.exp2(x + 0.5), rtol=1e-4)


def test_very_negative_and_minus_infinity_are_tiny():
    x = np.array([-126.0, -300.0, -np.inf], dtype=np.float32)
    y = exp2_fma(x)
    assert np.all(y > 0) and np.all(y < 2.0 ** -125)


def test_fit_script_reproduces_the_constants():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gen", os.path.join(os.path.dirname(HDR), "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, rel = gen.fit()
    assert rel < 1e-4
    np.testing.assert_allclose(np.array(c, np.float64), np.array(coeffs(), np.float64), rtol=1e-6)

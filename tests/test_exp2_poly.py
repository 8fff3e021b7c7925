"""The FMA-pipe exp2 of the forward kernel, emulated in float32 on the CPU.

The coefficients are read from the device header; the evaluation mirrors the
device steps on each half of a packed pair (clamp at -125, rounding by adding
1.5 * 2^23, fused multiply-adds, exponent add) and is checked against float64
2^x over the range the kernel feeds it. Below -125 (masked scores are -inf)
the result is about 2^-125 rather than 0; the kernel zeroes the row sum of a
row that has no visible key.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mask_aware_block_mfa_b200", "csrc", "mfa_device.cuh")


def coefficients():
    text = open(HDR).read()
    vals = dict(re.findall(r"constexpr float kExp2(C\d) = (0x[0-9a-fA-F.p+-]+)f;", text))
    return [np.float32(float.fromhex(vals[f"C{i}"])) for i in range(4)]


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_poly(x, c):
    x = np.float32(x)
    xc = np.float32(max(x, np.float32(-125.0)))
    t = np.float32(xc + np.float32(12582912.0))
    j = np.float32(t - np.float32(12582912.0))
    f = np.float32(xc - j)
    p = fma32(fma32(fma32(c[3], f, c[2]), f, c[1]), f, c[0])
    bits = (int(p.view(np.uint32)) + (int(t.view(np.uint32)) << 23)) & 0xFFFFFFFF
    return np.uint32(bits).view(np.float32)


def test_relative_error_bound():
    c = coefficients()
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(-124.9, 8.5, 20000), np.linspace(-3, 3, 6001),
                         np.arange(-124, 9).astype(np.float64) + 0.5])
    worst = 0.0
    for x in xs.astype(np.float32):
        got = float(exp2_poly(x, c))
        ref = 2.0 ** float(x)
        worst = max(worst, abs(got - ref) / ref)
    assert worst < 1e-4, worst


def test_masked_and_integer_inputs():
    c = coefficients()
    # Clamped: -inf and anything below -125 give 2^-125 within the fit's error,
    # a positive normal float (never a NaN, a negative or a denormal).
    for x in (-np.inf, -200.0, -125.0):
        got = float(exp2_poly(x, c))
        assert abs(got / 2.0 ** -125 - 1.0) < 1e-4
    for k in range(-120, 9):
        got = float(exp2_poly(float(k), c))
        assert abs(got / 2.0 ** k - 1.0) < 1e-4


def test_fit_script_reproduces_coefficients():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit", os.path.join(os.path.dirname(HDR), "exp2_poly_fit.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    got = [np.float32(x) for x in fit.remez(3)]
    assert got == coefficients()

"""The FMA-pipe 2^x of the prefill softmax (csrc/exp2_poly.cuh), emulated
step by step in float32 on the CPU with the coefficients read from the
header: relative error within the stated bound on [-126, 127], and a finite,
non-negative, tiny result below that (the exponent field must never wrap)."""
import os
import re
import struct

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_attention_21_b200", "csrc", "exp2_poly.cuh")


def coeffs():
    text = open(HDR).read()
    c = {k: float(v) for k, v in re.findall(r"k(C[0-3]) = ([0-9.e+-]+)f", text)}
    return np.float32(c["C0"]), np.float32(c["C1"]), np.float32(c["C2"]), np.float32(c["C3"])


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def emulate(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    j = (x + shift).astype(np.float32)
    r = (j - shift).astype(np.float32)
    f = fma32(r, np.float32(-1.0), x)
    p = fma32(fma32(fma32(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (j.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 127, 2_000_003, dtype=np.float64),
                        np.arange(-125, 128, dtype=np.float64)]).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 7.6e-5, rel.max()


def test_underflow_side_never_wraps():
    x = np.concatenate([np.linspace(-1e4, -126, 100_001), [-np.inf]]).astype(np.float32)
    with np.errstate(invalid="ignore"):
        y = emulate(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y <= 2.0 ** -125)
    xs = np.linspace(-126, -125, 10001).astype(np.float32)
    assert np.abs(emulate(xs).astype(np.float64) - np.exp2(xs.astype(np.float64))).max() < 2.0 ** -137


def test_header_coefficients_match_the_fit_script_output():
    """The coefficients in the header are float32 values of a near-minimax cubic:
    p(0) is within the bound of 1 and p(1/2)/p(-1/2) within it of 2."""
    c0, c1, c2, c3 = (float(v) for v in coeffs())
    p = lambda f: ((c3 * f + c2) * f + c1) * f + c0
    assert abs(p(0.0) - 1.0) < 7.6e-5
    assert abs(p(0.5) / p(-0.5) - 2.0) < 2 * 7.6e-5 * 2

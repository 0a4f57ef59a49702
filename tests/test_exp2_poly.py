"""The polynomial exp2 the softmax kernel uses for one in four of its exponentials.

The coefficients in ptx.cuh must be the ones fit_exp2_poly.py produces, and the
kernel's fp32 operation sequence (clamp, round via 1.5*2^23, reduce, Horner in
fma, exponent-field add) must stay within the fit's relative error bound of
2^x, emulated here in numpy float32 with each fma rounded once.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "threshold_gated_block_b200", "csrc")


def _kernel_coefficients():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", text)
    return [np.float32(float(v)) for v in m.groups()]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _poly_exp2(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.5))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    r = (t - k).astype(np.float32)
    f = _fma32(r, np.float32(-1.0) * np.ones_like(r), x)
    c0, c1, c2, c3 = _kernel_coefficients()
    q = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = (t.view(np.int32).astype(np.int64) * (1 << 23) + q.view(np.int32).astype(np.int64)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_match_the_fit():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py")], capture_output=True, text=True).stdout
    fitted = [np.float32(float(v)) for v in re.findall(r"c\d = np.float32\(([0-9.e+-]+)\)", out)]
    assert fitted == _kernel_coefficients()


def test_relative_error_bound_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = _poly_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.0e-4


def test_clamped_tail_is_a_tiny_positive_normal():
    for v in (-126.0, -200.0, -np.inf):
        y = _poly_exp2(np.array([v], dtype=np.float32))[0]
        assert 0 < y < 3e-38 and np.isfinite(y)
    assert _poly_exp2(np.array([0.0], dtype=np.float32))[0] == np.float32(0.99992806)

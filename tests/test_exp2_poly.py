"""The FMA-pipe exp2 of the softmax (csrc/exp2_poly.inc, csrc/common.cuh exp2_poly):
its fp32 evaluation, replayed here step by step in numpy, stays within 1.2e-4 of
2^x over [-125, 8] (the softmax feeds it x <= 8), and the stored coefficients are the
ones gen_exp2_poly.py derives."""

import os
import re
import subprocess
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "sequence_approximate_attention_b200", "csrc")


def _coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.inc")).read()
    return [np.float32(float(v.rstrip("f"))) for v in re.findall(r"kExp2C\d = ([0-9.e+-]+f)", text)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_ref(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    r = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = _fma32(_fma32(_fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f,
               np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.float32(-0.5) + np.arange(-2000, 2000, dtype=np.float32) * np.float32(1e-6)])
    y = exp2_poly_ref(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y / exact - 1.0)
    assert rel.max() < 1.2e-4, rel.max()


def test_underflow_and_masked_inputs():
    # below -125 the result only has to be tiny and non-negative (the softmax sum
    # cannot tell it from 0); at exactly -126 the integer exponent add lands on the
    # subnormal boundary
    y = exp2_poly_ref(np.array([-np.inf, -1e30, -200.0, -126.0, -125.5], dtype=np.float32))
    assert (y >= 0).all() and (y < 3e-38).all()


def test_coefficients_reproduce():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "gen_exp2_poly.py")], capture_output=True, text=True,
                         check=True).stdout
    assert out.strip() == open(os.path.join(CSRC, "exp2_poly.inc")).read().strip()

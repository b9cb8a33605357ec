"""The FMA-pipe exp2 of the attention kernels (exp2_poly in lh_sm100.cuh):
range reduction x = n + f, f in [-1/2, 1/2], a degree-4 polynomial for 2^f
and an exponent-field add for 2^n.  Checked on the CPU, step for step in
fp32, against numpy's exp2 (the error bound), with the coefficients read
from the CUDA source, and against the fitting script that produced them."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "hierarchical_selection_attention_b200", "csrc")


def _coefficients():
    src = open(os.path.join(CSRC, "lh_sm100.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    c4, c3, c2, c1 = (float.fromhex(h) for h in hexes)
    return [1.0, c1, c2, c3, c4]


def _fma32(a, b, c):
    # a*b is exact in fp64 for fp32 inputs; one rounding of the sum to fp32
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_poly_emulated(x):
    c = [np.float32(v) for v in _coefficients()]
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = _fma32(np.full_like(f, c[4]), f, c[3])
    p = _fma32(p, f, c[2])
    p = _fma32(p, f, c[1])
    p = _fma32(p, f, c[0])
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly_error_bound():
    x = np.concatenate([np.linspace(-125.0, 2.0, 400001, dtype=np.float32),
                        -np.abs(np.random.default_rng(0).standard_normal(100000)).astype(np.float32) * 20])
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 5e-6, rel.max()
    # integers are exact up to the polynomial's value at 0
    assert abs(float(exp2_poly_emulated(np.array([0.0], np.float32))[0]) - 1.0) < 4e-6
    assert abs(float(exp2_poly_emulated(np.array([-3.0], np.float32))[0]) - 0.125) < 0.125 * 4e-6
    # far below the range: clamped to 2^-126, never a large value
    assert np.all(exp2_poly_emulated(np.array([-200.0, -1e6], np.float32)) < 1.2e-38)


def test_coefficients_match_fitting_script():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    printed = [float.fromhex(m) for m in re.findall(r"c\d = (\S+)", out)]
    assert np.allclose(printed, _coefficients(), rtol=0, atol=0)

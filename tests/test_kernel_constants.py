"""Constants the CUDA sources carry, checked against their generators (CPU only).

The gate's logsigmoid evaluates log2(1 + t), t in [0, 1], as t q(t) with a
polynomial q whose coefficients are written out in tc_kernels.cuh (kL2q).
They must be the ones csrc/log2_1p_poly.py derives (Chebyshev interpolation of
log2(1 + t)/t at 9 nodes), and the polynomial must meet its stated bound.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_vision_backbone_b200", "csrc")


def _generator():
    spec = importlib.util.spec_from_file_location("log2_1p_poly", os.path.join(CSRC, "log2_1p_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _source_coefficients():
    text = open(os.path.join(CSRC, "tc_kernels.cuh")).read()
    m = re.search(r"kL2q\[9\]\s*=\s*\{([^}]*)\}", text)
    assert m, "kL2q not found"
    return np.array([float(v.strip().rstrip("f")) for v in m.group(1).split(",")], dtype=np.float32)


def test_polynomial_coefficients_match_their_generator():
    gen = _generator()
    np.testing.assert_array_equal(_source_coefficients(), gen.coefficients())


def test_polynomial_error_bound_and_sign():
    gen = _generator()
    coef = _source_coefficients()
    assert gen.max_error(coef) < 1.6e-7
    # t q(t) is 0 at t = 0 and positive above, so logsigmoid(u) = min(u,0) - ln2 t q(t) <= 0
    t = np.linspace(0.0, 1.0, 4097).astype(np.float32)
    acc = np.float32(coef[-1]) * np.ones_like(t)
    for a in coef[-2::-1]:
        acc = (acc * t + np.float32(a)).astype(np.float32)
    assert np.all(acc > 0.0)
    assert float((acc * t)[0]) == 0.0


def test_polynomial_against_log1p_closed_form():
    # an independent check of the interpolant: ln(1 + t) = ln2 * t q(t) within 1.1e-7 nats,
    # and q(0) = 1 / ln 2 (the derivative of log2(1 + t) at 0)
    coef = _source_coefficients().astype(np.float64)
    t = np.linspace(0.0, 1.0, 10001)
    q = np.polynomial.polynomial.polyval(t, coef)
    assert np.max(np.abs(np.log(2.0) * t * q - np.log1p(t))) < 1.2e-7
    assert abs(coef[0] - 1.0 / np.log(2.0)) < 1e-6

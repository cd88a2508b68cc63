"""The soft-cap polynomial (CPU only): the coefficients compiled into the
prefill kernels are the ones the fitting script prints, and their float32
Horner evaluation stays within 3e-6 of tanh on [-1, 1], the only interval
the kernels use it on (wider scores take tanh.approx)."""

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "alternative_normalizers_b200", "csrc")


def _script():
    spec = importlib.util.spec_from_file_location("tanh_poly",
                                                  os.path.join(CSRC, "tanh_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coeffs():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("void tanh_odd_coeffs"):]
    body = body[:body.index("}")]
    return np.array([float(v) for v in re.findall(r"p\.c\[\d\] = ([-0-9.e]+)f \* out", body)],
                    dtype=np.float32)


def test_header_matches_fit():
    c = _header_coeffs()
    assert c.size == 5
    fit = _script().coefficients()
    np.testing.assert_array_equal(c, fit)


def test_error_bound_on_unit_interval():
    mod = _script()
    c = _header_coeffs()
    x = np.linspace(-1.0, 1.0, 200001).astype(np.float32)
    err = np.abs(mod.horner_f32(c, x).astype(np.float64) - np.tanh(x.astype(np.float64)))
    assert err.max() < 3e-6
    # odd: p(-x) = -p(x) exactly in float32
    np.testing.assert_array_equal(mod.horner_f32(c, -x), -mod.horner_f32(c, x))


def test_bound_fails_outside_interval():
    """The range check matters: past |x| = 1 the polynomial leaves tanh."""
    mod = _script()
    c = _header_coeffs()
    x = np.array([1.5, 2.0, 4.0], dtype=np.float32)
    err = np.abs(mod.horner_f32(c, x).astype(np.float64) - np.tanh(x.astype(np.float64)))
    assert err.min() > 1e-4

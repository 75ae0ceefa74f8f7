"""CPU pin of the constants of the FMA-pipe exp2 (exp2_poly2 in csrc/sm100.cuh):
they are the ones csrc/fit_exp2_poly.py fits, and the cubic meets the stated
relative-error bound with p(0) = 1 exactly."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_31_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    m = re.search(r"constexpr float c1 = ([0-9.eE+-]+)f, c2 = ([0-9.eE+-]+)f, c3 = ([0-9.eE+-]+)f;", text)
    assert m, "exp2_poly2 coefficients not found"
    return np.array([float(x) for x in m.groups()])


def test_coefficients_match_the_fit():
    fit = _fit_module()
    c = np.float32(fit.fit())
    assert np.allclose(_header_coefficients(), c, rtol=1e-6, atol=0)


def test_cubic_error_bound_and_exact_one():
    fit = _fit_module()
    c = _header_coefficients()
    assert fit.max_rel_err(c) < 1.1e-4
    # 2^x = 2^j * p(f): whole exponents are exact, so the largest P (x = 0) stays 1
    f = np.linspace(-0.5, 0.5, 10001)
    p = 1.0 + c[0] * f + c[1] * f ** 2 + c[2] * f ** 3
    assert p[5000] == 1.0
    assert np.all(np.abs(p / np.exp2(f) - 1) < 1.1e-4)

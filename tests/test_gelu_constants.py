"""The producer kernel's GELU (csrc/producer.cu) evaluates erf by Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.26, whose published bound is |error| <= 1.5e-7 on x >= 0.  This
CPU test reads the coefficients as they stand in the kernel source (with the factors the kernel
folds into them) and checks, in fp64, that the kernel's form max(z, 0) - |z| h with
h = erfc(|z| / sqrt 2) / 2 meets that bound against the exact GELU z Phi(z) over a dense grid, so a
mistyped coefficient fails here rather than inside the looser GPU parity tolerance."""
import math
import os
import re

import numpy as np
from scipy.special import erf

SRC = os.path.join(os.path.dirname(__file__), "..", "delta_rule_sequence_b200", "csrc", "producer.cu")


def _constant(text, name):
    m = re.search(rf"\b{name}\s*=\s*([^,;]+)[,;]", text)
    assert m, name
    expr = m.group(1).replace("f", "")
    return float(eval(expr, {"__builtins__": {}}))  # products of decimal literals only


def _kernel_constants():
    text = open(SRC, encoding="utf-8").read()
    return {n: _constant(text, n) for n in ("kGeluP", "kGeluA1", "kGeluA2", "kGeluA3", "kGeluA4",
                                             "kGeluA5", "kGeluE")}


def test_gelu_form_meets_the_published_erf_bound():
    c = _kernel_constants()
    z = np.concatenate([np.linspace(-12.0, 12.0, 400001), np.array([0.0, -0.0, 1e-30, -1e-30])])
    az = np.abs(z)
    t = 1.0 / (1.0 + c["kGeluP"] * az)
    e = np.exp2(c["kGeluE"] * z * z)
    s = t * (c["kGeluA1"] + t * (c["kGeluA2"] + t * (c["kGeluA3"] + t * (c["kGeluA4"] + t * c["kGeluA5"]))))
    gelu = np.maximum(z, 0.0) + az * (s * e)  # s e = -h
    exact = 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))
    # |GELU error| = |z| |erf error| / 2 <= |z| 0.75e-7 (plus fp64 rounding)
    assert np.all(np.abs(gelu - exact) <= np.abs(z) * 0.75e-7 + 1e-15)


def test_gelu_constants_carry_the_folded_factors():
    c = _kernel_constants()
    assert math.isclose(c["kGeluP"], 0.3275911 / math.sqrt(2.0), rel_tol=1e-7)
    assert math.isclose(c["kGeluE"], -0.5 / math.log(2.0), rel_tol=1e-7)
    for name, a in (("kGeluA1", 0.254829592), ("kGeluA2", -0.284496736), ("kGeluA3", 1.421413741),
                    ("kGeluA4", -1.453152027), ("kGeluA5", 1.061405429)):
        assert math.isclose(c[name], -0.5 * a, rel_tol=1e-7), name

"""The 2^x polynomial the prefill softmax evaluates on the FMA pipe.

The coefficients in fa_common.cuh must be the ones exp2_poly.py derives
(Cody-Waite reduction + Remez minimax fit), and a float32 model of the
kernel's evaluation must stay within the error bound stated there."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rotary_embedding_b200", "csrc")


def _poly_module():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "fa_common.cuh")).read()
    body = src[src.index("ex2_poly2"):]
    nums = [float(v) for v in re.findall(r"f2_pack\((0\.\d+)f, \1f\)", body)[:4]]
    # listed in Horner order c3, c2, c1, c0
    return nums[::-1]


def test_coefficients_match_the_derivation():
    mod = _poly_module()
    derived = [float(np.float32(c)) for c in mod.remez()]
    assert np.allclose(_kernel_coefficients(), derived, rtol=0, atol=2e-7)


def test_error_bound_over_the_softmax_range():
    mod = _poly_module()
    err = mod.max_rel_error(_kernel_coefficients())
    assert err < 1e-4, err


def test_exact_at_integers_and_reduction_consistent():
    mod = _poly_module()
    c = _kernel_coefficients()
    x = np.arange(-20, 9, dtype=np.float32)
    rel = mod.exp2_emulated(x, c) / 2.0 ** x.astype(np.float64) - 1.0
    assert np.max(np.abs(rel)) < 1e-4

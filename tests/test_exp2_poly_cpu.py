"""CPU check of the FMA-pipe 2^x that the forward kernel uses for part of its
exponentials: the four polynomial coefficients are read from the kernel header as text and
the method its comment states (round-to-nearest split x = j + f, a degree-3 polynomial for
2^f on [-0.5, 0.5], j added to the exponent) is evaluated in float32 arithmetic.  The
polynomial's relative error must stay within the stated 7.5e-5 on [-0.5, 0.5], and the whole
function within 1e-4 of 2^x on [-125, 0] (the range the kernel feeds it: scores minus the
running maximum).  The GPU test `test_fma_pipe_exp2_accuracy` checks the compiled code."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "exact_tiled_attention_33_b200", "csrc", "sm100.cuh")


def _coefficients():
    src = open(HEADER, encoding="utf-8").read()
    body = src[src.index("exp2_poly2(float a, float b)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"f2_pack\(([-0-9.eE]+)f,", body)]
    # the shift constants 12582912 (1.5 * 2^23) and -1 come first, then c3, c2, c1, c0
    coeffs = [v for v in vals if abs(v) < 2.0 and v != -1.0]
    assert len(coeffs) == 4, vals
    return [np.float32(c) for c in coeffs]  # c3, c2, c1, c0


def _poly(f, c):
    c3, c2, c1, c0 = c
    p = c3 * f + c2
    p = p * f + c1
    return p * f + c0


def test_polynomial_relative_error_on_the_reduced_range():
    c = _coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(_poly(f, [float(x) for x in c]) / np.exp2(f) - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()


def test_whole_function_in_float32():
    c = _coefficients()
    x = np.concatenate([np.linspace(-125.0, 0.0, 400001, dtype=np.float32),
                        np.float32(-np.arange(0, 126)), np.float32([-0.5, -1.5, -2.5])])
    x = np.maximum(x, np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)               # 1.5 * 2^23 + j, j = rint(x)
    j = (t - shift).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = _poly(f, c).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (j.astype(np.int64) << 23)
    y = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1e-4, (rel.max(), x[rel.argmax()])


def test_header_constants_are_the_committed_fit():
    # the four constants in the kernel header are exactly the float32 output of the
    # committed Remez fit (exp2_poly_fit.py beside the header)
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "exp2_poly_fit", os.path.join(os.path.dirname(HEADER), "exp2_poly_fit.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    assert [float(c) for c in _coefficients()] == fit.float32_coefficients()
    assert fit.max_rel_error(fit.float32_coefficients()) <= 7.5e-5


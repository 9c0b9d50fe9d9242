"""The prefill kernel's FMA-pipe exp2 (exp2_poly2 in csrc/common.cuh), checked
on the CPU: its coefficients are the ones the committed Remez fit produces,
and its float32 steps (range reduction by the 1.5 * 2^23 rounding constant,
the quadratic, the exponent added to the bit pattern) stay within the fit's
relative error of exp2 over the whole clamped input range."""
import os
import re

import numpy as np

from llama_gqa_causal_b200.csrc.fit_exp2_poly import remez_rel

COMMON = os.path.join(os.path.dirname(__file__), "..", "llama_gqa_causal_b200", "csrc", "common.cuh")


def _kernel_coefficients():
    src = open(COMMON).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = dict(re.findall(r"\b(c\d) = ([0-9.eE+-]+)f", body))
    return np.array([float(vals[f"c{i}"]) for i in range(len(vals))], dtype=np.float32)


def _fma32(a, b, c):
    # one rounding of a*b + c to float32 (the float32 product is exact in float64)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    q = _fma32(np.full_like(f, c[2]), f, np.full_like(f, c[1]))
    q = _fma32(q, f, np.full_like(f, c[0]))
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_kernel_coefficients_are_the_committed_fit():
    c = _kernel_coefficients()
    fit, err = remez_rel()
    assert len(c) == 3
    assert np.array_equal(c, fit.astype(np.float32))
    assert err < 1.8e-3


def test_exp2_poly_relative_error_over_the_input_range():
    c = _kernel_coefficients()
    # the softmax feeds exponents at most the lazy-rescale threshold (8) and
    # arbitrarily negative ones; below -126 the result leaves the normal range
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.arange(-126, 9, dtype=np.float32),           # integers
                        np.arange(-126, 8, dtype=np.float32) + 0.5])    # rounding ties
    y = _exp2_poly(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.8e-3, rel.max()
    assert np.all(y > 0)


def test_exp2_poly_clamps_very_negative_inputs_to_tiny_positive_values():
    c = _kernel_coefficients()
    x = np.array([-127.0, -128.0, -1000.0, -3.0e38], dtype=np.float32)
    y = _exp2_poly(x, c)
    assert np.all(y >= 0) and np.all(y < 2.0 ** -126)

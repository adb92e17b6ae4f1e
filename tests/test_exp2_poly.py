"""The FMA-pipe exp2 used for part of the prefill softmax (CPU checks).

The kernel's coefficients must be the ones the fit script derives, and the
whole algorithm (magic-add rounding, polynomial, exponent-field add), emulated
bit for bit in float32, must stay within 2e-4 relative error of exp2 over the
range the softmax produces.
"""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "long_context_attention_pair_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly  # noqa: E402


def kernel_coefficients():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = text[text.index("float2 exp2_fma2"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body) if float(v) < 2.0]
    # Horner order in the kernel: c3, c2, then c1, then c0.
    c3, c2, c1, c0 = vals[0], vals[1], vals[2], vals[3]
    return np.array([c0, c1, c2, c3], dtype=np.float64)


def emulate(x, c):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    c = c.astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_kernel_coefficients_are_the_fitted_ones():
    np.testing.assert_allclose(kernel_coefficients(), exp2_poly.fit(), rtol=2e-7, atol=0)


def test_emulated_kernel_exp2_relative_error():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001), np.arange(-124, 9, dtype=np.float64)])
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 2e-4, rel.max()
    # exact integers give exact powers of two
    xi = np.arange(-124, 9, dtype=np.float32)
    assert np.array_equal(emulate(xi, c), np.exp2(xi).astype(np.float32))


def test_masked_scores_vanish():
    c = kernel_coefficients()
    v = emulate(np.array([-np.inf, -1e30, -500.0], dtype=np.float32), c)
    assert np.all(v <= 2.0 ** -124) and np.all(v >= 0)

"""The attention kernel's software 2^x: its coefficients come from the committed minimax
fit, and the whole algorithm (rint range reduction, float32 Horner, exponent insertion)
stays within its error bound over the range the softmax uses."""

import os
import re

import numpy as np

from tests import exp2_poly_fit

KERNEL = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "context_attention_dit_b200",
                      "csrc", "attn_fwd_sm100.cuh")


def kernel_coefficients():
    text = open(KERNEL).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1))) for i in range(4)]


def soft_exp2_f32(x):
    """The kernel's algorithm restated in numpy float32."""
    c = kernel_coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_constants_come_from_the_fit():
    fitted = exp2_poly_fit.coefficients()
    for a, b in zip(kernel_coefficients(), fitted):
        assert abs(float(a) - b) <= 2e-7 * max(1.0, abs(b))


def test_polynomial_error_bound():
    c, t = exp2_poly_fit.fit()
    assert t < 8e-5
    assert exp2_poly_fit.float32_error([np.float32(x) for x in c]) < 8e-5


def test_soft_exp2_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), -np.arange(0, 126, 0.25), [0.0, -0.5, 0.5, 7.99]])
    got = soft_exp2_f32(x).astype(np.float64)
    ref = np.exp2(np.maximum(x, -125.0).astype(np.float32).astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert abs(soft_exp2_f32(np.array([0.0]))[0] - 1.0) < 1e-4

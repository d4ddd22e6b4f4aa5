"""The scoring kernel's exponential on the FMA pipe (host check of its
arithmetic, no GPU): the coefficients in score_kernel.cuh are the relative-
error fit that fit_exp2_poly.py produces, and the kernel's steps -- n read off
the low mantissa bits of a + 1.5*2^23, f = a - n, p(f) in float32 Horner form,
2^n added into the exponent field -- give 2^a within 3e-6 relative over the
whole range a score term can take."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sequence_sparse_attention_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402


def kernel_coefficients():
    text = open(os.path.join(CSRC, "score_kernel.cuh")).read()
    return np.float32([float(re.search(rf"kExp2C{k} = ([0-9.e+-]+)f;", text).group(1)) for k in range(5)])


def exp2_like_kernel(a):
    c = kernel_coefficients()
    a = np.maximum(np.asarray(a, dtype=np.float32), np.float32(-126.0))
    shifter = np.float32(12582912.0)
    t = (a + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (a - n).astype(np.float32)
    p = fit_exp2_poly.horner_f32(c, f)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_coefficients_are_the_fit():
    np.testing.assert_allclose(kernel_coefficients(), fit_exp2_poly.fit(), rtol=1e-6, atol=0)


def test_exp2_relative_error_over_the_score_range():
    a = np.concatenate([np.linspace(-125.9, 0.0, 400001, dtype=np.float32),
                        np.float32([-0.5, 0.5, -1e-7, 1e-7, 0.25, 3.0, 7.99])])
    got = exp2_like_kernel(a).astype(np.float64)
    want = np.exp2(a.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 3e-6, rel.max()


def test_exp2_far_below_range_is_negligible():
    got = exp2_like_kernel(np.float32([-126.0, -200.0, -np.inf]))
    assert np.all(np.abs(got) < 1.2e-38)

"""The forward's FMA-pipe exp2 (exp2_poly_f2 in csrc/fa_ptx.cuh), checked on the
CPU: its coefficients are read from the kernel source and its steps (range
reduction by the 1.5 * 2^23 shift, degree-5 polynomial in fp32 fused
multiply-adds, exponent-field add) are replayed in NumPy binary32 against
numpy.exp2 in float64."""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bf16_numerics_b200", "csrc",
                   "fa_ptx.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("uint64_t exp2_poly_f2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.eE+-]+)f, \1f\)", body)]
    # order in the source: magic, c5, c4, c3, c2, c1, c0
    magic, coeffs = vals[0], vals[1:]
    return np.float32(magic), [np.float32(c) for c in coeffs]


def _fma32(a, b, c):
    # a*b + c with one rounding (float64 holds the exact product of two binary32)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(y):
    magic, (c5, c4, c3, c2, c1, c0) = _coefficients()
    y = np.maximum(np.asarray(y, np.float32), np.float32(-126.0))
    t = (y + magic).astype(np.float32)
    r = (y - (t - magic).astype(np.float32)).astype(np.float32)
    q = _fma32(np.full_like(r, c5), r, np.full_like(r, c4))
    for c in (c3, c2, c1, c0):
        q = _fma32(q, r, np.full_like(r, c))
    bits = q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << np.uint64(23)) &
                                                   np.uint64(0xFFFFFFFF))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_source_has_the_expected_form():
    magic, coeffs = _coefficients()
    assert magic == np.float32(1.5 * 2 ** 23)
    assert len(coeffs) == 6 and coeffs[-1] == np.float32(1.0)


def test_relative_error_over_the_softmax_range():
    # the softmax's arguments (S - m) * log2(e) are <= 0: m is at least the running row max
    y = np.concatenate([np.linspace(-126.0, 0.0, 400001), -np.logspace(-8, 0, 2000), [0.0, -0.5, -1.0]])
    y = y.astype(np.float32)
    got = exp2_poly(y).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= 5e-7, rel.max()


def test_exact_values():
    assert exp2_poly(np.float32(0.0)) == np.float32(1.0)        # the tied maximum of the standard shift
    for k in (-1, -7, -20, -100):
        assert exp2_poly(np.float32(k)) == np.float32(2.0 ** k)  # integer arguments: r = 0, q = 1


def test_masked_scores_are_negligible():
    v = exp2_poly(np.float32(-np.inf))
    assert 0.0 < v <= np.float32(2.0 ** -126)

"""The forward's FMA-pipe exp2 (exp2_poly_f2 in csrc/fa_ptx.cuh), checked on the
CPU: its coefficients are read from the kernel source and its steps (range
reduction by the 1.5 * 2^23 shift, degree-5 polynomial in fp32 fused
multiply-adds, exponent-field add, exact 0 below -126) are replayed in NumPy
binary32 against numpy.exp2 in float64.  The coefficients themselves are
re-derived here by the method the kernel names (relative least squares with
Lawson reweighting on [-1/2, 1/2], constant term fixed at 1)."""

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
    y_in = np.asarray(y, np.float32)
    y = np.maximum(y_in, np.float32(-126.0))
    t = (y + magic).astype(np.float32)
    r = (y - (t - magic).astype(np.float32)).astype(np.float32)
    q = _fma32(np.full_like(r, c5), r, np.full_like(r, c4))
    for c in (c3, c2, c1, c0):
        q = _fma32(q, r, np.full_like(r, c))
    bits = q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << np.uint64(23)) &
                                                   np.uint64(0xFFFFFFFF))
    e = (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    return np.where(y_in < np.float32(-126.0), np.float32(0.0), e).astype(np.float32)


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


def test_masked_scores_give_exact_zero():
    """A masked score (-inf) must not enter the row sum or P_bar V: on rows
    whose shift m is 0 with a negative row maximum, l can be tiny, and a
    leftover 2^-126 would not be negligible there."""
    assert exp2_poly(np.float32(-np.inf)) == np.float32(0.0)
    assert np.all(exp2_poly(np.array([-126.5, -200.0, -1e30], np.float32)) == 0.0)
    assert exp2_poly(np.float32(-126.0)) == np.float32(2.0 ** -126)


def _lawson_fit(n_points=20001, iterations=300, degree=5):
    """Minimax relative approximation of 2^r on [-1/2, 1/2] by
    p(r) = 1 + c1 r + ... + c5 r^5, via Lawson's algorithm: weighted least
    squares on the relative error (p(r) - 2^r) / 2^r, the weights multiplied
    by the absolute error after every solve (C. L. Lawson, 1961)."""
    r = np.linspace(-0.5, 0.5, n_points)
    f = np.exp2(r)
    a = np.stack([r ** k for k in range(1, degree + 1)], axis=1) / f[:, None]
    b = 1.0 - 1.0 / f
    w = np.full(n_points, 1.0 / n_points)
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)
        err = np.abs(a @ c - b)
        w = w * err
        w /= w.sum()
    return c, err.max()


def test_coefficients_are_the_lawson_minimax_fit():
    """The kernel's five non-constant coefficients are the refit rounded to
    binary32 (within one binary32 ulp each, so that another LAPACK build
    landing next to a rounding boundary still passes), and in exact
    arithmetic they stay within the refit's minimax relative error plus what
    rounding the coefficients to binary32 costs (c1's half-ulp times 1/2
    alone is 1.5e-8)."""
    c_fit, e_fit = _lawson_fit()
    _, coeffs = _coefficients()
    c_src = [coeffs[4 - k] for k in range(5)]  # c1..c5 (source order: c5..c1, then c0)
    assert coeffs[-1] == np.float32(1.0)
    for k in range(5):
        fit32 = np.float32(c_fit[k])
        assert abs(c_src[k] - fit32) <= np.spacing(fit32), (k + 1, c_src[k], fit32)
    r = np.linspace(-0.5, 0.5, 200001)
    p = 1.0 + sum(float(c_src[k - 1]) * r ** k for k in range(1, 6))
    e_src = np.abs(p / np.exp2(r) - 1.0).max()
    assert e_fit < 1e-7
    assert e_src <= e_fit + 2.5e-8, (e_src, e_fit)

"""Bit-accurate BF16 emulation (NumPy only).  TEST INFRASTRUCTURE ONLY.

BF16 is 1 sign bit, 8 exponent bits and 7 stored fraction bits (8 significant
bits): the top half of an IEEE binary32.  The pages (page 1, "mechanism two";
page 2, sections 1 and 4) describe BF16 storage and the rounding that happens
when two BF16 numbers are added; page 3 misstates the fraction width, and the
standard format is used here.

Conversions go through binary32 first, as hardware converts fp32 accumulators
to bf16: ``round_bf16(x)`` = RNE(fp32(x)).  The rounding itself is done on the
uint32 bit pattern: add 0x7FFF plus the lowest kept bit, then drop the low 16
bits (round to nearest, ties to even).  NaN stays a quiet NaN; +-Inf and
overflow to Inf follow from the same integer arithmetic.

``add_trace`` restates page 2, section 4 ("the physical mechanism behind the
mathematical magic"): two negative BF16 numbers are added, the significand
overflows, the sum is shifted right by one place and the bit shifted out
decides the rounding.  It returns every quantity of that description so that
a test can pin each one.
"""

from __future__ import annotations

import math

import numpy as np

BF16_SIG_BITS = 8  # 1 implicit + 7 stored fraction bits


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round binary32 values to BF16 (RNE) and return the 16-bit patterns."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    is_nan = np.isnan(x)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    quiet_nan = (u >> np.uint64(16)) | np.uint64(0x0040)
    out = np.where(is_nan, quiet_nan, rounded) & np.uint64(0xFFFF)
    return out.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Expand 16-bit BF16 patterns to the binary32 values they denote (exact)."""
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def round_bf16(x) -> np.ndarray:
    """Value of x after conversion to binary32 and then to BF16 (RNE)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32)))


def round_significand(x: float, sig_bits: int = BF16_SIG_BITS, mode: str = "rne") -> float:
    """Round a real (given exactly as a float64) to ``sig_bits`` significant bits.

    Normal range only (no subnormals, no overflow), which is all the worked
    example needs.  ``mode`` is "rne" (nearest, ties to even), "away"
    (nearest, ties away from zero) or "rz" (toward zero).
    """
    if x == 0.0 or not math.isfinite(x):
        return x
    mant, exp = math.frexp(abs(x))  # abs(x) = mant * 2**exp, 0.5 <= mant < 1
    scaled = mant * (1 << sig_bits)  # exact: a power-of-two scaling
    kept = math.floor(scaled)
    frac = scaled - kept  # exact
    if mode == "rz":
        q = kept
    elif mode == "away":
        q = kept + (1 if frac >= 0.5 else 0)
    elif mode == "rne":
        if frac > 0.5 or (frac == 0.5 and (kept & 1)):
            q = kept + 1
        else:
            q = kept
    else:
        raise ValueError(f"unknown rounding mode {mode!r}")
    return math.copysign(math.ldexp(q, exp - sig_bits), x)


def _exponent(x: float) -> int:
    """e such that 2**e <= |x| < 2**(e+1)."""
    return math.frexp(abs(x))[1] - 1


def add_trace(a: float, b: float, sig_bits: int = BF16_SIG_BITS) -> dict:
    """Exact account of adding two BF16 numbers and rounding the sum to BF16.

    a and b must be BF16 values (8 significant bits).  Their exact sum is a
    float64 (8-bit significands with exponents this close add exactly).
    Returns the exact sum, whether the significand overflowed (exponent of the
    sum above both inputs' exponents, i.e. a right shift by one place), the
    guard bit (first bit below the kept ``sig_bits``), the sticky bit (OR of
    all lower bits) and the sum rounded under RNE, ties-away and toward zero.
    """
    for v in (a, b):
        if round_significand(v, sig_bits, "rz") != v:
            raise ValueError(f"{v!r} is not representable with {sig_bits} significant bits")
    exact = a + b
    e_sum = _exponent(exact)
    e_in = max(_exponent(a), _exponent(b))
    ulp_exp = e_sum - (sig_bits - 1)  # weight of the last kept bit
    half_ulps = abs(exact) / math.ldexp(1.0, ulp_exp - 1)  # exact (power-of-two scaling)
    guard = int(math.floor(half_ulps)) & 1
    sticky = int(half_ulps != math.floor(half_ulps))
    return {
        "exact": exact,
        "exponent_in": e_in,
        "exponent_sum": e_sum,
        "shifted_right": e_sum > e_in,
        "guard": guard,
        "sticky": sticky,
        "rne": round_significand(exact, sig_bits, "rne"),
        "away": round_significand(exact, sig_bits, "away"),
        "rz": round_significand(exact, sig_bits, "rz"),
    }

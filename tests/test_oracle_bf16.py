"""Pins for the BF16 emulator of the oracle (CPU only).

The emulator is checked against things it does not compute itself: every
BF16 bit pattern (round trip), torch's own float32->bfloat16 cast (an
independent library), closed-form ties, IEEE special values, and the worked
BF16 addition of page 2, section 4 of the pages (golden file, expected values
worked by hand in binary).
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split()
            out[key] = float(val)
    return out


def _torch_bits(x32):
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_roundtrip_every_bf16_pattern():
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bf16.bf16_bits_to_f32(pats)
    back = bf16.f32_to_bf16_bits(vals)
    finite_or_inf = ~np.isnan(vals)
    assert np.array_equal(back[finite_or_inf], pats[finite_or_inf])
    # NaNs stay NaN and come back quiet
    nan_back = back[~finite_or_inf]
    assert np.all(np.isnan(bf16.bf16_bits_to_f32(nan_back)))
    assert np.all(nan_back & 0x0040)


def test_matches_torch_cast_random_and_ties():
    rng = np.random.default_rng(123)
    x = rng.standard_normal(200_000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200_000).astype(np.float32)
    # exact halfway cases: a bf16 value plus half of its last place, both parities
    base = bf16.round_bf16(rng.standard_normal(50_000).astype(np.float32))
    u = base.view(np.uint32) | np.uint32(0x8000)
    ties = u.view(np.float32)
    allx = np.concatenate([x, ties, -ties]).astype(np.float32)
    allx = allx[np.isfinite(allx)]
    assert np.array_equal(bf16.f32_to_bf16_bits(allx), _torch_bits(allx))


def test_ties_go_to_even_closed_form():
    # 1 + 2^-8 lies halfway between 1 (even) and 1 + 2^-7 (odd): goes to 1
    assert bf16.round_bf16(np.float32(1.0 + 2.0 ** -8)) == np.float32(1.0)
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): goes up
    assert bf16.round_bf16(np.float32(1.0 + 3 * 2.0 ** -8)) == np.float32(1.0 + 2.0 ** -6)
    # just above halfway rounds up, just below rounds down
    assert bf16.round_bf16(np.float32(1.0 + 2.0 ** -8 + 2.0 ** -20)) == np.float32(1.0 + 2.0 ** -7)
    assert bf16.round_bf16(np.float32(1.0 + 2.0 ** -8 - 2.0 ** -20)) == np.float32(1.0)


def test_special_values():
    f = np.float32
    assert bf16.round_bf16(f(np.inf)) == np.inf
    assert bf16.round_bf16(f(-np.inf)) == -np.inf
    assert np.isnan(bf16.round_bf16(f(np.nan)))
    assert bf16.round_bf16(np.finfo(np.float32).max) == np.inf  # overflows under RNE
    # largest finite bf16 is 0x7F7F = (2 - 2^-7) * 2^127
    assert bf16.bf16_bits_to_f32(np.uint16(0x7F7F)) == f((2 - 2.0 ** -7) * 2.0 ** 127)
    assert bf16.round_bf16(f(0.0)) == 0.0
    assert math.copysign(1.0, float(bf16.round_bf16(f(-0.0)))) == -1.0


def test_float64_goes_through_float32_first():
    # double rounding: 1 + 2^-8 + 2^-30 rounds to 1 + 2^-8 in fp32 (a tie for
    # bf16), which then goes to even (1.0), while direct rounding would go up.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert np.float32(x) == np.float32(1.0 + 2.0 ** -8)
    assert bf16.round_bf16(x) == np.float32(1.0)
    assert bf16.round_significand(x, 8, "rne") == 1.0 + 2.0 ** -7


def test_worked_bf16_sum_page2():
    g = _read_kv("worked_bf16_sum.txt")
    t = bf16.add_trace(g["a"], g["b"])
    assert t["exact"] == g["exact"]
    assert t["exponent_in"] == g["exponent_in"]
    assert t["exponent_sum"] == g["exponent_sum"]
    assert t["shifted_right"] is True
    assert t["guard"] == g["guard"]
    assert t["sticky"] == g["sticky"]
    assert t["rne"] == g["rne"]
    assert t["away"] == g["away"]
    assert t["rz"] == g["rz"]
    # a nonzero sticky below the guard bit tips RNE to the more negative value
    assert bf16.round_significand(t["exact"] - 2.0 ** -20, 8, "rne") == g["rne_with_sticky"]
    # hardware-like path: fp32 sum (exact here) then RNE to bf16, and torch's bf16 add
    s32 = np.float32(g["a"]) + np.float32(g["b"])
    assert float(s32) == g["exact"]
    assert float(bf16.round_bf16(s32)) == g["rne"]
    ta = torch.tensor(g["a"], dtype=torch.bfloat16)
    tb = torch.tensor(g["b"], dtype=torch.bfloat16)
    assert float(ta + tb) == g["rne"]


def test_add_trace_rejects_non_bf16():
    with pytest.raises(ValueError):
        bf16.add_trace(1.0 + 2.0 ** -9, 1.0)


def test_add_trace_no_overflow_case():
    # 1.5 + 0.25 = 1.75: no significand overflow, exact, no rounding
    t = bf16.add_trace(1.5, 0.25)
    assert t["shifted_right"] is False and t["guard"] == 0 and t["sticky"] == 0
    assert t["rne"] == 1.75

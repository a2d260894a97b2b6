"""The two-pass forward variant, examined on the CPU (a reading, not a kernel).

The one-pass tiled forward finds a row's tie only when the tile holding the
second copy of the maximum arrives.  Until then the stabilised rule leaves
m = rm, so the first copy enters the P_bar V product as an exact bf16 1.0;
when the tie appears, m moves to beta * rm and the O accumulator is rescaled
by exp(m_old - m_new).  A two-pass forward would find (rm, rs, m) first, so no
operand ever holds that transient 1.0.

Both schedules are emulated here in binary32 with P_bar rounded to bf16 before
the product and the product accumulated in binary32, as the tensor cores do
with a TMEM accumulator.  On such hardware the transient 1.0 does no harm: the
one-pass result carries the exact 1.0 scaled in binary32, the two-pass result
the bf16 rounding of exp(rm - m), and both stay within bf16 rounding of the
float64 oracle.  This is why the two-pass variant is not built.
"""

import numpy as np

import workloads
from oracle import attention as A
from oracle import bf16

TILE = 128


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _exp32(x):
    return _f32(np.exp(np.asarray(x, dtype=np.float64)))


def _emulate(q, k, v, beta, two_pass):
    """One head, non-causal: O in binary32 from tiles of 128 keys."""
    N, d = q.shape
    scale = A.scale_f32(d)
    s = _f32(_f32(q.astype(np.float64) @ k.astype(np.float64).T) * scale)
    if two_pass:
        rm_f, rs_f, m_f = A.row_stats(s, A.STABILIZED, beta)
    o = np.zeros((N, v.shape[1]), np.float32)
    l = np.zeros(N, np.float32)
    rm = np.full(N, -np.inf, np.float32)
    rs = np.zeros(N, np.int32)
    m = np.full(N, -np.inf, np.float32)
    ones = np.zeros(N, np.int64)  # exact bf16 ones that entered P_bar V, per row
    for j0 in range(0, N, TILE):
        st = s[:, j0:j0 + TILE]
        if two_pass:
            m_new = m_f
        else:
            t_max = st.max(axis=1)
            t_cnt = (st == t_max[:, None]).sum(axis=1)
            rise = t_max > rm
            same = t_max == rm
            rs = np.where(rise, t_cnt, np.where(same, rs + t_cnt, rs)).astype(np.int32)
            rm = np.where(rise, t_max, rm).astype(np.float32)
            m_new = A.select_shift(rm, rs, beta, A.STABILIZED)
        alpha = np.where(np.isneginf(m), np.float32(0), _exp32(m.astype(np.float64) - m_new.astype(np.float64)))
        o = _f32(o * alpha[:, None])
        l = _f32(l * alpha)
        pbar = _exp32(st.astype(np.float64) - m_new.astype(np.float64)[:, None])
        l = _f32(l + pbar.sum(axis=1, dtype=np.float32))
        p16 = bf16.round_bf16(pbar)
        ones += (p16 == 1.0).sum(axis=1)
        o = _f32(o + _f32(p16.astype(np.float64) @ v[j0:j0 + TILE].astype(np.float64)))
        m = _f32(m_new)
    return _f32(o / l[:, None]), ones


def _late_tie_head(seed=5):
    """N = 256 (two key tiles), d = 64, dyadic Q and K so S is exact.  Rows
    0-63 see their maximum once in tile 0 and a second copy in tile 1; V has
    negative-mean columns, as in the pages' bias mechanism."""
    rng = np.random.default_rng(seed)
    N, d = 256, 64
    q = _f32(rng.integers(-2, 3, (N, d)) / 8.0)
    k = _f32(rng.integers(-2, 3, (N, d)) / 8.0)
    v = workloads.to_bf16_values(rng.standard_normal((N, d)).astype(np.float32))
    v[:, :16] -= np.float32(1.0)
    for i in range(64):
        k[3 + i] = q[i] * np.float32(2.0)      # a large score in tile 0 ...
        k[128 + 3 + i] = k[3 + i]              # ... and its copy in tile 1
    return q, k, workloads.to_bf16_values(v)


def test_one_pass_holds_transient_ones_two_pass_none():
    q, k, v = _late_tie_head()
    f = A.attention_fwd(q[None, None], k[None, None], v[None, None], False, A.STABILIZED, return_pbar=True)
    late = np.arange(64)
    assert np.all(f["rs"][0, 0, late] >= 2)  # the planted rows do tie
    _, ones_1 = _emulate(q, k, v, 2.0, two_pass=False)
    _, ones_2 = _emulate(q, k, v, 2.0, two_pass=True)
    # exact ones of the final P_bar after bf16 rounding: one per untied row,
    # and on tied rows only where exp(rm - m) is within 2^-9 of 1 (reading 3)
    final_ones = (bf16.round_bf16(_f32(f["pbar"][0, 0])) == 1.0).sum(axis=1)
    assert np.array_equal(ones_2, final_ones)  # two-pass: nothing transient
    transient = ones_1[late] - final_ones[late]
    assert np.all(transient >= 1)  # one-pass: the first copy of each late tie entered as 1.0


def test_both_schedules_within_bf16_rounding_of_the_oracle():
    q, k, v = _late_tie_head()
    ref = A.attention_fwd(q[None, None], k[None, None], v[None, None], False, A.STABILIZED)["o"][0, 0]
    o1, _ = _emulate(q, k, v, 2.0, two_pass=False)
    o2, _ = _emulate(q, k, v, 2.0, two_pass=True)
    late = slice(0, 64)
    scale = np.abs(ref[late]).max()
    e1 = np.abs(o1[late] - ref[late]).max() / scale
    e2 = np.abs(o2[late] - ref[late]).max() / scale
    assert e1 < 2.0 ** -8 and e2 < 2.0 ** -8
    # the schedules differ only by where the rounding falls; neither is biased
    # on the negative-mean columns
    d1 = (o1[late, :16] - ref[late, :16]).mean()
    d2 = (o2[late, :16] - ref[late, :16]).mean()
    assert abs(d1) < 2.0 ** -9 * scale and abs(d2) < 2.0 ** -9 * scale

"""Pins for the float64 attention oracle (CPU only).

Each check compares the oracle with something it does not compute itself:
the pages' shift rule worked by hand (golden table), brute-force softmax with
pure-Python loops, torch's scaled_dot_product_attention in float64 with
autograd (an independent library), central finite differences, exact
identities (delta = rowsum(P o dP), shift invariance), and closed-form special
cases.  Planted-mistake tests at the end show that a plausible slip in the
oracle (a dropped scale, a swapped branch, a transposed operand, a dropped
delta) makes one of these pins fail.
"""

import math
import os

import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from oracle import bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _shift_table():
    rows = []
    with open(os.path.join(GOLDEN, "shift_rule.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            mode, rm, rs, beta, m = line.split()
            rows.append((int(mode), float(rm), int(rs), float(beta), float(m)))
    return rows


def _rand_bf16(rng, shape, std=1.0):
    return workloads.to_bf16_values(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


# ---------------------------------------------------------------- shift rule

def check_shift_rule(fn):
    for mode, rm, rs, beta, m in _shift_table():
        got = fn(np.array([rm], np.float32), np.array([rs]), beta, mode)[0]
        assert got == np.float32(m), (mode, rm, rs, beta, m, got)


def test_shift_rule_golden_table():
    check_shift_rule(A.select_shift)


# --------------------------------------------------------- brute force (N<=8)

def _brute_fwd(q, k, v, causal):
    """Unshifted softmax with pure-Python loops: exp(S)/sum(exp(S))."""
    N, d = q.shape
    sc = 1.0 / math.sqrt(d)
    o = np.zeros((N, v.shape[1]))
    lse = np.zeros(N)
    for i in range(N):
        js = range(i + 1) if causal else range(N)
        s = {j: sum(float(q[i, c]) * float(k[j, c]) for c in range(d)) * sc for j in js}
        z = sum(math.exp(s[j]) for j in js)
        lse[i] = math.log(z)
        for c in range(v.shape[1]):
            o[i, c] = sum(math.exp(s[j]) / z * float(v[j, c]) for j in js)
    return o, lse


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("mode", [0, 1])
def test_forward_brute_force(causal, mode):
    rng = np.random.default_rng(7)
    for N, d in [(1, 4), (5, 4), (8, 16)]:
        q, k, v = (_rand_bf16(rng, (1, 1, N, d)) for _ in range(3))
        # add a tie: key 0 duplicated, query aimed at it
        if N > 2:
            k[0, 0, 2] = k[0, 0, 0]
            q[0, 0, N - 1] = k[0, 0, 0]
        out = A.attention_fwd(q, k, v, causal, mode, 2.0)
        o_ref, lse_ref = _brute_fwd(q[0, 0], k[0, 0], v[0, 0], causal)
        np.testing.assert_allclose(out["o"][0, 0], o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out["lse"][0, 0], lse_ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------ independent library (torch)

def _torch_ref(q, k, v, do, causal):
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("mode", [0, 1])
def test_against_torch_sdpa_float64(causal, mode):
    rng = np.random.default_rng(11)
    B, H, N, d = 2, 2, 64, 64
    q, k, v, do = (_rand_bf16(rng, (B, H, N, d)) for _ in range(4))
    k[:, :, 40] = k[:, :, 0]
    q[:, :, 50:60] = k[:, :, :1] * np.float32(0.5)
    fwd = A.attention_fwd(q, k, v, causal, mode, 2.0)
    bwd = A.attention_bwd(q, k, v, do, causal, mode, 2.0, fwd=fwd)
    o, dq, dk, dv = _torch_ref(q, k, v, do, causal)
    for got, ref in ((fwd["o"], o), (bwd["dq"], dq), (bwd["dk"], dk), (bwd["dv"], dv)):
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("d", [64, 128])
def test_against_torch_sdpa_head_dims(d):
    rng = np.random.default_rng(5)
    q, k, v, do = (_rand_bf16(rng, (1, 2, 32, d)) for _ in range(4))
    fwd = A.attention_fwd(q, k, v, True, 1, 2.0)
    bwd = A.attention_bwd(q, k, v, do, True, 1, 2.0, fwd=fwd)
    o, dq, dk, dv = _torch_ref(q, k, v, do, True)
    np.testing.assert_allclose(fwd["o"], o, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(bwd["dq"], dq, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(bwd["dk"], dk, rtol=1e-9, atol=1e-11)


# ------------------------------------------------------- finite differences

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("mode", [0, 1])
def test_gradients_finite_differences(causal, mode):
    rng = np.random.default_rng(3)
    N, d = 6, 4
    q, k, v, do = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
    k[0, 0, 3] = k[0, 0, 1]  # a tie for the rows that aim at key 1
    q[0, 0, 4] = k[0, 0, 1]
    bwd = A.attention_bwd(q, k, v, do, causal, mode, 2.0)
    h = 1e-6

    def loss(q_, k_, v_):
        return float((A.attention_fwd(q_, k_, v_, causal, mode, 2.0)["o"] * do).sum())

    for name, x, g in (("q", q, bwd["dq"]), ("k", k, bwd["dk"]), ("v", v, bwd["dv"])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        rel = np.linalg.norm(fd - g) / max(np.linalg.norm(g), 1e-30)
        assert rel <= 1e-6, (name, rel)


# -------------------------------------------------------- exact identities

def test_delta_identity():
    rng = np.random.default_rng(9)
    q, k, v, do = (_rand_bf16(rng, (1, 2, 48, 16)) for _ in range(4))
    fwd = A.attention_fwd(q, k, v, True, 1, 2.0)
    bwd = A.attention_bwd(q, k, v, do, True, 1, 2.0, fwd=fwd)
    for h in range(2):
        s = q[0, h].astype(np.float64) @ k[0, h].astype(np.float64).T / 4.0
        s = np.where(np.tril(np.ones((48, 48), bool)), s, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        dp = do[0, h].astype(np.float64) @ v[0, h].astype(np.float64).T
        np.testing.assert_allclose(bwd["delta"][0, h], (p * dp).sum(1), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny", "tiestress"])
def test_mode_invariance(name):
    w = workloads.make(name) if name == "tiny" else workloads.make(name).heads([(0, 0)])
    if name == "tiestress":
        w = workloads.Workload(w.name, 1, 1, 512, w.d, w.causal, w.seed, w.q[:, :, :512].copy(),
                               w.k[:, :, :512].copy(), w.v[:, :, :512].copy(), w.do[:, :, :512].copy(),
                               w.forced_tie_rows[:, :, :512])
    f0 = A.attention_fwd(w.q, w.k, w.v, w.causal, 0)
    f1 = A.attention_fwd(w.q, w.k, w.v, w.causal, 1)
    b0 = A.attention_bwd(w.q, w.k, w.v, w.do, w.causal, 0, fwd=f0)
    b1 = A.attention_bwd(w.q, w.k, w.v, w.do, w.causal, 1, fwd=f1)
    assert (f1["m"] != f0["m"]).any()  # the rule actually moved some shifts
    for x0, x1 in ((f0["o"], f1["o"]), (f0["lse"], f1["lse"]), (b0["dq"], b1["dq"]),
                   (b0["dk"], b1["dk"]), (b0["dv"], b1["dv"])):
        assert np.linalg.norm(x1 - x0) <= 1e-12 * np.linalg.norm(x0)


@pytest.mark.parametrize("mode", [0, 1])
def test_repeated_sequence_invariance(mode):
    """Q, K, V, dO repeated r times along the sequence (non-causal): every
    softmax weight is divided by r and each key's r copies share the mass, so
    O, dQ, dK, dV are those of one copy, lse grows by ln r, rm is unchanged
    and rs is multiplied by r (every row becomes tied)."""
    n, r = 48, 4
    rng = np.random.default_rng(17)
    q, k, v, do = (_rand_bf16(rng, (1, 2, n, 16)) for _ in range(4))
    rep = lambda x: np.tile(x, (1, 1, r, 1))
    f = A.attention_fwd(q, k, v, False, mode, 2.0)
    b = A.attention_bwd(q, k, v, do, False, mode, 2.0, fwd=f)
    fr = A.attention_fwd(rep(q), rep(k), rep(v), False, mode, 2.0)
    br = A.attention_bwd(rep(q), rep(k), rep(v), rep(do), False, mode, 2.0, fwd=fr)
    for c in range(r):
        rows = slice(c * n, (c + 1) * n)
        for x, xr in ((f["o"], fr["o"]), (b["dq"], br["dq"]), (b["dk"], br["dk"]), (b["dv"], br["dv"])):
            np.testing.assert_allclose(xr[:, :, rows], x, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(fr["lse"][:, :, rows], f["lse"] + math.log(r), rtol=0, atol=1e-12)
        assert np.array_equal(fr["rm"][:, :, rows], f["rm"])
        assert np.array_equal(fr["rs"][:, :, rows], r * f["rs"])
        assert np.array_equal(fr["m"][:, :, rows], A.select_shift(f["rm"], r * f["rs"], 2.0, mode))


# ------------------------------------------- the trigger and the fix (pages)

def test_trigger_exact_ones_standard_mode():
    """Page 1, "trigger condition": tied maxima give several exact ones."""
    w = workloads.make("tiny")
    f = A.attention_fwd(w.q, w.k, w.v, True, 0, return_pbar=True)
    tied = f["rs"] > 1
    assert tied.sum() > 10
    for b, h, i in zip(*np.nonzero(tied)):
        row = f["pbar"][b, h, i]
        assert (row == 1.0).sum() == f["rs"][b, h, i]
    # every row of the standard shift has P_bar == 1 at each maximum
    assert np.all(f["pbar"].max(axis=-1) == 1.0)


def test_fix_keeps_pbar_below_one_on_tied_rows():
    """Page 1, "minimal fix": with the moved shift, max(P_bar) < 1 on tied rows;
    untied rows keep m = rm and exactly one entry equal to 1."""
    w = workloads.make("tiny")
    f = A.attention_fwd(w.q, w.k, w.v, True, 1, return_pbar=True)
    tied = f["rs"] > 1
    rowmax = f["pbar"].max(axis=-1)
    assert np.all(rowmax[tied] < 1.0)
    assert np.all(f["pbar_max"][tied] < 1.0)
    assert np.all(f["pbar_max"][~tied] == 1.0)
    ones = (f["pbar"] == 1.0).sum(axis=-1)
    assert np.all(ones[~tied] == 1) and np.all(ones[tied] == 0)
    assert tied.any()


def test_tiestress_forced_rows_have_the_target_class():
    w = workloads.make("tiestress", B=1, H=2, N=1024)
    f = A.attention_fwd(w.q, w.k, w.v, False, 1)
    cls = w.notes["tie_class"]
    forced = cls >= 0
    assert np.all(f["rs"][forced] == 2)
    assert np.all(f["rm"][cls == 0] > 0)
    assert np.all(f["rm"][cls == 1] < 0)
    assert np.all(f["rm"][cls == 2] == 0)
    assert np.all(f["m"][cls == 2] == 1.0)
    assert np.all(f["m"][cls == 1] == 0.0)
    np.testing.assert_array_equal(f["m"][cls == 0], 2.0 * f["rm"][cls == 0])
    frac = forced.mean()
    assert 0.22 <= frac <= 0.28
    # the fix holds on every tied row, whatever the sign class
    tied = f["rs"] > 1
    assert np.all(f["pbar_max"][tied] < 1.0)


def test_g2s_sink_rows_are_tied():
    w = workloads.make("g2s", B=1, H=2)
    f = A.attention_fwd(w.q, w.k, w.v, True, 1)
    assert np.all(f["rs"][w.forced_tie_rows] >= 2)
    assert np.all(f["rm"][w.forced_tie_rows] > 0)
    assert abs(w.forced_tie_rows.mean() - 0.10) < 0.01


# ------------------------------------------------------------ special cases

def test_causal_first_row_and_zero_query():
    rng = np.random.default_rng(1)
    N, d = 16, 8
    q, k, v, do = (_rand_bf16(rng, (1, 1, N, d)) for _ in range(4))
    q[0, 0, 9] = 0.0  # a zero query: all visible scores are 0, a tie at rm == 0
    f = A.attention_fwd(q, k, v, True, 1)
    b = A.attention_bwd(q, k, v, do, True, 1, fwd=f)
    assert np.array_equal(f["o"][0, 0, 0], v[0, 0, 0].astype(np.float64))  # row 0 sees only key 0
    assert np.all(b["dq"][0, 0, 0] == 0.0)
    np.testing.assert_allclose(f["o"][0, 0, 9], v[0, 0, :10].astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)
    assert f["rm"][0, 0, 9] == 0.0 and f["rs"][0, 0, 9] == 10
    assert f["m"][0, 0, 9] == 1.0  # beta - 1 with beta = 2
    np.testing.assert_allclose(f["pbar_max"][0, 0, 9], math.exp(-1.0), rtol=1e-15)


def test_o_for_delta_changes_only_delta_path():
    rng = np.random.default_rng(2)
    q, k, v, do = (_rand_bf16(rng, (1, 1, 32, 16)) for _ in range(4))
    f = A.attention_fwd(q, k, v, True, 1)
    b_ref = A.attention_bwd(q, k, v, do, True, 1, fwd=f)
    b_same = A.attention_bwd(q, k, v, do, True, 1, fwd=f, o_for_delta=f["o"])
    for key in ("dq", "dk", "dv", "delta"):
        assert np.array_equal(b_ref[key], b_same[key])
    o_bf = workloads.to_bf16_values(f["o"].astype(np.float32))
    b_bf = A.attention_bwd(q, k, v, do, True, 1, fwd=f, o_for_delta=o_bf)
    assert np.array_equal(b_bf["dv"], b_ref["dv"])
    assert not np.array_equal(b_bf["delta"], b_ref["delta"])


# ------------------------------------------------ margin variant (mode 2)

def _small_tie_rows():
    """One head of d = 64 on the 1/8 grid in which every row has a tied
    maximum rm = 2^-9: q = +-e_i / 8; keys 0, 1 are (1/8) on dims 0-3 and the
    other keys -(1/8) there, so even rows tie on keys 0, 1 and odd rows on the
    other fourteen (S = +-2^-9)."""
    N, d = 16, 64
    q = np.zeros((1, 1, N, d), np.float32)
    k = np.zeros((1, 1, N, d), np.float32)
    v = workloads.to_bf16_values(np.random.default_rng(3).standard_normal((1, 1, N, d)).astype(np.float32))
    for i in range(N):
        q[0, 0, i, i % 4] = 0.125 if i % 2 == 0 else -0.125
    for j in (0, 1):
        k[0, 0, j, :4] = 0.125                    # tie pair for every query
    k[0, 0, 2:, :4] = -0.125
    return q, k, v


def test_margin_keeps_bf16_pbar_below_one():
    """Reading of the pages' goal max(P_bar) < 1 for the bf16 operand: with
    |rm| = 2^-9 the fp32 rule leaves exp(rm - m) within 2^-9 of 1, which
    rounds to 1.0 in bf16; the margin mode moves m by 2^-8 and the bf16 value
    stays below 1.  (Closed form: bf16(exp(-2^-8)) = 1 - 2^-8.)"""
    q, k, v = _small_tie_rows()
    f1 = A.attention_fwd(q, k, v, False, 1)
    f2 = A.attention_fwd(q, k, v, False, 2)
    tied = f1["rs"] > 1
    assert tied.all() and np.all(f1["rm"] == np.float32(2.0 ** -9))
    bf1 = bf16.round_bf16(f1["pbar_max"].astype(np.float32))
    bf2 = bf16.round_bf16(f2["pbar_max"].astype(np.float32))
    assert np.all(f1["pbar_max"][tied] < 1.0)          # the fp32 rule holds ...
    assert np.all(bf1[tied] == 1.0)                    # ... but its bf16 value is 1
    assert np.all(bf2[tied] < 1.0)
    assert np.all(bf2[tied] <= np.float32(1.0 - 2.0 ** -8))
    assert np.all(f2["m"][~tied] == f2["rm"][~tied])
    # the margin is a shift: O and lse are unchanged (softmax shift invariance)
    np.testing.assert_allclose(f2["o"], f1["o"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(f2["lse"], f1["lse"], rtol=1e-12)


def test_margin_sweep_over_tied_maxima():
    """Every tied row, whatever rm, ends with bf16(exp(rm - m)) < 1 in mode 2."""
    rng = np.random.default_rng(5)
    rm = np.concatenate([rng.uniform(-1e-2, 1e-2, 20000), rng.uniform(-50, 50, 20000),
                         np.array([0.0, 2.0 ** -9, -(2.0 ** -9), 2.0 ** -8, -(2.0 ** -8)])]).astype(np.float32)
    rs = np.full(rm.shape, 2)
    for beta in (1.001, 1.5, 2.0, 4.0):
        m = A.select_shift(rm, rs, beta, 2)
        assert np.all((m - rm).astype(np.float32) >= np.float32(2.0 ** -8) * np.float32(0.999))
        pmax = np.exp(rm.astype(np.float64) - m.astype(np.float64)).astype(np.float32)
        ok = np.isfinite(pmax) & (pmax > 0)
        assert np.all(bf16.round_bf16(pmax[ok]) < 1.0)


# ------------------------------------------------------- planted mistakes
# Each test plants one plausible slip in the oracle (on the CPU) and checks
# that a pin above would catch it.

def test_planted_mistake_dropped_scale_is_caught(monkeypatch):
    monkeypatch.setattr(A, "scale_f64", lambda d: 1.0)
    rng = np.random.default_rng(7)
    q, k, v = (_rand_bf16(rng, (1, 1, 8, 16)) for _ in range(3))
    out = A.attention_fwd(q, k, v, True, 1)
    o_ref, _ = _brute_fwd(q[0, 0], k[0, 0], v[0, 0], True)
    assert not np.allclose(out["o"][0, 0], o_ref, rtol=1e-6)


def test_planted_mistake_swapped_branch_is_caught(monkeypatch):
    orig = A.select_shift

    def swapped(rm, rs, beta, mode=1):
        m = orig(rm, rs, beta, mode)
        rm = np.asarray(rm, np.float32)
        tied = np.asarray(rs) > 1
        return np.where(tied & (rm < 0), np.float32(beta) * rm, m).astype(np.float32)

    with pytest.raises(AssertionError):
        check_shift_rule(swapped)


def _oracle_bwd_with(monkeypatch, old: str, new: str):
    """Replace one expression in the source of oracle.attention.attention_bwd
    and install the result in the oracle module (undone by monkeypatch)."""
    import inspect
    import textwrap

    src = textwrap.dedent(inspect.getsource(A.attention_bwd))
    assert src.count(old) == 1, old
    ns = dict(vars(A))
    exec(compile(src.replace(old, new), A.__file__, "exec"), ns)
    monkeypatch.setattr(A, "attention_bwd", ns["attention_bwd"])


def test_planted_mistake_transposed_dk_is_caught(monkeypatch):
    """The slip planted in the oracle itself: dK = dS Q instead of dS^T Q (a
    transposed operand; square shapes keep it well-formed).  The torch SDPA
    pin rejects it."""
    _oracle_bwd_with(monkeypatch, "ds.T @ q[b, h]", "ds @ q[b, h]")
    with pytest.raises(AssertionError):
        test_against_torch_sdpa_float64(True, 1)
    with pytest.raises(AssertionError):
        test_gradients_finite_differences(False, 1)


def test_planted_mistake_dq_without_scale_is_caught(monkeypatch):
    """The slip planted in the oracle itself: dQ without the softmax scale."""
    _oracle_bwd_with(monkeypatch, "ds @ k[b, h].astype(np.float64) * sc", "ds @ k[b, h].astype(np.float64)")
    with pytest.raises(AssertionError):
        test_against_torch_sdpa_head_dims(64)


def test_planted_mistake_dropped_delta_is_caught():
    rng = np.random.default_rng(4)
    N, d = 6, 4
    q, k, v, do = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
    f = A.attention_fwd(q, k, v, True, 1)
    b_wrong = A.attention_bwd(q, k, v, do, True, 1, fwd=f, o_for_delta=np.zeros_like(f["o"]))
    h = 1e-6
    x = q.copy()
    x[0, 0, 3, 1] += h
    lp = float((A.attention_fwd(x, k, v, True, 1)["o"] * do).sum())
    x[0, 0, 3, 1] -= 2 * h
    lm = float((A.attention_fwd(x, k, v, True, 1)["o"] * do).sum())
    fd = (lp - lm) / (2 * h)
    assert abs(b_wrong["dq"][0, 0, 3, 1] - fd) > 1e-4


def test_planted_mistake_flipped_causal_mask_is_caught(monkeypatch):
    """Keys after the query visible instead of keys before it: the brute-force
    softmax (key j <= query i) disagrees."""
    monkeypatch.setattr(A, "_mask", lambda n, causal: np.triu(np.ones((n, n), bool)) if causal
                        else np.ones((n, n), bool))
    rng = np.random.default_rng(21)
    q, k, v = (_rand_bf16(rng, (1, 1, 8, 16)) for _ in range(3))
    out = A.attention_fwd(q, k, v, True, 1)
    o_ref, _ = _brute_fwd(q[0, 0], k[0, 0], v[0, 0], True)
    assert not np.allclose(out["o"][0, 0], o_ref, rtol=1e-6)


def test_planted_mistake_tie_count_of_one_is_caught(monkeypatch):
    """A tie count that never exceeds 1 (the equality test dropped) leaves the
    shift on the row maximum: the exact ones the fix must remove come back on
    the tied rows of the tiny workload."""
    real = A.row_stats

    def no_ties(s32, mode, beta):
        rm, rs, _ = real(s32, mode, beta)
        rs = np.minimum(rs, 1).astype(np.int32)
        return rm, rs, A.select_shift(rm, rs, beta, mode)

    w = workloads.make("tiny")
    tied = A.attention_fwd(w.q, w.k, w.v, True, 1)["rs"] > 1
    monkeypatch.setattr(A, "row_stats", no_ties)
    f = A.attention_fwd(w.q, w.k, w.v, True, 1, return_pbar=True)
    assert tied.any()
    assert np.all(f["pbar"].max(axis=-1)[tied] == 1.0)  # the fix's pin (max P_bar < 1) fails



# ------------------------------------- BF16 dS operand (rounding point of dQ, dK)

def _brute_bwd_bf16_ds(q, k, v, do, causal):
    """dQ, dK with dS rounded to BF16 before the two products, written with
    pure-Python loops; the rounding is torch's float32 -> bfloat16 cast (an
    implementation independent of oracle.bf16)."""
    N, d = q.shape
    sc = 1.0 / math.sqrt(d)
    vis = [[(j <= i) if causal else True for j in range(N)] for i in range(N)]
    s = [[sum(float(q[i, c]) * float(k[j, c]) for c in range(d)) * sc for j in range(N)] for i in range(N)]
    p = [[0.0] * N for _ in range(N)]
    for i in range(N):
        z = sum(math.exp(s[i][j]) for j in range(N) if vis[i][j])
        for j in range(N):
            p[i][j] = math.exp(s[i][j]) / z if vis[i][j] else 0.0
    o = [[sum(p[i][j] * float(v[j, c]) for j in range(N)) for c in range(d)] for i in range(N)]
    dlt = [sum(float(do[i, c]) * o[i][c] for c in range(d)) for i in range(N)]
    ds = [[p[i][j] * (sum(float(do[i, c]) * float(v[j, c]) for c in range(d)) - dlt[i]) for j in range(N)]
          for i in range(N)]
    dsb = torch.tensor(ds, dtype=torch.float64).to(torch.float32).to(torch.bfloat16).to(torch.float64).tolist()
    dq = [[sum(dsb[i][j] * float(k[j, c]) for j in range(N)) * sc for c in range(d)] for i in range(N)]
    dk = [[sum(dsb[i][j] * float(q[i, c]) for i in range(N)) * sc for c in range(d)] for j in range(N)]
    return np.array(dq), np.array(dk), np.array(ds)


@pytest.mark.parametrize("causal", [True, False])
def test_bf16_ds_operand_brute_force(causal):
    rng = np.random.default_rng(17)
    N, d = 7, 8
    q, k, v, do = (_rand_bf16(rng, (1, 1, N, d)) for _ in range(4))
    k[0, 0, 4] = k[0, 0, 1]
    q[0, 0, 5] = k[0, 0, 1]
    f = A.attention_fwd(q, k, v, causal, 1)
    b = A.attention_bwd(q, k, v, do, causal, 1, fwd=f, ds_bf16=True)
    dq, dk, ds = _brute_bwd_bf16_ds(q[0, 0], k[0, 0], v[0, 0], do[0, 0], causal)
    np.testing.assert_allclose(b["dq"][0, 0], dq, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b["dk"][0, 0], dk, rtol=1e-12, atol=1e-13)
    # dV and delta do not go through the rounded operand
    b0 = A.attention_bwd(q, k, v, do, causal, 1, fwd=f)
    assert np.array_equal(b["dv"], b0["dv"]) and np.array_equal(b["delta"], b0["delta"])
    # the rounding moved dQ, and by no more than its a-priori bound
    # |bf16(x) - x| <= 2^-8 |x|, summed over the product: 2^-8 * scale * |dS| |K|
    bound = 2.0 ** -8 / math.sqrt(d) * (np.abs(ds) @ np.abs(k[0, 0].astype(np.float64)))
    diff = np.abs(b["dq"][0, 0] - b0["dq"][0, 0])
    assert diff.max() > 0 and np.all(diff <= bound * (1 + 1e-9) + 1e-300)


def test_bf16_ds_floor_exceeds_the_float_bar_on_two_hot_rows():
    """Why the reading is needed: where a row's softmax mass sits on two
    bitwise-equal keys, dQ of that row is the small difference of two large,
    nearly opposite dS terms times the same key, and the BF16 rounding of dS
    alone moves it by more than 1e-2 of max|dQ| -- an exact product of
    BF16-rounded dS cannot meet the float bar on such inputs, whatever the
    kernel."""
    # two existence cases (seed, N, query = s * key 0); over 36 such draws
    # (three seeds, N in {64, 128, 200, 384}, s in {0.5, 0.75, 1}) the floor
    # ranged from 0.17 % to 1.9 % of max|dQ|
    errs = []
    for seed, N, s in ((2, 200, 0.75), (31, 384, 1.0)):
        rng = np.random.default_rng(seed)
        q, k, v, do = (_rand_bf16(rng, (1, 1, N, 128)) for _ in range(4))
        k[0, 0, N // 2] = k[0, 0, 0]
        q[0, 0, N - 8:] = k[0, 0, 0] * np.float32(s)
        f = A.attention_fwd(q, k, v, False, 1)
        exact = A.attention_bwd(q, k, v, do, False, 1, fwd=f)
        rounded = A.attention_bwd(q, k, v, do, False, 1, fwd=f, ds_bf16=True)
        errs.append(np.abs(rounded["dq"] - exact["dq"]).max() / np.abs(exact["dq"]).max())
    assert min(errs) > 1e-2, errs

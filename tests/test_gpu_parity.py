"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases are compared on every output element; the full-size workloads run
in the launch configuration the benchmark uses and are compared on sampled
(batch, head) pairs that the oracle computes exactly (heads are independent).
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import bf16
from tests import parity as P

pytestmark = pytest.mark.gpu


def _small(name, B, H, N, seed=None):
    return workloads.make(name, B=B, H=H, N=N, seed=seed)


def _check_fix_invariants(gpu, mode):
    tied = gpu["rs"] > 1
    if mode in (1, 2):
        assert np.all(gpu["pbar_max"][tied] < 1.0)
        assert np.all(gpu["pbar_max"][~tied] == 1.0)
    else:
        assert np.all(gpu["pbar_max"] == 1.0)
    if mode == 2:  # the margin keeps the bf16 operand below 1 as well
        assert np.all(bf16.round_bf16(gpu["pbar_max"][tied].astype(np.float32)) < 1.0)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tiny_exact_stats(cuda_device, mode):
    w = workloads.make("tiny")
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=True)
    _check_fix_invariants(gpu, mode)
    assert (ref["rs"] > 1).any()


def _d128_case(N, causal, tie_scale):
    rng = np.random.default_rng(N)
    shape = (1, 2, N, 128)
    mk = lambda: workloads.to_bf16_values(rng.standard_normal(shape).astype(np.float32))
    w = workloads.Workload("d128", 1, 2, N, 128, causal, 0, mk(), mk(), mk(), mk(), np.zeros((1, 2, N), bool))
    w.k[:, :, N // 2] = w.k[:, :, 0]
    w.q[:, :, N - 10:] = np.float32(tie_scale) * w.k[:, :, :1]
    w.forced_tie_rows[:, :, N - 10:] = True
    return w


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [384, 200])
def test_small_grid(cuda_device, mode, causal, d, N):
    """Several tiles plus a ragged tail (N = 200), both masks, both head dims,
    with the workloads' forced ties (query = 0.5 * key 0, key 0 duplicated).

    At d = 128 and these lengths the two tied keys carry most of the softmax
    mass of their rows, so dQ and dK of those rows are cancellations of
    BF16-rounded dS terms: they are held to the bar against the oracle with
    the BF16 dS operand modelled (the float64 error is printed beside it)."""
    if d == 64:
        w = workloads.make("g2s", B=1, H=2, N=N, seed=100 + N + d)
    else:
        w = _d128_case(N, causal, 0.5)
    w.causal = causal
    gpu = P.run_gpu(w, mode)
    ds_keys = ("dq", "dk") if d == 128 else ()
    ref = P.oracle(w, mode, o_gpu=gpu["o"], ds_bf16=bool(ds_keys))
    errs = P.compare(gpu, ref, exact_stats=False, bf16_ds_keys=ds_keys)
    print(f"N={N} d={d} causal={causal} mode={mode}:", {k: tuple(round(x, 5) for x in v) for k, v in errs.items()})
    _check_fix_invariants(gpu, mode)
    assert np.all(gpu["rs"][w.forced_tie_rows] >= 2)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [384, 200])
def test_two_hot_ties_against_the_bf16_ds_reference(cuda_device, causal, N):
    """Rows whose softmax mass sits mostly on two bitwise-equal keys (d = 128,
    query = 0.5 * key 0).  There dQ is the difference of two large, nearly
    opposite terms (dS[t,0] + dS[t,j*]) K[0]; rounding dS to BF16 -- the
    operand precision of the dQ product -- moves it by up to about 2 % of
    max|dQ| (tests/test_oracle_attention.py: the floor exceeds 1e-2 on such
    rows).  dQ and dK meet the 1e-2 bar against the oracle with that
    operand modelled; O and dV against the float64 oracle."""
    w = _d128_case(N, causal, 0.5)
    mode = 1
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"], ds_bf16=True)
    errs = P.compare(gpu, ref, exact_stats=False, bf16_ds_keys=("dq", "dk"))
    print(f"two-hot N={N} causal={causal}:", {k: tuple(round(x, 5) for x in v) for k, v in errs.items()})


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tiestress_small_exact(cuda_device, mode):
    """Quantised scores (exact in fp32): rm, rs, m bit-exact, all three tie classes."""
    w = workloads.make("tiestress", B=1, H=2, N=640)
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=True)
    _check_fix_invariants(gpu, mode)
    cls = w.notes["tie_class"]
    assert np.all(gpu["rs"][cls >= 0] == 2)
    if mode in (1, 2):
        assert np.all(gpu["m"][cls == 2] == 1.0)
        if mode == 1:
            assert np.all(gpu["m"][cls == 1] == 0.0)


def _margin_case(N, causal):
    """Every row has a tied maximum rm = 2^-9 (1/8-grid inputs, exact scores):
    q = +-e_i / 8 on dims 0-3; keys 0 and N/2 are +(1/8) there, the rest -(1/8)."""
    rng = np.random.default_rng(N)
    q = np.zeros((1, 2, N, 64), np.float32)
    k = np.zeros((1, 2, N, 64), np.float32)
    for i in range(N):
        q[:, :, i, i % 4] = 0.125 if i % 2 == 0 else -0.125
    k[:, :, :, :4] = -0.125
    k[:, :, 0, :4] = 0.125
    k[:, :, N // 2, :4] = 0.125
    mk = lambda: workloads.to_bf16_values(rng.standard_normal((1, 2, N, 64)).astype(np.float32))
    return workloads.Workload("margin", 1, 2, N, 64, causal, 0, q, k, mk(), mk(), np.zeros((1, 2, N), bool))


@pytest.mark.parametrize("causal", [True, False])
def test_margin_mode_small_ties(cuda_device, causal):
    """Tied maxima of size 2^-9: the fp32 rule leaves bf16(P_bar) = 1 on those
    rows; the margin mode moves m by 2^-8 (bit-exact against the oracle) and
    keeps it below 1.  Forward outputs and dV are compared with the oracle;
    dQ and dK of this construction are sums of nearly uniform dS over two
    key (query) values, pure cancellation below the bf16 dS rounding, so
    their parity is left to the general grid (which runs mode 2 too)."""
    w = _margin_case(384, causal)
    for mode in (1, 2):
        gpu = P.run_gpu(w, mode)
        ref = P.oracle(w, mode, o_gpu=gpu["o"])
        P.assert_close("o", gpu["o"], ref["o"])
        P.assert_close("dv", gpu["dv"], ref["dv"])
        assert np.abs(gpu["lse"] - ref["lse"]).max() <= P.LSE_ABS
        for key in ("rm", "rs", "m"):
            assert np.array_equal(gpu[key], ref[key]), key
        _check_fix_invariants(gpu, mode)
        tied = gpu["rs"] > 1
        small = tied & (np.abs(gpu["rm"]) < 2.0 ** -8)
        assert small.sum() > 100
        b = bf16.round_bf16(gpu["pbar_max"][small].astype(np.float32))
        if mode == 1:
            assert np.all(b == 1.0)
        else:
            assert np.all(b < 1.0)
            assert np.all(gpu["m"][small] == gpu["rm"][small] + np.float32(2.0 ** -8))


@pytest.mark.parametrize("d", [64, 128])
def test_empty_problem_is_noop(cuda_device, d):
    import bf16_numerics_b200 as fa
    q = torch.empty(1, 2, 0, d, device=cuda_device, dtype=torch.bfloat16)
    o, lse, st = fa.attention_forward(q, q, q, True, 1, 2.0)
    assert o.numel() == 0
    dq, dk, dv, ws = fa.attention_backward(q, q, q, o, q, lse, st.m, True, 1, 2.0,
                                           workspace=torch.empty(256, device=cuda_device, dtype=torch.uint8))
    assert dq.numel() == 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 7, 129])
def test_tiny_lengths(cuda_device, N, d):
    """Lengths below and just above one tile."""
    if d == 64:
        w = workloads.make("g2s", B=1, H=1, N=N, seed=N)
    else:
        rng = np.random.default_rng(1000 + N)
        mk = lambda: workloads.to_bf16_values(rng.standard_normal((1, 1, N, 128)).astype(np.float32))
        w = workloads.Workload("d128", 1, 1, N, 128, True, 0, mk(), mk(), mk(), mk(), np.zeros((1, 1, N), bool))
    for mode in (0, 1):
        gpu = P.run_gpu(w, mode)
        ref = P.oracle(w, mode, o_gpu=gpu["o"])
        P.compare(gpu, ref, exact_stats=False)


@pytest.mark.parametrize("causal", [True, False])
def test_d128_several_items_per_cta(cuda_device, causal):
    """More work items (key blocks x heads) than SMs at d = 128, compared on
    every head: each persistent CTA of the backward walks several items, so
    the K/V reloads, the accumulator hand-over between items and the dQ
    reduce-adds from different CTAs into the same query block are exercised."""
    rng = np.random.default_rng(4242)
    B, H, N = 2, 48, 256 + 40
    mk = lambda: workloads.to_bf16_values(rng.standard_normal((B, H, N, 128)).astype(np.float32))
    w = workloads.Workload("d128", B, H, N, 128, causal, 0, mk(), mk(), mk(), mk(), np.zeros((B, H, N), bool))
    assert B * H * ((N + 127) // 128) > 148
    gpu = P.run_gpu(w, 1)
    ref = P.oracle(w, 1, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=False)


# ------------------------------------------------- full-size workloads (sampled)

# (batch, head) pairs the oracle computes, per workload and softmax mode; the
# GPU runs the whole workload in the launch configuration the bench times
FULL = {
    "g2s": {0: [(1, 2), (6, 10)], 1: [(0, 0), (3, 7), (7, 11)], 2: [(2, 4), (5, 1)]},
    "g2m": {0: [(4, 3)], 1: [(0, 0), (5, 9)], 2: [(7, 15)]},
    "tiestress": {0: [(1, 1)], 1: [(0, 0), (2, 5)], 2: [(3, 11)]},
    "long": {0: [(0, 3), (1, 8)], 1: [(0, 0), (0, 9), (1, 4), (1, 15)], 2: [(0, 12), (1, 6)]},
}


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("name", ["g2s", "g2m", "tiestress", "long"])
def test_full_size_sampled_heads(cuda_device, name, mode):
    w = workloads.make(name)
    gpu = P.run_gpu(w, mode)
    pairs = FULL[name][mode]
    ref = P.oracle(w, mode, pairs=pairs, o_gpu=P.head_slice(gpu["o"], pairs))
    errs = P.compare(gpu, ref, exact_stats=(name == "tiestress"), pairs=pairs)
    print(f"{name} mode {mode} heads {pairs}:", {k: tuple(round(x, 5) for x in v) for k, v in errs.items()})
    _check_fix_invariants(gpu, mode)
    # properties that hold at any size, on every row
    for key in ("o", "dq", "dk", "dv", "lse"):
        assert np.all(np.isfinite(gpu[key])), key
    if name in ("g2s", "long"):
        assert np.all(gpu["rs"][w.forced_tie_rows] >= 2)
    if name == "tiestress":
        cls = w.notes["tie_class"]
        assert np.all(gpu["rs"][cls >= 0] == 2)
        assert np.all(gpu["rm"][cls == 0] > 0) and np.all(gpu["rm"][cls == 1] < 0)
        assert np.all(gpu["rm"][cls == 2] == 0)


@pytest.mark.parametrize("name", ["tiestress", "g2s"])
def test_delta_bias_diagnostic(cuda_device, name):
    """Size of the delta bias: the gradient the GPU computes (delta from its own
    bf16 O, as any FlashAttention backward does) against the chained float64
    gradient (delta from the exact O).  dS is linear in delta, so the oracle's
    given-O and chained gradients differ by exactly the propagated delta
    error; by the triangle inequality the chained error is at most the
    given-O bar plus that difference, element by element.  The sizes are
    printed for the record."""
    w = workloads.make(name).heads([(0, 0)])
    gpu = P.run_gpu(w, 1)
    ref = P.oracle(w, 1, o_gpu=gpu["o"])
    for key in ("dq", "dk", "dv"):
        given = np.abs(gpu[key] - ref[key]).max() / np.abs(ref[key]).max()
        chained = np.abs(gpu[key] - ref[key + "_chained"]).max() / np.abs(ref[key + "_chained"]).max()
        print(f"{name} {key}: max err vs given-O oracle {given:.4f}, vs chained float64 oracle {chained:.4f}")
        bar = P.MAXABS * max(np.abs(ref[key]).max(), np.abs(ref[key + "_chained"]).max()) + P.ATOL
        propagated = np.abs(ref[key] - ref[key + "_chained"])
        assert np.all(np.abs(gpu[key] - ref[key + "_chained"]) <= bar + propagated)
    assert np.array_equal(ref["dv"], ref["dv_chained"])  # dV does not depend on delta
    d_bias = (ref["delta"] - ref["delta_chained"]).mean()
    print(f"{name}: mean delta(bf16 O) - delta(float64 O) = {d_bias:.3e}")


def test_modes_agree_on_gpu(cuda_device):
    """Shift invariance: both modes give the same attention up to rounding."""
    w = workloads.make("g2s", B=2, H=3)
    g0 = P.run_gpu(w, 0)
    g1 = P.run_gpu(w, 1)
    for key in ("o", "dq", "dk", "dv"):
        P.assert_close(key, g1[key], g0[key])


# --------------------------------------- high-precision O for the delta term

@pytest.mark.parametrize("d", [64, 128])
def test_o_hp_forward(cuda_device, d):
    """fa_fwd_o_hp: o_hp carries P_bar to ~16 bits, so it matches the float64
    O far inside the bf16 tolerance (1e-4 of max|O| here, against 1e-2 for
    the bf16 o); every other output equals fa_fwd's bit for bit."""
    w = workloads.make("g2s", B=1, H=2, N=200, seed=7) if d == 64 else _d128_case(200, True, 0.5)
    hp = P.run_gpu_o_hp(w, 1)
    lp = P.run_gpu(w, 1)
    ref = P.oracle(w, 1, o_gpu=hp["o"])
    err_hp = np.abs(hp["o_hp"] - ref["o"]).max() / np.abs(ref["o"]).max()
    err_lp = np.abs(lp["o"] - ref["o"]).max() / np.abs(ref["o"]).max()
    print(f"d={d}: max |O - O_float64| / max|O|: o_hp {err_hp:.2e}, bf16 o {err_lp:.2e}")
    assert err_hp <= 1e-4
    for key in ("o", "lse", "m"):
        assert np.array_equal(lp[key], hp[key]), key


@pytest.mark.parametrize("name", ["tiestress", "g2s"])
def test_o_hp_backward_removes_the_delta_bias(cuda_device, name):
    """The pages' remedy (P in higher precision wherever it feeds dP): delta
    from the ~16-bit-P O_hp is the float64 delta to ~1e-5, and the gradients
    come close to the chained float64 gradient; with delta from the bf16 O
    they carry its error (biased on rows with tied maxima)."""
    w = workloads.make(name).heads([(0, 0)])
    lp = P.run_gpu(w, 1)
    hp = P.run_gpu_o_hp(w, 1)
    ref = P.oracle(w, 1)   # chained: delta from the oracle's float64 O
    scale = np.abs(ref["delta"]).max()
    d_lp = np.abs(lp["delta"] - ref["delta"]).max() / scale
    d_hp = np.abs(hp["delta"] - ref["delta"]).max() / scale
    print(f"{name}: max |delta - delta(float64 O)| / max|delta|: bf16 O {d_lp:.2e}, O_hp {d_hp:.2e}")
    assert d_hp <= 1e-4 and d_hp < d_lp
    for key in ("dq", "dk", "dv"):
        e_lp = np.abs(lp[key] - ref[key]).max() / np.abs(ref[key]).max()
        e_hp = np.abs(hp[key] - ref[key]).max() / np.abs(ref[key]).max()
        print(f"{name} {key}: max err vs chained float64: delta from bf16 O {e_lp:.4f}, from O_hp {e_hp:.4f}")
        P.assert_close(key, hp[key], ref[key])


@pytest.mark.parametrize("name", ["tiestress", "g2s", "long"])
def test_o_hp_pair_meets_the_bar_end_to_end(cuda_device, name):
    """End to end against the chained float64 oracle (delta from the exact O):
    fa_fwd_o_hp -> fa_bwd_o_hp at full size meets the 1e-2 bar on O,
    dQ, dK and dV of sampled heads.  (The default fa_fwd -> fa_bwd pair carries
    the delta bias of its bf16 O and misses it on the tie-stress dQ; see
    test_o_hp_backward_removes_the_delta_bias.)"""
    w = workloads.make(name)
    pairs = {"tiestress": [(0, 0), (3, 11)], "g2s": [(0, 0), (7, 11)], "long": [(1, 15)]}[name]
    hp = P.run_gpu_o_hp(w, 1)
    ref = P.oracle(w, 1, pairs=pairs)  # chained
    sel = lambda x: P.head_slice(x, pairs)
    errs = {key: P.assert_close(key, sel(hp[key]), ref[key]) for key in ("dq", "dk", "dv")}
    errs["o_hp"] = P.assert_close("o_hp", sel(hp["o_hp"]), ref["o"])
    errs["o"] = P.assert_close("o", sel(hp["o"]), ref["o"])
    print(f"{name} o_hp pair vs chained float64 oracle:", {k: tuple(round(x, 5) for x in v) for k, v in errs.items()})


# ---------------------------------------------- bias diagnostic (negative V)

@pytest.mark.parametrize("name", ["tiestress", "tiny"])
def test_bias_diagnostic_negative_v(cuda_device, name):
    """The pages' Figure 6 question on this hardware: on rows with a tied
    maximum, does O drift in one direction on the value columns whose mean is
    negative?  Reports mean(O_gpu - O_float64) over the tied rows, for the
    negative-mean columns and for the rest, and the mean delta error, in all
    three modes.  Here the P V product accumulates in fp32 (TMEM) and only
    P_bar and O are rounded to bf16 (RNE); the bound is one bf16 step of the
    mean |O| (2^-8 relative), a drift of that size would be visible in every
    row."""
    w = workloads.make(name) if name == "tiny" else workloads.make(name).heads([(0, 0)])
    neg_cols = 16 if name == "tiny" else 32
    for mode in (0, 1, 2):
        gpu = P.run_gpu(w, mode)
        ref = P.oracle(w, mode)
        tied = ref["rs"] > 1
        err = gpu["o"] - ref["o"]
        e_neg = err[tied][:, :neg_cols].mean()
        e_rest = err[tied][:, neg_cols:].mean()
        scale = np.abs(ref["o"][tied]).mean()
        d_err = (gpu["delta"] - ref["delta"])[tied].mean()
        print(f"{name} mode {mode}: tied rows {int(tied.sum())}, mean O error on negative-mean columns "
              f"{e_neg:+.3e}, other columns {e_rest:+.3e} (mean |O| {scale:.3f}); mean delta error {d_err:+.3e}")
        assert abs(e_neg) <= 2.0 ** -8 * scale and abs(e_rest) <= 2.0 ** -8 * scale

"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases are compared on every output element; the full-size workloads run
in the launch configuration the benchmark uses and are compared on sampled
(batch, head) pairs that the oracle computes exactly (heads are independent).
"""

import numpy as np
import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


def _small(name, B, H, N, seed=None):
    return workloads.make(name, B=B, H=H, N=N, seed=seed)


def _check_fix_invariants(gpu, mode):
    tied = gpu["rs"] > 1
    if mode == 1:
        assert np.all(gpu["pbar_max"][tied] < 1.0)
        assert np.all(gpu["pbar_max"][~tied] == 1.0)
    else:
        assert np.all(gpu["pbar_max"] == 1.0)


@pytest.mark.parametrize("mode", [0, 1])
def test_tiny_exact_stats(cuda_device, mode):
    w = workloads.make("tiny")
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=True)
    _check_fix_invariants(gpu, mode)
    assert (ref["rs"] > 1).any()


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [384, 200])
def test_small_grid(cuda_device, mode, causal, d, N):
    """Several tiles plus a ragged tail (N = 200), both masks, both head dims."""
    w = workloads.make("g2s", B=1, H=2, N=N, seed=100 + N + d)
    if d == 128:
        rng = np.random.default_rng(N)
        shape = (1, 2, N, 128)
        mk = lambda: workloads.to_bf16_values(rng.standard_normal(shape).astype(np.float32))
        w = workloads.Workload("d128", 1, 2, N, 128, causal, 0, mk(), mk(), mk(), mk(), np.zeros((1, 2, N), bool))
        w.k[:, :, N // 2] = w.k[:, :, 0]
        w.q[:, :, N - 10:] = np.float32(0.5) * w.k[:, :, :1]
    w.causal = causal
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=False)
    _check_fix_invariants(gpu, mode)


@pytest.mark.parametrize("mode", [0, 1])
def test_tiestress_small_exact(cuda_device, mode):
    """Quantised scores (exact in fp32): rm, rs, m bit-exact, all three tie classes."""
    w = workloads.make("tiestress", B=1, H=2, N=640)
    gpu = P.run_gpu(w, mode)
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=True)
    _check_fix_invariants(gpu, mode)
    cls = w.notes["tie_class"]
    assert np.all(gpu["rs"][cls >= 0] == 2)
    if mode == 1:
        assert np.all(gpu["m"][cls == 2] == 1.0) and np.all(gpu["m"][cls == 1] == 0.0)


def test_empty_problem_is_noop(cuda_device):
    import bf16_numerics_b200 as fa
    q = torch.empty(1, 2, 0, 64, device=cuda_device, dtype=torch.bfloat16)
    o, lse, st = fa.attention_forward(q, q, q, True, 1, 2.0)
    assert o.numel() == 0
    dq, dk, dv, ws = fa.attention_backward(q, q, q, o, q, lse, st.m, True, 1, 2.0,
                                           workspace=torch.empty(256, device=cuda_device, dtype=torch.uint8))
    assert dq.numel() == 0


@pytest.mark.parametrize("N", [1, 7, 129])
def test_tiny_lengths(cuda_device, N):
    """Lengths below and just above one tile."""
    w = workloads.make("g2s", B=1, H=1, N=N, seed=N)
    for mode in (0, 1):
        gpu = P.run_gpu(w, mode)
        ref = P.oracle(w, mode, o_gpu=gpu["o"])
        P.compare(gpu, ref, exact_stats=False)


# ------------------------------------------------- full-size workloads (sampled)

FULL = {
    "g2s": [(0, 0), (3, 7), (7, 11)],
    "g2m": [(0, 0), (5, 9)],
    "tiestress": [(0, 0), (2, 5)],
    "long": [(1, 15)],
}


@pytest.mark.parametrize("name", ["g2s", "g2m", "tiestress", "long"])
def test_full_size_sampled_heads(cuda_device, name):
    w = workloads.make(name)
    mode = 1
    gpu = P.run_gpu(w, mode)
    pairs = FULL[name]
    ref = P.oracle(w, mode, pairs=pairs, o_gpu=P.head_slice(gpu["o"], pairs))
    P.compare(gpu, ref, exact_stats=(name == "tiestress"), pairs=pairs)
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


def test_modes_agree_on_gpu(cuda_device):
    """Shift invariance: both modes give the same attention up to rounding."""
    w = workloads.make("g2s", B=2, H=3)
    g0 = P.run_gpu(w, 0)
    g1 = P.run_gpu(w, 1)
    for key in ("o", "dq", "dk", "dv"):
        P.assert_close(key, g1[key], g0[key])

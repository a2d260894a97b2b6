"""The backward's workspace across calls (GPU).

fa_bwd's workspace holds delta, the fp32 dQ accumulator and the d = 128
work-item counter; its contents on entry must not matter.  These tests run
fa_bwd on workspaces filled with garbage, left by a previous call of the same
shape, with the accumulator overwritten in between, last used by a call of
another head dimension, and shared with the high-precision-O backward, and
check dQ, dK, dV and delta against the oracle each time (and that the same
inputs give the same bits).
"""

import numpy as np
import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


def _workload(B, H, N, d, causal, seed):
    rng = np.random.default_rng(seed)
    mk = lambda: workloads.to_bf16_values(rng.standard_normal((B, H, N, d)).astype(np.float32))
    return workloads.Workload(f"ws{d}", B, H, N, d, causal, 0, mk(), mk(), mk(), mk(), np.zeros((B, H, N), bool))


def _check_call(w, ws, mode=1):
    """One forward + backward on workspace ws; compare with the oracle."""
    dev = ws.device
    q, k, v, do = (P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    o, lse, st = fa.attention_forward(q, k, v, w.causal, mode, 2.0)
    dq, dk, dv, _ = fa.attention_backward(q, k, v, o, do, lse, st.m, w.causal, mode, 2.0, workspace=ws)
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    B, H, N, d = q.shape
    off_delta, _ = fa.fa_bwd_workspace_offsets(B, H, N, d)
    delta = ws[off_delta:off_delta + B * H * N * 4].view(torch.float32).view(B, H, N)
    gpu = {"o": o, "lse": lse, "rm": st.rm, "rs": st.rs, "m": st.m, "dq": dq, "dk": dk, "dv": dv, "delta": delta}
    gpu = {k_: v_.float().cpu().numpy() if v_.dtype != torch.int32 else v_.cpu().numpy() for k_, v_ in gpu.items()}
    ref = P.oracle(w, mode, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=False)
    return gpu


def test_garbage_then_reuse_then_overwritten_accumulator():
    w = _workload(1, 3, 384, 64, True, 11)
    B, H, N, d = w.q.shape
    nbytes = fa.fa_bwd_workspace_bytes(B, H, N, d)
    g = torch.Generator(device="cuda:0").manual_seed(5)
    ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device="cuda:0", generator=g)
    first = _check_call(w, ws)
    second = _check_call(w, ws)
    for key in ("dq", "dk", "dv", "delta"):
        assert np.array_equal(first[key], second[key]), key  # the same inputs give the same bits
    _, off_acc = fa.fa_bwd_workspace_offsets(B, H, N, d)
    ws[off_acc:off_acc + B * H * N * d * 4] = 0x7F  # accumulator overwritten between calls
    third = _check_call(w, ws)
    assert np.array_equal(first["dq"], third["dq"])


def test_zero_filled_workspace_noncausal_ragged():
    w = _workload(2, 2, 200, 64, False, 12)
    B, H, N, d = w.q.shape
    ws = torch.zeros(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda:0")
    _check_call(w, ws, mode=0)
    _check_call(w, ws, mode=2)


def test_workspace_last_used_at_d128_then_d64():
    w128 = _workload(1, 2, 256, 128, True, 13)
    w64 = _workload(1, 4, 256, 64, True, 14)
    nbytes = max(fa.fa_bwd_workspace_bytes(*x.q.shape) for x in (w128, w64))
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda:0")
    _check_call(w128, ws[:fa.fa_bwd_workspace_bytes(*w128.q.shape)])
    _check_call(w64, ws[:fa.fa_bwd_workspace_bytes(*w64.q.shape)])
    _check_call(w128, ws[:fa.fa_bwd_workspace_bytes(*w128.q.shape)])
    _check_call(w64, ws[:fa.fa_bwd_workspace_bytes(*w64.q.shape)])


def test_workspace_shared_with_the_high_precision_backward():
    """fa_bwd, then fa_bwd_o_hp (delta from the fp32 O), then fa_bwd again on
    one workspace."""
    w = _workload(1, 2, 384, 64, True, 15)
    B, H, N, d = w.q.shape
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda:0")
    _check_call(w, ws)
    dev = ws.device
    q, k, v, do = (P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    o = torch.empty_like(q)
    o_hp = torch.empty(B, H, N, d, device=dev, dtype=torch.float32)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    st = fa.RowStats.empty(B, H, N, dev)
    fa.fa_fwd_o_hp(q, k, v, o, o_hp, lse, st, True, 1, 2.0)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa.fa_bwd_o_hp(q, k, v, o_hp, do, lse, st.m, dq, dk, dv, ws, True, 1, 2.0)
    torch.cuda.synchronize(dev)
    assert fa.fa_device_error()[0] == 0
    _check_call(w, ws)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_calls_back_to_back_on_one_workspace(d):
    """Two fa_bwd calls in a row on one stream and one workspace, with no
    forward between them: the second call's delta kernel follows the first
    call's dQ convert directly, and it clears the accumulator the convert
    reads.  Both calls must match the oracle (the second has another dO, so a
    clear that overtook the convert would show in the first call's dQ)."""
    w1 = _workload(1, 2, 384, d, True, 21 + d)
    rng = np.random.default_rng(99 + d)
    do2 = workloads.to_bf16_values(rng.standard_normal(w1.do.shape).astype(np.float32))
    w2 = workloads.Workload(f"ws{d}b", *w1.q.shape, w1.causal, 0, w1.q, w1.k, w1.v, do2, w1.forced_tie_rows)
    dev = torch.device("cuda:0")
    B, H, N, _ = w1.q.shape
    q, k, v, do1 = (P.to_dev(x, dev) for x in (w1.q, w1.k, w1.v, w1.do))
    do2_t = P.to_dev(do2, dev)
    o, lse, st = fa.attention_forward(q, k, v, True, 1, 2.0)
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, N, d),), 0x5A, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    res = []
    for do_t in (do1, do2_t):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fa.fa_bwd(q, k, v, o, do_t, lse, st.m, dq, dk, dv, ws, True, 1, 2.0)
        res.append((dq, dk, dv))
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    o_np = o.float().cpu().numpy()
    for w, (dq, dk, dv) in zip((w1, w2), res):
        gpu = {"o": o_np, "lse": lse.float().cpu().numpy(), "rm": st.rm.float().cpu().numpy(),
               "rs": st.rs.cpu().numpy(), "m": st.m.float().cpu().numpy(),
               "dq": dq.float().cpu().numpy(), "dk": dk.float().cpu().numpy(), "dv": dv.float().cpu().numpy()}
        ref = P.oracle(w, 1, o_gpu=o_np)
        P.compare(gpu, ref, exact_stats=False)

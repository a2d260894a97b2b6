"""Out-of-bounds writes (GPU).

Every output of fa_fwd / fa_bwd (and of the high-precision pair), and the
backward's workspace, is placed between two 4 KiB guard regions filled with a
known byte pattern.  After the calls the guards must be unchanged, and the
outputs must still match the oracle.  The lengths are ragged (N not a multiple
of the 128-row tile, down to N = 7), so the TMA stores of O, dK and dV, the
row-statistic stores, the delta kernel's accumulator clear and the dQ
reduce-adds all run up to the ends of their buffers.
"""

import numpy as np
import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (keeps every view 256-byte aligned)
PATTERN = 0xA5


class Guarded:
    """Views into guard-padded byte buffers, and the check of the guards."""

    def __init__(self, dev):
        self.dev = dev
        self.bufs = {}

    def view(self, name, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=self.dev)
        self.bufs[name] = (buf, nbytes)
        return buf[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check(self):
        for name, (buf, nbytes) in self.bufs.items():
            head, tail = buf[:GUARD], buf[GUARD + nbytes:]
            assert bool((head == PATTERN).all()), f"{name}: bytes before the buffer were written"
            assert bool((tail == PATTERN).all()), f"{name}: bytes after the buffer were written"


def _workload(B, H, N, d, causal, seed):
    rng = np.random.default_rng(seed)
    mk = lambda: workloads.to_bf16_values(rng.standard_normal((B, H, N, d)).astype(np.float32))
    return workloads.Workload(f"canary{d}", B, H, N, d, causal, 0, mk(), mk(), mk(), mk(), np.zeros((B, H, N), bool))


def _host(x):
    return x.cpu().numpy() if x.dtype == torch.int32 else x.float().cpu().numpy()


@pytest.mark.parametrize("d,N,causal", [(64, 200, True), (64, 129, False), (128, 200, True), (128, 7, False)])
def test_outputs_stay_inside_their_buffers(d, N, causal):
    B, H = 1, 2
    w = _workload(B, H, N, d, causal, 31 + N + d)
    dev = torch.device("cuda:0")
    q, k, v, do = (P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    g = Guarded(dev)
    o = g.view("o", (B, H, N, d), torch.bfloat16)
    lse = g.view("lse", (B, H, N), torch.float32)
    st = fa.RowStats(g.view("rm", (B, H, N), torch.float32), g.view("rs", (B, H, N), torch.int32),
                     g.view("m", (B, H, N), torch.float32), g.view("pbar_max", (B, H, N), torch.float32))
    fa.fa_fwd(q, k, v, o, lse, st, causal, 1, 2.0)
    dq = g.view("dq", (B, H, N, d), torch.bfloat16)
    dk = g.view("dk", (B, H, N, d), torch.bfloat16)
    dv = g.view("dv", (B, H, N, d), torch.bfloat16)
    ws = g.view("workspace", (fa.fa_bwd_workspace_bytes(B, H, N, d),), torch.uint8)
    fa.fa_bwd(q, k, v, o, do, lse, st.m, dq, dk, dv, ws, causal, 1, 2.0)
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    g.check()
    gpu = {"o": o, "lse": lse, "rm": st.rm, "rs": st.rs, "m": st.m, "dq": dq, "dk": dk, "dv": dv}
    gpu = {key: _host(val) for key, val in gpu.items()}
    P.compare(gpu, P.oracle(w, 1, o_gpu=gpu["o"]), exact_stats=False)


@pytest.mark.parametrize("d,N", [(64, 200), (128, 129)])
def test_high_precision_outputs_stay_inside_their_buffers(d, N):
    """fa_fwd_o_hp (also writes the fp32 O_hp with plain stores) and
    fa_bwd_o_hp (delta from O_hp)."""
    B, H = 1, 2
    w = _workload(B, H, N, d, True, 41 + N + d)
    dev = torch.device("cuda:0")
    q, k, v, do = (P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    g = Guarded(dev)
    o = g.view("o", (B, H, N, d), torch.bfloat16)
    o_hp = g.view("o_hp", (B, H, N, d), torch.float32)
    lse = g.view("lse", (B, H, N), torch.float32)
    st = fa.RowStats(g.view("rm", (B, H, N), torch.float32), g.view("rs", (B, H, N), torch.int32),
                     g.view("m", (B, H, N), torch.float32), g.view("pbar_max", (B, H, N), torch.float32))
    fa.fa_fwd_o_hp(q, k, v, o, o_hp, lse, st, True, 1, 2.0)
    dq = g.view("dq", (B, H, N, d), torch.bfloat16)
    dk = g.view("dk", (B, H, N, d), torch.bfloat16)
    dv = g.view("dv", (B, H, N, d), torch.bfloat16)
    ws = g.view("workspace", (fa.fa_bwd_workspace_bytes(B, H, N, d),), torch.uint8)
    fa.fa_bwd_o_hp(q, k, v, o_hp, do, lse, st.m, dq, dk, dv, ws, True, 1, 2.0)
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    g.check()
    assert np.isfinite(_host(o_hp)).all()
    for key, val in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.isfinite(_host(val)).all(), key

"""The bounded-wait exit path on the GPU, without a fault.

Every mbarrier wait in the kernels gives up after a time limit: the waiting
thread records kernel id << 24 | site << 16 | block in a device word, raises
its CTA's abort flag, and every role of the CTA drains its copies and
products, frees its tensor memory and returns.  Here a test hook
(fa_debug_inject_stall) makes CTA 0 withhold one arrive on the barrier that
hands P to the MMA warp -- a flag that nothing else sets, with no bulk copy
outstanding on it -- under a short wait limit (fa_debug_set_wait_limit_ns).
The call must end with FA_ERR_TIMEOUT naming that kernel and CTA 0, and the
next normal call on the same context must run and match the oracle (the
stalled CTA released its tensor memory and left no copy in flight).
"""

import time

import numpy as np
import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from bf16_numerics_b200 import _abi
from tests import parity as P

pytestmark = pytest.mark.gpu

LIMIT_NS = 50_000_000  # 50 ms: far above every legitimate wait of these small problems


def _workload(d):
    if d == 64:
        return workloads.make("g2s", B=1, H=2, N=384, seed=515)
    rng = np.random.default_rng(516)
    mk = lambda: workloads.to_bf16_values(rng.standard_normal((1, 2, 384, 128)).astype(np.float32))
    return workloads.Workload("d128", 1, 2, 384, 128, True, 0, mk(), mk(), mk(), mk(), np.zeros((1, 2, 384), bool))


def _stalled_call(w, kernel_id, dev):
    q, k, v, do = (P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    st = fa.RowStats.empty(B, H, N, dev)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), device=dev, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    torch.cuda.synchronize(dev)
    assert fa.fa_device_error() == (0, 0)
    try:
        fa.fa_debug_set_wait_limit_ns(LIMIT_NS)
        fa.fa_debug_inject_stall(kernel_id)
        t0 = time.perf_counter()
        fa.fa_fwd(q, k, v, o, lse, st, True, 1, 2.0)
        if kernel_id != _abi.FA_ERRWORD_FWD:
            fa.fa_bwd(q, k, v, o, do, lse, st.m, dq, dk, dv, ws, True, 1, 2.0)
        status, word = fa.fa_device_error()  # synchronises the device
        elapsed = time.perf_counter() - t0
    finally:
        fa.fa_debug_inject_stall(0)
        fa.fa_debug_set_wait_limit_ns(0)
    return status, word, elapsed


@pytest.mark.parametrize("kernel_id, d", [(_abi.FA_ERRWORD_FWD, 64), (_abi.FA_ERRWORD_FWD, 128),
                                          (_abi.FA_ERRWORD_BWD_D64, 64), (_abi.FA_ERRWORD_BWD_D128, 128)])
def test_withheld_arrive_ends_in_timeout_and_context_stays_usable(cuda_device, kernel_id, d):
    w = _workload(d)
    status, word, elapsed = _stalled_call(w, kernel_id, cuda_device)
    print(f"kernel {kernel_id} d={d}: status {status}, error word {word:#010x} "
          f"(site {(word >> 16) & 0xff}), {elapsed * 1e3:.1f} ms")
    assert status == _abi.FA_ERR_TIMEOUT
    assert word >> 24 == kernel_id
    assert word & 0xFFFF == 0                     # CTA 0, the one that withheld the arrive
    assert elapsed < 5.0                          # the 50 ms limit, not the 2 s default many times over
    assert fa.fa_device_error() == (0, 0)         # reading cleared the word
    # the next normal call runs on the same context and matches the oracle
    gpu = P.run_gpu(w, 1)
    ref = P.oracle(w, 1, o_gpu=gpu["o"])
    P.compare(gpu, ref, exact_stats=False)


def test_inject_rejects_unknown_kernel_ids(cuda_device):
    with pytest.raises(fa.FaError):
        fa.fa_debug_inject_stall(2)

"""The allocation-free backward (fa_bwd_noalloc) against the workspace one.

fa_bwd_noalloc serves callers that cannot allocate device memory (a runtime
with a static memory plan fixed at start-up, or a plug-in that owns no
allocator): its scratch lives in a static device array inside the library.
This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from bf16_numerics_b200 import _abi
from tests import parity as P

pytestmark = pytest.mark.gpu

NOALLOC_MAX = 32 * 1024 * 1024  # FA_NOALLOC_SCRATCH_BYTES in include/fa_b200.h


def _noalloc_fn():
    lib = _abi.load()
    fn = lib.fa_bwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp]
    fn.restype = i
    return fn


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name, mode", [("g2s", 1), ("tiestress", 0)])
def test_noalloc_matches_workspace_backward(cuda_device, name, mode):
    w = workloads.make(name) if name == "g2s" else workloads.make(name, B=1, H=2, N=1024)
    assert fa.fa_bwd_workspace_bytes(*w.shape) <= NOALLOC_MAX
    q, k, v, do = (P.to_dev(x, cuda_device) for x in (w.q, w.k, w.v, w.do))
    o, lse, st = fa.attention_forward(q, k, v, w.causal, mode, 2.0)
    dq_ref, dk_ref, dv_ref, _ = fa.attention_backward(q, k, v, o, do, lse, st.m, w.causal, mode, 2.0)
    ref = [t.float().cpu().numpy() for t in (dq_ref, dk_ref, dv_ref)]
    fn = _noalloc_fn()
    B, H, N, d = w.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):  # the scratch keeps the previous call's contents
        dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
        code = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(st.m), _ptr(dq), _ptr(dk), _ptr(dv),
                  B, H, N, d, int(w.causal), mode, 2.0, stream)
        assert code == _abi.FA_OK, _abi.status_string(code)
        torch.cuda.synchronize()
        assert fa.fa_device_error()[0] == 0
        for key, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            P.assert_close(f"{key} (call {call})", got.float().cpu().numpy(), want)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    fn = _noalloc_fn()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    B, H, N, d = 8, 16, 8192, 64  # needs 8*16*8192*(4 + 256) bytes, far above 32 MiB
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) > NOALLOC_MAX
    code = fn(*([fake] * 10), B, H, N, d, 1, 1, 2.0, None)
    assert code == _abi.FA_ERR_WORKSPACE

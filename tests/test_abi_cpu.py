"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status before
touching CUDA.  (Nothing here launches a kernel.)"""

import ctypes
import os
import re

import pytest

from bf16_numerics_b200 import _abi
from bf16_numerics_b200.build import INCLUDE, build_library

HEADER = os.path.join(INCLUDE, "fa_b200.h")


@pytest.fixture(scope="module")
def lib():
    build_library()
    return _abi.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared_functions() == sorted(_abi.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_library_is_sm100a_only():
    # the build command targets exactly one architecture
    from bf16_numerics_b200.build import nvcc_command
    cmd = " ".join(nvcc_command())
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert cmd.count("-gencode") == 1


def test_status_strings(lib):
    for code in range(6):
        assert _abi.status_string(code)
    assert _abi.status_string(0) == "ok"


P = ctypes.c_void_p(0x10000)      # aligned fake device pointer (never dereferenced)
MIS = ctypes.c_void_p(0x10008)    # 8-byte aligned only
NUL = None


def fwd(lib, q=P, k=P, v=P, o=P, lse=P, stats=None, B=1, H=2, N=128, d=64, causal=1, mode=1, beta=2.0):
    return lib.fa_fwd(q, k, v, o, lse, stats, B, H, N, d, causal, mode, beta, None)


def bwd(lib, q=P, lse=P, row_m=P, ws=ctypes.c_void_p(0x100000), ws_bytes=1 << 30, B=1, H=2, N=128, d=64,
        causal=1, mode=1, beta=2.0):
    return lib.fa_bwd(q, P, P, P, P, lse, row_m, P, P, P, ws, ws_bytes, B, H, N, d, causal, mode, beta, None)


def test_fwd_argument_errors(lib):
    assert fwd(lib, d=96) == _abi.FA_ERR_UNSUPPORTED
    assert fwd(lib, d=32) == _abi.FA_ERR_UNSUPPORTED
    assert fwd(lib, beta=1.0) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, beta=0.5) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, beta=float("nan")) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, beta=float("inf")) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, mode=3) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, mode=-1) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, mode=2, beta=1.0) == _abi.FA_ERR_INVALID_ARG  # the margin mode is a stabilised mode
    assert fwd(lib, causal=2) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, B=-1) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, q=NUL) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, lse=NUL) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, o=MIS) == _abi.FA_ERR_INVALID_ARG
    assert fwd(lib, B=1 << 20, H=1 << 10, N=1 << 10) == _abi.FA_ERR_INVALID_ARG  # B*H*N*d >= 2^40


def test_fwd_standard_mode_ignores_beta(lib):
    # beta <= 1 is only an error in the stabilised mode; an empty problem launches nothing
    assert fwd(lib, mode=0, beta=0.0, N=0) == _abi.FA_OK


def test_empty_problems_are_noops(lib):
    assert fwd(lib, N=0, q=NUL, k=NUL, v=NUL, o=NUL, lse=NUL) == _abi.FA_OK
    assert fwd(lib, B=0) == _abi.FA_OK
    assert fwd(lib, H=0) == _abi.FA_OK
    assert bwd(lib, N=0, q=NUL) == _abi.FA_OK


def test_bwd_argument_errors(lib):
    need = lib.fa_bwd_workspace_bytes(1, 2, 128, 64)
    assert bwd(lib, ws_bytes=need - 1) == _abi.FA_ERR_WORKSPACE
    assert bwd(lib, ws=ctypes.c_void_p(0x100010)) == _abi.FA_ERR_WORKSPACE  # not 256-byte aligned
    assert bwd(lib, ws=None) == _abi.FA_ERR_WORKSPACE
    assert bwd(lib, row_m=None) == _abi.FA_ERR_INVALID_ARG                 # required when stabilised
    assert bwd(lib, row_m=None, mode=2) == _abi.FA_ERR_INVALID_ARG
    assert bwd(lib, mode=3) == _abi.FA_ERR_INVALID_ARG
    assert bwd(lib, q=MIS) == _abi.FA_ERR_INVALID_ARG
    assert bwd(lib, d=80) == _abi.FA_ERR_UNSUPPORTED
    assert bwd(lib, beta=1.0) == _abi.FA_ERR_INVALID_ARG


def test_o_hp_entry_points_argument_errors(lib):
    # forward: o_hp is required and 16-byte aligned; everything else as fa_fwd
    def fwd_hp(o_hp=P, mode=1, N=128, d=64):
        return lib.fa_fwd_o_hp(P, P, P, P, o_hp, P, None, 1, 2, N, d, 1, mode, 2.0, None)
    assert fwd_hp(o_hp=NUL) == _abi.FA_ERR_INVALID_ARG
    assert fwd_hp(o_hp=MIS) == _abi.FA_ERR_INVALID_ARG
    assert fwd_hp(mode=3) == _abi.FA_ERR_INVALID_ARG
    assert fwd_hp(d=96) == _abi.FA_ERR_UNSUPPORTED
    assert fwd_hp(N=0, o_hp=NUL) == _abi.FA_OK  # empty problem: nothing to write
    # backward: same checks as fa_bwd with the fp32 O in place of the bf16 one
    def bwd_hp(o_hp=P, ws_bytes=1 << 30, row_m=P, mode=1):
        return lib.fa_bwd_o_hp(P, P, P, o_hp, P, P, row_m, P, P, P, ctypes.c_void_p(0x100000), ws_bytes, 1, 2, 128,
                               64, 1, mode, 2.0, None)
    assert bwd_hp(o_hp=NUL) == _abi.FA_ERR_INVALID_ARG
    assert bwd_hp(o_hp=MIS) == _abi.FA_ERR_INVALID_ARG
    assert bwd_hp(row_m=None) == _abi.FA_ERR_INVALID_ARG
    assert bwd_hp(ws_bytes=16) == _abi.FA_ERR_WORKSPACE


def test_workspace_layout(lib):
    # delta | fp32 dQ accumulator | 256 bytes holding the work-item counter of the d = 128 kernel
    B, H, N, d = 8, 12, 1024, 64
    rows = B * H * N
    r256 = lambda x: (x + 255) // 256 * 256
    assert lib.fa_bwd_workspace_bytes(B, H, N, d) == r256(rows * 4) + r256(rows * d * 4) + 256
    assert lib.fa_bwd_workspace_delta_offset(B, H, N, d) == 0
    assert lib.fa_bwd_workspace_dq_offset(B, H, N, d) == r256(rows * 4)
    assert lib.fa_bwd_workspace_bytes(1, 1, 100, 128) == r256(400) + r256(100 * 128 * 4) + 256
    assert lib.fa_bwd_workspace_bytes(1, 1, 128, 96) == 0


def test_timing_read_empty(lib):
    launches = (ctypes.c_int * 4)()
    total = (ctypes.c_double * 4)()
    assert lib.fa_timing_enable(1) == _abi.FA_OK
    assert lib.fa_timing_read(launches, total) == _abi.FA_OK
    assert list(launches) == [0, 0, 0, 0]
    assert lib.fa_timing_enable(0) == _abi.FA_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libfa_b200.so"))
    with pytest.raises(ImportError):
        _abi.load()


def test_inject_stall_rejects_unknown_kernel_ids_before_touching_cuda(lib):
    # only the error-word ids of the three kernels with bounded waits (and 0) are accepted
    for bad in (2, 5, 255, 1 << 24):
        assert lib.fa_debug_inject_stall(bad) == _abi.FA_ERR_INVALID_ARG
    assert (_abi.FA_ERRWORD_FWD, _abi.FA_ERRWORD_BWD_D64, _abi.FA_ERRWORD_BWD_D128) == (1, 3, 4)

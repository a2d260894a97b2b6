"""ctypes view of libfa_b200.so (include/fa_b200.h).  Argument marshalling only.

The library must exist in-tree (``python -m bf16_numerics_b200.build``);
there is no fallback of any kind: a missing or unloadable library raises.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_WORKSPACE = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5

FA_SOFTMAX_STANDARD = 0
FA_SOFTMAX_STABILIZED = 1
FA_SOFTMAX_STABILIZED_MARGIN = 2

FA_KERNEL_FWD = 0
FA_KERNEL_BWD_DELTA = 1
FA_KERNEL_BWD_MAIN = 2
FA_KERNEL_BWD_DQ = 3
FA_NUM_KERNELS = 4

# kernel ids in the device error word (fa_device_error) and for fa_debug_inject_stall
FA_ERRWORD_FWD = 1
FA_ERRWORD_BWD_D64 = 3
FA_ERRWORD_BWD_D128 = 4
KERNEL_NAMES = ("fa_fwd_kernel", "fa_bwd_delta_kernel", "fa_bwd_main_kernel", "fa_bwd_dq_convert_kernel")

# every symbol include/fa_b200.h declares
EXPORTS = ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_bwd_workspace_delta_offset",
           "fa_bwd_workspace_dq_offset", "fa_status_string", "fa_device_error", "fa_timing_enable",
           "fa_timing_read", "fa_bwd_noalloc", "fa_last_error_string", "fa_fwd_o_hp", "fa_bwd_o_hp",
           "fa_debug_set_wait_limit_ns", "fa_debug_inject_stall")


class FaRowStats(ctypes.Structure):
    _fields_ = [("rm", ctypes.c_void_p), ("rs", ctypes.c_void_p), ("m", ctypes.c_void_p),
                ("pbar_max", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bf16_numerics_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ctypes.POINTER(FaRowStats), i, i, i, i, i, i, f, vp]
    lib.fa_fwd.restype = i
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, f, vp]
    lib.fa_bwd.restype = i
    lib.fa_fwd_o_hp.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(FaRowStats), i, i, i, i, i, i, f, vp]
    lib.fa_fwd_o_hp.restype = i
    lib.fa_bwd_o_hp.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, f, vp]
    lib.fa_bwd_o_hp.restype = i
    for name in ("fa_bwd_workspace_bytes", "fa_bwd_workspace_delta_offset", "fa_bwd_workspace_dq_offset"):
        getattr(lib, name).argtypes = [i, i, i, i]
        getattr(lib, name).restype = sz
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_error_string.argtypes = []
    lib.fa_last_error_string.restype = ctypes.c_char_p
    lib.fa_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.fa_device_error.restype = i
    lib.fa_debug_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.fa_debug_set_wait_limit_ns.restype = i
    lib.fa_debug_inject_stall.argtypes = [ctypes.c_uint]
    lib.fa_debug_inject_stall.restype = i
    lib.fa_timing_enable.argtypes = [i]
    lib.fa_timing_enable.restype = i
    lib.fa_timing_read.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    lib.fa_timing_read.restype = i
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().fa_status_string(code).decode()

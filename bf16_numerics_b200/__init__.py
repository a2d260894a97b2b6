"""Stabilised BF16 FlashAttention for B200 (sm_100a): Python binding.

Thin marshalling layer over the C ABI of ``libfa_b200.so`` (include/fa_b200.h).
Every function with an ``fa_`` name maps 1:1 to the C entry point of the same
name; tensors are passed as device pointers, the stream as the CUDA stream
handle.  PyTorch only provides device memory and streams.  There is no CPU or
library fallback: if the CUDA library is missing, importing the entry points
raises.

Method: Qiu & Yao, "Why Low-Precision Transformer Training Fails: An Analysis
on Flash Attention" (arXiv 2510.04212) -- the safe softmax P_bar = exp(S - m)
with the shift m moved off the row maximum when that maximum is tied
(itsolotime.com/archives/23922, "minimal fix").
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi

STANDARD = _abi.FA_SOFTMAX_STANDARD
STABILIZED = _abi.FA_SOFTMAX_STABILIZED
STABILIZED_MARGIN = _abi.FA_SOFTMAX_STABILIZED_MARGIN

__all__ = ["FaError", "STANDARD", "STABILIZED", "STABILIZED_MARGIN", "RowStats", "fa_fwd", "fa_bwd", "fa_fwd_o_hp", "fa_bwd_o_hp", "fa_bwd_workspace_bytes",
           "fa_bwd_workspace_offsets", "fa_status_string", "fa_device_error", "fa_timing_enable",
           "fa_timing_read", "fa_debug_set_wait_limit_ns", "fa_debug_inject_stall", "attention_forward",
           "attention_backward", "library_path"]


class FaError(RuntimeError):
    def __init__(self, code: int, what: str):
        detail = ""
        if code == _abi.FA_ERR_CUDA:
            detail = " [" + _abi.load().fa_last_error_string().decode() + "]"
        super().__init__(f"{what}: {_abi.status_string(code)} (status {code}){detail}")
        self.code = code


def library_path() -> str:
    _abi.load()
    return _abi.LIB_PATH


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_qkv(name, t, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor [B, H, N, d]")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_vec(name, t, shape, dtype=torch.float32):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of shape {tuple(shape)}")


@dataclass
class RowStats:
    rm: torch.Tensor | None = None
    rs: torch.Tensor | None = None
    m: torch.Tensor | None = None
    pbar_max: torch.Tensor | None = None

    @staticmethod
    def empty(B, H, N, device) -> "RowStats":
        return RowStats(torch.empty(B, H, N, device=device, dtype=torch.float32),
                        torch.empty(B, H, N, device=device, dtype=torch.int32),
                        torch.empty(B, H, N, device=device, dtype=torch.float32),
                        torch.empty(B, H, N, device=device, dtype=torch.float32))


def fa_status_string(code: int) -> str:
    return _abi.status_string(code)


def _stats_struct(stats, B, H, N):
    if stats is None:
        return None
    for name in ("rm", "m", "pbar_max"):
        t = getattr(stats, name)
        if t is not None:
            _check_vec(f"stats.{name}", t, (B, H, N))
    if stats.rs is not None:
        _check_vec("stats.rs", stats.rs, (B, H, N), torch.int32)
    return _abi.FaRowStats(*(None if getattr(stats, n) is None else getattr(stats, n).data_ptr()
                             for n in ("rm", "rs", "m", "pbar_max")))


def fa_fwd(q, k, v, o, lse, stats: RowStats | None = None, causal: bool = True, softmax_mode: int = STABILIZED,
           beta: float = 2.0, stream=None) -> None:
    """C ``fa_fwd``: writes o (bf16) and lse (fp32 [B,H,N]) and, if given, the row stats."""
    lib = _abi.load()
    _check_qkv("q", q)
    B, H, N, d = q.shape
    for name, t in (("k", k), ("v", v), ("o", o)):
        _check_qkv(name, t, q.shape)
    _check_vec("lse", lse, (B, H, N))
    st = _stats_struct(stats, B, H, N)
    code = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(st) if st is not None else None,
                      B, H, N, d, int(bool(causal)), int(softmax_mode), float(beta), _stream_handle(stream))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_fwd")


def fa_fwd_o_hp(q, k, v, o, o_hp, lse, stats: RowStats | None = None, causal: bool = True,
                softmax_mode: int = STABILIZED, beta: float = 2.0, stream=None) -> None:
    """C ``fa_fwd_o_hp``: fa_fwd plus the fp32 O before rounding (o_hp, fp32 [B,H,N,d])."""
    lib = _abi.load()
    _check_qkv("q", q)
    B, H, N, d = q.shape
    for name, t in (("k", k), ("v", v), ("o", o)):
        _check_qkv(name, t, q.shape)
    _check_vec("o_hp", o_hp, (B, H, N, d))
    _check_vec("lse", lse, (B, H, N))
    st = _stats_struct(stats, B, H, N)
    code = lib.fa_fwd_o_hp(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o_hp), _ptr(lse),
                           ctypes.byref(st) if st is not None else None, B, H, N, d, int(bool(causal)),
                           int(softmax_mode), float(beta), _stream_handle(stream))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_fwd_o_hp")


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(_abi.load().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd_workspace_offsets(B: int, H: int, N: int, d: int) -> tuple[int, int]:
    lib = _abi.load()
    return int(lib.fa_bwd_workspace_delta_offset(B, H, N, d)), int(lib.fa_bwd_workspace_dq_offset(B, H, N, d))


def _bwd_checks(q, k, v, dO, lse, row_m, dq, dk, dv, workspace):
    _check_qkv("q", q)
    B, H, N, d = q.shape
    for name, t in (("k", k), ("v", v), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check_qkv(name, t, q.shape)
    _check_vec("lse", lse, (B, H, N))
    if row_m is not None:
        _check_vec("row_m", row_m, (B, H, N))
    if workspace.dtype != torch.uint8 or not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    return B, H, N, d


def fa_bwd(q, k, v, o, dO, lse, row_m, dq, dk, dv, workspace, causal: bool = True, softmax_mode: int = STABILIZED,
           beta: float = 2.0, stream=None) -> None:
    """C ``fa_bwd``: writes dq, dk, dv (bf16); workspace is a uint8 CUDA tensor."""
    lib = _abi.load()
    B, H, N, d = _bwd_checks(q, k, v, dO, lse, row_m, dq, dk, dv, workspace)
    _check_qkv("o", o, q.shape)
    code = lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(row_m), _ptr(dq), _ptr(dk),
                      _ptr(dv), _ptr(workspace), workspace.numel(), B, H, N, d, int(bool(causal)),
                      int(softmax_mode), float(beta), _stream_handle(stream))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_bwd")


def fa_bwd_o_hp(q, k, v, o_hp, dO, lse, row_m, dq, dk, dv, workspace, causal: bool = True,
                softmax_mode: int = STABILIZED, beta: float = 2.0, stream=None) -> None:
    """C ``fa_bwd_o_hp``: fa_bwd with delta taken from the fp32 O (o_hp, fp32 [B,H,N,d])."""
    lib = _abi.load()
    B, H, N, d = _bwd_checks(q, k, v, dO, lse, row_m, dq, dk, dv, workspace)
    _check_vec("o_hp", o_hp, (B, H, N, d))
    code = lib.fa_bwd_o_hp(_ptr(q), _ptr(k), _ptr(v), _ptr(o_hp), _ptr(dO), _ptr(lse), _ptr(row_m), _ptr(dq),
                           _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(), B, H, N, d, int(bool(causal)),
                           int(softmax_mode), float(beta), _stream_handle(stream))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_bwd_o_hp")


def fa_device_error() -> tuple[int, int]:
    """(status, raw device error word); synchronises the device."""
    word = ctypes.c_uint(0)
    code = _abi.load().fa_device_error(ctypes.byref(word))
    return int(code), int(word.value)


def fa_debug_set_wait_limit_ns(ns: int) -> None:
    """C ``fa_debug_set_wait_limit_ns`` (test hook): limit of every bounded wait; 0 restores 2 s."""
    code = _abi.load().fa_debug_set_wait_limit_ns(int(ns))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_debug_set_wait_limit_ns")


def fa_debug_inject_stall(kernel_id: int) -> None:
    """C ``fa_debug_inject_stall`` (test hook): CTA 0 of that kernel withholds its first P arrive; 0 = off."""
    code = _abi.load().fa_debug_inject_stall(int(kernel_id))
    if code != _abi.FA_OK:
        raise FaError(code, "fa_debug_inject_stall")


def fa_timing_enable(enable: bool = True) -> None:
    _abi.load().fa_timing_enable(int(bool(enable)))


def fa_timing_read() -> dict:
    """{kernel name: (launches, total ms)} since the last read."""
    n = _abi.FA_NUM_KERNELS
    launches = (ctypes.c_int * n)()
    total = (ctypes.c_double * n)()
    code = _abi.load().fa_timing_read(launches, total)
    if code != _abi.FA_OK:
        raise FaError(code, "fa_timing_read")
    return {_abi.KERNEL_NAMES[i]: (int(launches[i]), float(total[i])) for i in range(n)}


# ---------------------------------------------------------------- convenience

def attention_forward(q, k, v, causal: bool = True, softmax_mode: int = STABILIZED, beta: float = 2.0,
                      with_stats: bool = True, stream=None):
    """Allocate outputs (torch) and run fa_fwd.  Returns (o, lse, stats)."""
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32)
    stats = RowStats.empty(B, H, N, q.device) if with_stats else None
    fa_fwd(q, k, v, o, lse, stats, causal, softmax_mode, beta, stream)
    return o, lse, stats


def attention_backward(q, k, v, o, dO, lse, row_m, causal: bool = True, softmax_mode: int = STABILIZED,
                       beta: float = 2.0, workspace=None, stream=None):
    """Allocate gradients (torch) and run fa_bwd.  Returns (dq, dk, dv, workspace)."""
    B, H, N, d = q.shape
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_bytes(B, H, N, d), device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa_bwd(q, k, v, o, dO, lse, row_m, dq, dk, dv, workspace, causal, softmax_mode, beta, stream)
    return dq, dk, dv, workspace

"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
on a workload, run the oracle on the same inputs (all heads or a sample), and
compare with the tolerances the tests state.

Tolerances (floating point): for O, dQ, dK, dV
    max |gpu - ref| <= 1e-2 * max |ref| + 1e-5   and   ||gpu - ref||_F <= 5e-3 * ||ref||_F
(the 1e-5 absolute term only matters where the exact result is zero, e.g. dQ
of a row that sees a single key); lse: |gpu - ref| <= 1e-3.  The reference is
the float64 oracle; only where a row's dQ is a cancellation of BF16-rounded
dS terms (two bitwise-equal keys sharing most of the softmax mass) are dQ and
dK held to the same bar against the oracle with the BF16 dS operand modelled
(``ds_bf16``): there no product of BF16 dS can meet the float64 bar.

The backward is an operation on (Q, K, V, O, dO, lse): its delta is
rowsum(dO o O) of the O it is given.  The backward reference is therefore the
oracle's backward evaluated on the O the GPU forward produced (bf16); the
oracle's own float64 O gives the chained reference, whose difference from the
given-O reference is the delta bias the pages describe (a bf16-rounded O
entering delta), reported separately.  Integer / selection outputs (rm, rs, m) are compared
bit for bit where S is exact in fp32 (inputs on a dyadic grid with d = 64);
elsewhere rs and the branch of the shift rule must match and rm agrees to
fp32 accumulation-order rounding.
"""

from __future__ import annotations

import numpy as np
import torch

import bf16_numerics_b200 as fa
from oracle import attention as A

MAXABS = 1e-2
ATOL = 1e-5
FROB = 5e-3
LSE_ABS = 1e-3


def to_dev(x: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(dev)


def run_gpu(w, mode: int, beta: float = 2.0, dev="cuda:0", bwd: bool = True):
    q, k, v, do = (to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    o, lse, st = fa.attention_forward(q, k, v, w.causal, mode, beta)
    out = {"o": o, "lse": lse, "rm": st.rm, "rs": st.rs, "m": st.m, "pbar_max": st.pbar_max}
    if bwd:
        dq, dk, dv, ws = fa.attention_backward(q, k, v, o, do, lse, st.m, w.causal, mode, beta)
        off_delta, _ = fa.fa_bwd_workspace_offsets(*q.shape)
        B, H, N, _ = q.shape
        delta = ws[off_delta:off_delta + B * H * N * 4].view(torch.float32).view(B, H, N)
        out.update(dq=dq, dk=dk, dv=dv, delta=delta)
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    return {k_: v_.float().cpu().numpy() if v_.dtype != torch.int32 else v_.cpu().numpy() for k_, v_ in out.items()}


def run_gpu_o_hp(w, mode: int, beta: float = 2.0, dev="cuda:0"):
    """Forward with the fp32 O (fa_fwd_o_hp), backward with delta from it
    (fa_bwd_o_hp)."""
    q, k, v, do = (to_dev(x, dev) for x in (w.q, w.k, w.v, w.do))
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    o_hp = torch.empty(B, H, N, d, device=dev, dtype=torch.float32)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    st = fa.RowStats.empty(B, H, N, dev)
    fa.fa_fwd_o_hp(q, k, v, o, o_hp, lse, st, w.causal, mode, beta)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), device=dev, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa.fa_bwd_o_hp(q, k, v, o_hp, do, lse, st.m, dq, dk, dv, ws, w.causal, mode, beta)
    off_delta, _ = fa.fa_bwd_workspace_offsets(B, H, N, d)
    delta = ws[off_delta:off_delta + B * H * N * 4].view(torch.float32).view(B, H, N)
    out = {"o": o, "o_hp": o_hp, "lse": lse, "m": st.m, "dq": dq, "dk": dk, "dv": dv, "delta": delta}
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"
    res = {k_: v_.float().cpu().numpy() for k_, v_ in out.items()}
    res["o_bits"] = o.view(torch.int16).cpu().numpy()
    return res


def head_slice(x, pairs):
    return np.stack([x[b, h] for b, h in pairs])[None]


def oracle(w, mode, beta=2.0, pairs=None, o_gpu=None, ds_bf16=False):
    """Oracle outputs for workload w (or the (b, h) pairs given).  With o_gpu
    the backward keys are the given-O reference (delta from o_gpu) and the
    chained ones carry a "_chained" suffix; with ds_bf16 also "dq_r3" and
    "dk_r3": the given-O reference with the BF16 dS operand modelled."""
    if pairs is not None:
        w = w.heads(pairs)
    f = A.attention_fwd(w.q, w.k, w.v, w.causal, mode, beta)
    chained = A.attention_bwd(w.q, w.k, w.v, w.do, w.causal, mode, beta, fwd=f)
    res = dict(f)
    if o_gpu is None:
        res.update(chained)
    else:
        given = A.attention_bwd(w.q, w.k, w.v, w.do, w.causal, mode, beta, fwd=f, o_for_delta=o_gpu)
        res.update(given)
        res["delta_from_gpu_o"] = given["delta"]
        for key in ("dq", "dk", "dv", "delta"):
            res[key + "_chained"] = chained[key]
    if ds_bf16:
        r3 = A.attention_bwd(w.q, w.k, w.v, w.do, w.causal, mode, beta, fwd=f, o_for_delta=o_gpu, ds_bf16=True)
        res["dq_r3"], res["dk_r3"] = r3["dq"], r3["dk"]
    return res


def rel_errors(got, ref):
    """(max |got - ref| / max |ref|, ||got - ref||_F / ||ref||_F)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return (float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)),
            float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)))


def assert_close(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    scale = np.abs(ref).max()
    maxerr = np.abs(got - ref).max()
    assert maxerr <= MAXABS * scale + ATOL, f"{name}: max abs err {maxerr:.3e} > {MAXABS} * {scale:.3e} + {ATOL}"
    nref = np.linalg.norm(ref)
    frob = np.linalg.norm(got - ref) / nref if nref > 0 else 0.0
    if nref > ATOL * np.sqrt(ref.size):
        assert frob <= FROB, f"{name}: relative Frobenius err {frob:.3e} > {FROB}"
    return maxerr / max(scale, 1e-30), frob


def compare(gpu, ref, exact_stats: bool, pairs=None, bf16_ds_keys=()):
    """gpu: dict of full-size arrays; ref: oracle on `pairs` (or all heads).
    Keys listed in bf16_ds_keys ("dq", "dk") are held to the bar against the
    reference with the BF16 dS operand modelled (oracle(..., ds_bf16=True));
    their error against the float64 reference is returned as "<key>_exact"."""
    sel = (lambda x: head_slice(x, pairs)) if pairs is not None else (lambda x: x)
    errs = {}
    for key in ("o", "dq", "dk", "dv"):
        if key in gpu:
            if key in bf16_ds_keys:
                errs[key] = assert_close(key, sel(gpu[key]), ref[key + "_r3"])
                errs[key + "_exact"] = rel_errors(sel(gpu[key]), ref[key])
            else:
                errs[key] = assert_close(key, sel(gpu[key]), ref[key])
    lse_err = np.abs(sel(gpu["lse"]) - ref["lse"]).max()
    assert lse_err <= LSE_ABS, f"lse: max abs err {lse_err:.3e}"
    if "delta" in gpu and "delta_from_gpu_o" in ref:
        d_ref = ref["delta_from_gpu_o"]
        d_err = np.abs(sel(gpu["delta"]) - d_ref).max()
        assert d_err <= 1e-4 * max(np.abs(d_ref).max(), 1.0), f"delta: max abs err {d_err:.3e}"
    rs_g, rs_r = sel(gpu["rs"]), ref["rs"]
    if exact_stats:
        assert np.array_equal(sel(gpu["rm"]), ref["rm"]), "rm not bit-exact"
        assert np.array_equal(rs_g, rs_r), "rs not bit-exact"
        assert np.array_equal(sel(gpu["m"]), ref["m"]), "m not bit-exact"
    else:
        assert np.array_equal(rs_g, rs_r), "rs differs"
        rm_g, rm_r = sel(gpu["rm"]), ref["rm"]
        np.testing.assert_allclose(rm_g, rm_r, rtol=1e-5, atol=1e-5)
        branch = lambda rm, rs: np.where(rs > 1, np.sign(rm), 2)
        assert np.array_equal(branch(rm_g, rs_g), branch(rm_r, rs_r)), "shift-rule branch differs"
        np.testing.assert_allclose(sel(gpu["m"]), ref["m"], rtol=1e-5, atol=1e-5)
    return errs

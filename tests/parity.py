"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
on a workload, run the oracle on the same inputs (all heads or a sample), and
compare with the tolerances the tests state.

Tolerances (floating point): for O, dQ, dK, dV
    max |gpu - ref| <= 1e-2 * max |ref| + 1e-5   and   ||gpu - ref||_F <= 5e-3 * ||ref||_F
(the 1e-5 absolute term only matters where the exact result is zero, e.g. dQ
of a row that sees a single key); lse: |gpu - ref| <= 1e-3.

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


def oracle(w, mode, beta=2.0, pairs=None, o_gpu=None):
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
    return res


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


def bf16_ds_dq_floor(w, ref, o_gpu):
    """max|dQ_emul - dQ_ref| / max|dQ_ref| where dQ_emul = bf16(dS) K * scale,
    with P, dP and delta taken from float64/fp32 arithmetic (delta from the
    given bf16 O) and only dS rounded to bf16: the part of the dQ error that
    comes from the operand precision of the dQ product alone."""
    from oracle import bf16

    B, H, N, d = w.q.shape
    sc = 1.0 / np.sqrt(d)
    num = 0.0
    for b in range(B):
        for h in range(H):
            q, k, v, do = (x[b, h].astype(np.float64) for x in (w.q, w.k, w.v, w.do))
            s = q @ k.T * sc
            if w.causal:
                s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
            p = np.exp(s - ref["lse"][b, h][:, None])
            dlt = (do * np.asarray(o_gpu, np.float64)[b, h]).sum(1)
            ds = p * (do @ v.T - dlt[:, None])
            dq = bf16.round_bf16(ds.astype(np.float32)).astype(np.float64) @ k * sc
            num = max(num, np.abs(dq - ref["dq"][b, h]).max())
    return num / np.abs(ref["dq"]).max()


def compare(gpu, ref, exact_stats: bool, pairs=None):
    """gpu: dict of full-size arrays; ref: oracle on `pairs` (or all heads)."""
    sel = (lambda x: head_slice(x, pairs)) if pairs is not None else (lambda x: x)
    errs = {}
    for key in ("o", "dq", "dk", "dv"):
        if key in gpu:
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

"""Plain float64 attention forward/backward with the stabilised shift rule.

TEST INFRASTRUCTURE ONLY (see the package docstring).  NumPy only; every step
is the definition written out, one (batch, head) at a time, with a library
matmul as the only building block.  No tiling, no online softmax, no fusion.

Notation follows the pages (Qiu & Yao, arXiv 2510.04212, as summarised on
itsolotime.com/archives/23922, "mechanism two" and "minimal fix"):

  S     = Q K^T * scale                     (scale = 1/sqrt(d))
  rm    = rowmax(S)                         ("minimal fix" pseudocode)
  rs    = rowsum(S == rm)                   (number of times the max occurs)
  m     = beta*rm  if rs > 1 and rm > 0     (beta > 1)
          0        if rs > 1 and rm < 0
          rm       otherwise                (standard safe softmax: m = rm)
  P_bar = exp(S - m)                        ("mechanism two", safe softmax)
  P     = P_bar / rowsum(P_bar)
  O     = P V
  lse   = m + ln(rowsum(P_bar))

Backward (page 2, section 3 for delta; the rest is the standard attention
gradient, which the pages take as given):

  delta = rowsum(dO o O)
  dV = P^T dO,  dP = dO V^T,  dS = P o (dP - delta),
  dQ = dS K * scale,  dK = dS^T Q * scale

Readings where the pages are silent (each listed in the design notes):

* rm == 0 with a tied maximum: the pseudocode's ``else`` would give m = 0 and
  exact ones in P_bar, against the stated goal max(P_bar) < 1.  Here
  m = beta - 1 (the rm > 0 rule with |rm| replaced by 1).
* rm, rs and m are taken on the binary32 scores the GPU holds:
  S32 = fp32(fp32(Q K^T) * fp32(scale)); the comparisons S == rm and the
  products beta*rm are binary32 operations.  Every other quantity is float64,
  with S = (Q K^T) * scale in float64.  Where Q K^T is exact in binary32 and
  scale is a power of two (d = 64) the two coincide.
* The backward's softmax recompute follows the mode switch: mode 0 uses
  P = exp(S - lse); modes 1 and 2 rebuild P_bar = exp(S - m) and
  P = P_bar * (1/l) with l = exp(lse - m).  All equal softmax(S) in exact
  arithmetic.
* Mode 2 (margin variant, the pages' fix carried to the bf16 operand): the
  rule keeps max(P_bar) < 1 in fp32, but bf16(P_bar) still rounds to 1.0
  when m - rm < 2^-9.  Mode 2 takes mode 1's m and, on tied rows where
  m - rm < 2^-8 (binary32 subtraction), uses m = rm + 2^-8 (binary32 add)
  instead, so exp(rm - m) <= exp(-2^-8) < 1 - 2^-9 and its bf16 value is
  below 1 as well.
* Causal masking: key j is visible to query i iff j <= i (equal lengths).
"""

from __future__ import annotations

import numpy as np

from .bf16 import round_bf16

STANDARD = 0
STABILIZED = 1
STABILIZED_MARGIN = 2
MARGIN = np.float32(2.0 ** -8)  # mode 2: minimum m - rm on tied rows


def scale_f64(d: int) -> float:
    return 1.0 / np.sqrt(float(d))


def scale_f32(d: int) -> np.float32:
    return np.float32(1.0 / np.sqrt(float(d)))


def select_shift(rm, rs, beta: float, mode: int = STABILIZED) -> np.ndarray:
    """Row shift m from the row max rm and tie count rs ("minimal fix" rule).

    Evaluated in binary32 (beta*rm is a binary32 product).  Mode 0 returns rm;
    mode 2 applies the margin of the module docstring on top of mode 1.
    """
    rm = np.asarray(rm, dtype=np.float32)
    rs = np.asarray(rs)
    if mode == STANDARD:
        return rm.copy()
    b = np.float32(beta)
    tied = rs > 1
    pos = (b * rm).astype(np.float32)
    zero_case = np.float32(b - np.float32(1.0))
    m = np.where(tied & (rm > 0), pos,
                 np.where(tied & (rm < 0), np.float32(0.0),
                          np.where(tied & (rm == 0), zero_case, rm))).astype(np.float32)
    if mode == STABILIZED_MARGIN:
        gap = (m - rm).astype(np.float32)
        m = np.where(tied & (gap < MARGIN), (rm + MARGIN).astype(np.float32), m).astype(np.float32)
    return m


def _mask(n: int, causal: bool) -> np.ndarray:
    """Boolean [n, n]: True where key j is visible to query i."""
    if not causal:
        return np.ones((n, n), dtype=bool)
    return np.tril(np.ones((n, n), dtype=bool))


def _head_scores(q: np.ndarray, k: np.ndarray, causal: bool):
    """(S64, S32) for one head; masked entries are -inf in both."""
    d = q.shape[-1]
    qk = q.astype(np.float64) @ k.astype(np.float64).T
    s64 = qk * scale_f64(d)
    s32 = (qk.astype(np.float32) * scale_f32(d)).astype(np.float32)
    vis = _mask(q.shape[0], causal)
    s64 = np.where(vis, s64, -np.inf)
    s32 = np.where(vis, s32, np.float32(-np.inf)).astype(np.float32)
    return s64, s32


def row_stats(s32: np.ndarray, mode: int, beta: float):
    """rm, rs, m (binary32) for each row of binary32 scores."""
    rm = s32.max(axis=-1).astype(np.float32)
    rs = (s32 == rm[..., None]).sum(axis=-1).astype(np.int32)
    m = select_shift(rm, rs, beta, mode)
    return rm, rs, m


def _split_heads(x: np.ndarray):
    x = np.asarray(x)
    if x.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    return x


def attention_fwd(q, k, v, causal: bool = True, mode: int = STABILIZED, beta: float = 2.0,
                  return_pbar: bool = False) -> dict:
    """Forward pass on [B, H, N, d] inputs (values already BF16-representable).

    Returns float64 ``o`` [B,H,N,d] and ``lse`` [B,H,N]; binary32 ``rm``,
    ``m`` and int32 ``rs`` [B,H,N]; float64 ``pbar_max`` = exp(rm - m); and,
    if asked, the float64 ``pbar`` [B,H,N,N].
    """
    q, k, v = _split_heads(q), _split_heads(k), _split_heads(v)
    B, H, N, d = q.shape
    o = np.zeros((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    rm = np.zeros((B, H, N), dtype=np.float32)
    rs = np.zeros((B, H, N), dtype=np.int32)
    m = np.zeros((B, H, N), dtype=np.float32)
    pbar_all = np.zeros((B, H, N, N), dtype=np.float64) if return_pbar else None
    for b in range(B):
        for h in range(H):
            s64, s32 = _head_scores(q[b, h], k[b, h], causal)
            rm_h, rs_h, m_h = row_stats(s32, mode, beta)
            pbar = np.exp(s64 - m_h.astype(np.float64)[:, None])  # exp(-inf) = 0
            l = pbar.sum(axis=-1)
            p = pbar / l[:, None]
            o[b, h] = p @ v[b, h].astype(np.float64)
            lse[b, h] = m_h.astype(np.float64) + np.log(l)
            rm[b, h], rs[b, h], m[b, h] = rm_h, rs_h, m_h
            if return_pbar:
                pbar_all[b, h] = pbar
    out = {"o": o, "lse": lse, "rm": rm, "rs": rs, "m": m,
           "pbar_max": np.exp(rm.astype(np.float64) - m.astype(np.float64))}
    if return_pbar:
        out["pbar"] = pbar_all
    return out


def attention_bwd(q, k, v, do, causal: bool = True, mode: int = STABILIZED, beta: float = 2.0,
                  fwd: dict | None = None, o_for_delta=None, ds_bf16: bool = False) -> dict:
    """Backward pass: float64 dq, dk, dv [B,H,N,d] and delta [B,H,N].

    ``fwd`` is this module's forward result (recomputed if None).  delta uses
    the oracle's own O unless ``o_for_delta`` (e.g. a BF16 O from elsewhere)
    is given.  ``ds_bf16`` models the BF16 operand of the dQ and dK products
    (the pages' training runs in BF16, page 1 "mechanism two"): dS is rounded
    to the nearest BF16 value (through binary32, RNE, by the emulator in
    oracle.bf16) before dQ = dS K * scale and dK = dS^T Q * scale; every other
    step stays float64.
    """
    q, k, v, do = (_split_heads(x) for x in (q, k, v, do))
    if fwd is None:
        fwd = attention_fwd(q, k, v, causal, mode, beta)
    B, H, N, d = q.shape
    o_delta = fwd["o"] if o_for_delta is None else np.asarray(o_for_delta, dtype=np.float64)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    delta = np.zeros((B, H, N), dtype=np.float64)
    sc = scale_f64(d)
    for b in range(B):
        for h in range(H):
            s64, _ = _head_scores(q[b, h], k[b, h], causal)
            lse = fwd["lse"][b, h]
            if mode == STANDARD:
                p = np.exp(s64 - lse[:, None])
            else:
                m = fwd["m"][b, h].astype(np.float64)
                inv_l = 1.0 / np.exp(lse - m)
                p = np.exp(s64 - m[:, None]) * inv_l[:, None]
            dob = do[b, h].astype(np.float64)
            dlt = (dob * o_delta[b, h]).sum(axis=-1)
            dv[b, h] = p.T @ dob
            dp = dob @ v[b, h].astype(np.float64).T
            ds = p * (dp - dlt[:, None])
            if ds_bf16:
                ds = round_bf16(ds.astype(np.float32)).astype(np.float64)
            dq[b, h] = ds @ k[b, h].astype(np.float64) * sc
            dk[b, h] = ds.T @ q[b, h].astype(np.float64) * sc
            delta[b, h] = dlt
    return {"dq": dq, "dk": dk, "dv": dv, "delta": delta}

"""Seeded synthetic inputs for the attention path (shared by tests and bench).

This module holds no step of the method: it only draws random tensors with the
shapes and value structure of the pages' workloads (GPT-2 small/medium
attention on OpenWebText in Qiu & Yao, arXiv 2510.04212 -- itsolotime.com
archives/23922, "core finding": 12 layers, 12 heads, hidden 768, context
1024).  The dataset is not available here, so seeded Gaussian/quantised
tensors of the same attention shapes stand in for it.

Every tensor is returned as float32 holding exactly BF16-representable values
(drawn in float32, then converted by torch's own float->bfloat16 cast), so that
the CUDA path and the oracle see identical inputs.

Input structure that the pages motivate:
* tied row maxima ("trigger condition" on page 1: several identical maxima in
  one row of S) -- forced by duplicating key 0 at a second position (the
  attention-sink pattern of page 1, "core insight") or, in ``tiestress``, by a
  quantised construction that fixes the sign class of the tied maximum;
* value / upstream-gradient columns with a negative mean (page 1, "source of
  the bias": V[:, i] mostly negative, dO negative in the same dimensions).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = ["Workload", "CONFIGS", "make", "to_bf16_values"]


@dataclass
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    do: np.ndarray
    forced_tie_rows: np.ndarray  # bool [B, H, N]: rows built to hold a tied maximum
    notes: dict = field(default_factory=dict)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def flops_fwd(self) -> float:
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def flops_total(self) -> float:
        return 3.5 * self.flops_fwd()

    def heads(self, pairs):
        """Copy of this workload restricted to the (b, h) pairs given."""
        idx_b = [p[0] for p in pairs]
        idx_h = [p[1] for p in pairs]

        def sl(x):
            return np.ascontiguousarray(x[idx_b, idx_h][None])

        return Workload(self.name + "[heads]", 1, len(pairs), self.N, self.d, self.causal, self.seed,
                        sl(self.q), sl(self.k), sl(self.v), sl(self.do), sl(self.forced_tie_rows),
                        dict(self.notes))


# name -> (B, H, N, d, causal, seed)
CONFIGS = {
    "tiny": (1, 2, 128, 64, True, 0),
    "g2s": (8, 12, 1024, 64, True, 1),
    "g2m": (8, 16, 1024, 64, True, 2),
    "long": (2, 16, 8192, 128, True, 3),
    "tiestress": (4, 12, 4096, 64, False, 4),
}

DESCRIPTIONS = {
    "tiny": "B1 H2 N128 d64 causal; Q,K = 0.125*U{-2..2}; V~N(0,1) cols 0-15 mean -1; dO~N(0,1) cols 0-15 mean -0.5",
    "g2s": "GPT-2 small attention B8 H12 N1024 d64 causal; Q,K,V,dO~N(0,1); key 0 duplicated, 10% of rows tied on it; V cols 0-7 mean -0.75",
    "g2m": "GPT-2 medium attention B8 H16 N1024 d64 causal; Q,K~N(0,1.5^2); V,dO~N(0,1); no forced ties",
    "long": "long context B2 H16 N8192 d128 causal; N(0,1); key 0 duplicated, 5% of rows tied on it",
    "tiestress": "B4 H12 N4096 d64 non-causal; Q,K on the 1/8 grid in [-2,2]; 25% of rows tied (rm>0, rm<0, rm==0 in equal parts); V,dO dims 0-31 mean -0.5",
}


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 array -> float32 array of the nearest BF16 values (torch's cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _normal(rng, shape, std=1.0):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def _sink_ties(rng, q, k, frac):
    """Duplicate key 0 at a position j* and aim a fraction of rows at it.

    For each (b, h): j* is drawn in [1, N/2) so that at least N/2 query rows
    (those t >= j*) see both copies under a causal mask; K[j*] = K[0]; a
    fraction ``frac`` of all N rows, drawn among t >= j*, get Q[t] = 0.5*K[0],
    which makes S[t,0] = S[t,j*] = 0.5*|K[0]|^2*scale the row maximum (well
    above the other keys for Gaussian data).  The two key rows are bitwise
    equal, so their scores are equal in any arithmetic.
    """
    B, H, N, _ = q.shape
    tie = np.zeros((B, H, N), dtype=bool)
    if N < 4:
        return tie
    n_rows = max(1, int(round(frac * N)))
    for b in range(B):
        for h in range(H):
            j_star = int(rng.integers(1, max(2, N // 2)))
            k[b, h, j_star] = k[b, h, 0]
            cand = np.arange(j_star, N)
            rows = rng.choice(cand, size=min(n_rows, cand.size), replace=False)
            q[b, h, rows] = np.float32(0.5) * k[b, h, 0]
            tie[b, h, rows] = True
    return tie


def _tiestress(rng, B, H, N, d):
    """Quantised Q, K with tied maxima of controlled sign.

    Q, K entries are multiples of 1/8 in [-2, 2].  The last head dimension is
    a bias dimension: K[:, d-1] = 2 for every key except a tie pair (j1, j2)
    per (b, h), which both hold k* (ones in 4 random dimensions, zeros
    elsewhere, 0 in the bias dimension).  A tied row t of class a gets
    Q[t, :d-1] = a*k*[:d-1] and Q[t, d-1] = -2, so the tie keys score a*4*scale
    and every other key scores at most (8|a| - 4)*scale < a*4*scale.  With
    d = 64 (scale 1/8): a = 0.25 gives rm = +0.125, a = -0.125 gives
    rm = -0.0625 and a = 0 gives rm = 0, each with rs = 2.
    """
    q = (rng.integers(-16, 17, size=(B, H, N, d)).astype(np.float32) / np.float32(8.0))
    k = (rng.integers(-16, 17, size=(B, H, N, d)).astype(np.float32) / np.float32(8.0))
    k[..., d - 1] = 2.0
    tie = np.zeros((B, H, N), dtype=bool)
    cls = np.full((B, H, N), -1, dtype=np.int8)
    classes = [np.float32(0.25), np.float32(-0.125), np.float32(0.0)]
    n_tied = int(round(0.25 * N))
    for b in range(B):
        for h in range(H):
            j1, j2 = rng.choice(N, size=2, replace=False)
            kstar = np.zeros(d, dtype=np.float32)
            kstar[rng.choice(d - 1, size=4, replace=False)] = 1.0
            k[b, h, j1] = kstar
            k[b, h, j2] = kstar
            rows = rng.choice(N, size=n_tied, replace=False)
            for i, t in enumerate(rows):
                a = classes[i % 3]
                q[b, h, t, : d - 1] = a * kstar[: d - 1]
                q[b, h, t, d - 1] = -2.0
                tie[b, h, t] = True
                cls[b, h, t] = i % 3
    return q, k, tie, cls


def make(name: str, seed: int | None = None, B: int | None = None, H: int | None = None,
         N: int | None = None) -> Workload:
    """Build a named workload; B, H, N and the seed may be overridden (for
    smaller cases of the same construction, e.g. ragged N)."""
    if name not in CONFIGS:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}")
    B0, H0, N0, d, causal, seed0 = CONFIGS[name]
    B = B0 if B is None else B
    H = H0 if H is None else H
    N = N0 if N is None else N
    seed = seed0 if seed is None else seed
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    notes: dict = {"description": DESCRIPTIONS[name]}
    tie = np.zeros((B, H, N), dtype=bool)

    if name == "tiny":
        q = rng.integers(-2, 3, size=shape).astype(np.float32) * np.float32(0.125)
        k = rng.integers(-2, 3, size=shape).astype(np.float32) * np.float32(0.125)
        v = _normal(rng, shape)
        v[..., :16] -= 1.0
        do = _normal(rng, shape)
        do[..., :16] -= 0.5
    elif name in ("g2s", "long"):
        q = to_bf16_values(_normal(rng, shape))
        k = to_bf16_values(_normal(rng, shape))
        v = _normal(rng, shape)
        do = _normal(rng, shape)
        if name == "g2s":
            v[..., :8] -= 0.75
        tie = _sink_ties(rng, q, k, 0.10 if name == "g2s" else 0.05)
    elif name == "g2m":
        q = _normal(rng, shape, 1.5)
        k = _normal(rng, shape, 1.5)
        v = _normal(rng, shape)
        do = _normal(rng, shape)
    elif name == "tiestress":
        q, k, tie, cls = _tiestress(rng, B, H, N, d)
        notes["tie_class"] = cls  # 0: rm>0, 1: rm<0, 2: rm==0, -1: not forced
        v = _normal(rng, shape)
        do = _normal(rng, shape)
        v[..., :32] -= 0.5
        do[..., :32] -= 0.5
    else:  # pragma: no cover
        raise AssertionError(name)

    q, k, v, do = (to_bf16_values(x) for x in (q, k, v, do))
    return Workload(name, B, H, N, d, causal, seed, q, k, v, do, tie, notes)

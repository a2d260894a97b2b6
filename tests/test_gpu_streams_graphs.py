"""The library on several streams and inside a CUDA graph.

Every launch takes its stream from the caller and keeps no per-call state on
the device, so (i) two problems on two streams at once give the same results
as one after the other, and (ii) a forward + backward captured into a CUDA
graph (tensor maps travel by value as kernel parameters) replays to the same
results as the eager calls.  dK, dV, O, lse and the row statistics are
deterministic; dQ sums the partials of several CTAs with reduce-adds in an
order that varies, so it is compared with a tolerance of a few fp32 ulps of
the accumulator (then rounded to bf16).
"""

import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


def _inputs(name, dev, seed=None, **kw):
    w = workloads.make(name, seed=seed, **kw)
    return w, [P.to_dev(x, dev) for x in (w.q, w.k, w.v, w.do)]


def _run(q, k, v, do, causal, stream, out):
    B, H, N, d = q.shape
    with torch.cuda.stream(stream):
        fa.fa_fwd(q, k, v, out["o"], out["lse"], out["st"], causal, 1, 2.0, stream)
        fa.fa_bwd(q, k, v, out["o"], do, out["lse"], out["st"].m, out["dq"], out["dk"], out["dv"], out["ws"], causal,
                  1, 2.0, stream)


def _alloc(q):
    B, H, N, d = q.shape
    dev = q.device
    return {"o": torch.empty_like(q), "lse": torch.empty(B, H, N, device=dev),
            "st": fa.RowStats.empty(B, H, N, dev), "dq": torch.empty_like(q), "dk": torch.empty_like(q),
            "dv": torch.empty_like(q),
            "ws": torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), device=dev, dtype=torch.uint8)}


def _same(a, b, dq_tol=True):
    for key in ("o", "lse", "dk", "dv"):
        assert torch.equal(a[key], b[key]), key
    for key in ("rm", "rs", "m", "pbar_max"):
        assert torch.equal(getattr(a["st"], key), getattr(b["st"], key)), key
    diff = (a["dq"].float() - b["dq"].float()).abs().max().item()
    scale = b["dq"].float().abs().max().item()
    assert diff <= 1e-2 * scale if dq_tol else diff == 0.0


def test_two_streams_match_sequential(cuda_device):
    w1, t1 = _inputs("g2s", cuda_device, seed=21, B=2, H=6)
    w2, t2 = _inputs("g2s", cuda_device, seed=22, B=2, H=6)
    ref1, ref2 = _alloc(t1[0]), _alloc(t2[0])
    s0 = torch.cuda.current_stream(cuda_device)
    _run(*t1, True, s0, ref1)
    _run(*t2, True, s0, ref2)
    torch.cuda.synchronize(cuda_device)
    a, b = _alloc(t1[0]), _alloc(t2[0])
    sa, sb = torch.cuda.Stream(cuda_device), torch.cuda.Stream(cuda_device)
    torch.cuda.synchronize(cuda_device)
    for _ in range(3):
        _run(*t1, True, sa, a)
        _run(*t2, True, sb, b)
    torch.cuda.synchronize(cuda_device)
    assert fa.fa_device_error()[0] == 0
    _same(a, ref1)
    _same(b, ref2)


def test_cuda_graph_replay_matches_eager(cuda_device):
    w, t = _inputs("g2s", cuda_device, seed=23, B=2, H=4)
    eager = _alloc(t[0])
    s0 = torch.cuda.current_stream(cuda_device)
    _run(*t, True, s0, eager)
    torch.cuda.synchronize(cuda_device)
    out = _alloc(t[0])
    side = torch.cuda.Stream(cuda_device)
    side.wait_stream(s0)
    with torch.cuda.stream(side):  # warm-up on the capture stream
        _run(*t, True, side, out)
    s0.wait_stream(side)
    torch.cuda.synchronize(cuda_device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cap = torch.cuda.current_stream(cuda_device)
        _run(*t, True, cap, out)
    for key in ("o", "dq", "dk", "dv"):
        out[key].zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(cuda_device)
    assert fa.fa_device_error()[0] == 0
    _same(out, eager)

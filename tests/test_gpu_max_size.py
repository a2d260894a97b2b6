"""Maximum sizes (GPU): problems past 2^31 elements per tensor, and rows of
64K keys.

Past 2^31 elements.
B*H*N*d is just above 2^31, so in the last heads every element offset into
Q, K, V, O, dO, dQ, dK, dV and the fp32 dQ accumulator passes 2^31 (and every
byte offset of the accumulator passes 2^33).  The library accepts any
B*H*N*d below 2^40; this checks that its kernels' offsets, the delta/clear
and convert kernels' grid-stride loops and the tensor maps hold there.

The heads compared with the oracle sit at the start, on both sides of 2^30
elements (2^31 bytes of a bf16 tensor, 2^32 of the accumulator), on both
sides of 2^31 elements, and at the very end of the buffers.  Their inputs come
from the named workload's construction (seeded, on the host); every other head
holds seeded normal values drawn on the device by torch's generator, which
only fill the problem to its size: a head's outputs depend on its own inputs
alone.  Over the whole problem, properties that hold at any size are checked
on the device: finite outputs, a tie count of at least one on every row, and
the stabilised shift's bound P_bar < 1 on every tied row.

Rows of 64K keys.  A non-causal problem of n = 1024 rows whose Q, K, V and
dO are repeated r = 64 times along the sequence (N = 65536) has, row for row,
the small problem's outputs: each key appears r times, so every softmax
weight is the small problem's divided by r, and the r copies of a key or of a
query collect the same sums (O, dQ, dK and dV are unchanged, lse grows by
ln r, the row maximum is unchanged and its tie count is r times the small
one's, so every row is tied and the shift rule takes its tied branch).  The
oracle runs on the small problem; the GPU runs the whole long one (512 key
tiles per row, 512 query blocks adding into every dQ block).
"""

import dataclasses
import math

import numpy as np
import pytest
import torch

import bf16_numerics_b200 as fa
import workloads
from oracle import attention as A
from tests import parity as P

pytestmark = pytest.mark.gpu

N = 1024
H = 16
MODE = fa.STABILIZED


def _shape(d):
    per_head = N * d
    BH = (1 << 31) // per_head + H  # at least one batch entry past 2^31 elements
    B = -(-BH // H)
    return B, B * H, per_head


def _bytes_needed(B, d):
    E = B * H * N * d
    rows = B * H * N
    return 8 * 2 * E + fa.fa_bwd_workspace_bytes(B, H, N, d) + 5 * 4 * rows


@pytest.mark.parametrize("d,name", [(64, "g2s"), (128, "long")])
def test_problem_past_2_31_elements(cuda_device, d, name):
    dev = cuda_device
    B, BH, per_head = _shape(d)
    assert BH * per_head > (1 << 31)
    free, _ = torch.cuda.mem_get_info(dev)
    need = _bytes_needed(B, d)
    if free < need + (4 << 30):
        pytest.skip(f"needs {need / 2**30:.1f} GiB free, {free / 2**30:.1f} GiB available")

    at = lambda elem: elem // per_head  # the head holding element `elem`
    sample = sorted({0, at(1 << 30) - 1, at(1 << 30), at(1 << 31) - 1, at(1 << 31), BH - 1})
    small = workloads.make(name, seed=11 + d, B=1, H=len(sample), N=N)

    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + d)

    def big(x_small):
        t = torch.randn((B, H, N, d), generator=gen, device=dev, dtype=torch.bfloat16)
        flat = t.view(BH, N, d)
        for j, bh in enumerate(sample):
            flat[bh].copy_(P.to_dev(x_small[0, j], dev))
        return t

    q, k, v, do = big(small.q), big(small.k), big(small.v), big(small.do)
    o, lse, st = fa.attention_forward(q, k, v, small.causal, MODE, 2.0)
    dq, dk, dv, ws = fa.attention_backward(q, k, v, o, do, lse, st.m, small.causal, MODE, 2.0)
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    assert status == 0, f"device error word {word:#x}"

    # properties of every row and element
    for key, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv), ("lse", lse)):
        assert bool(torch.isfinite(t).all()), key
    assert bool((st.rs >= 1).all())
    tied = st.rs > 1
    assert bool((st.pbar_max[tied] < 1.0).all())
    assert bool((st.pbar_max[~tied] == 1.0).all())

    # the sampled heads against the oracle
    off_delta, _ = fa.fa_bwd_workspace_offsets(B, H, N, d)
    delta = ws[off_delta:off_delta + BH * N * 4].view(torch.float32).view(BH, N)
    idx = torch.tensor(sample, device=dev)

    def pick(t, per_row):
        flat = t.reshape(BH, N) if per_row else t.reshape(BH, N, d)
        x = flat.index_select(0, idx)[None]
        return x.cpu().numpy() if x.dtype == torch.int32 else x.float().cpu().numpy()

    gpu = {key: pick(t, False) for key, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv))}
    gpu.update({key: pick(t, True) for key, t in (("lse", lse), ("rm", st.rm), ("rs", st.rs), ("m", st.m),
                                                   ("delta", delta))})
    del q, k, v, do, o, lse, st, dq, dk, dv, ws, delta, tied
    torch.cuda.empty_cache()

    ref = P.oracle(small, MODE, o_gpu=gpu["o"])
    errs = P.compare(gpu, ref, exact_stats=False)
    print(f"d={d} B={B} H={H} heads {sample}:", {key: tuple(round(x, 5) for x in val) for key, val in errs.items()})
    assert np.all(gpu["rs"][small.forced_tie_rows] >= 2)


REPEAT = 64


@pytest.mark.parametrize("d,name,mode", [(64, "tiestress", 0), (64, "tiestress", 1), (128, "long", 1)])
def test_rows_of_64k_keys_by_repetition(cuda_device, d, name, mode):
    small = dataclasses.replace(workloads.make(name, seed=21 + d, B=1, H=1, N=1024), causal=False)
    n, r = small.N, REPEAT
    rep = lambda x: np.ascontiguousarray(np.tile(x, (1, 1, r, 1)))
    big = workloads.Workload(f"{name}x{r}", 1, 1, n * r, d, False, small.seed, rep(small.q), rep(small.k),
                             rep(small.v), rep(small.do), np.tile(small.forced_tie_rows, (1, 1, r)))
    gpu = P.run_gpu(big, mode, dev=cuda_device)
    for key in ("o", "dq", "dk", "dv", "lse"):
        assert np.all(np.isfinite(gpu[key])), key
    assert np.all(gpu["rs"] >= r)
    if mode == 1:
        assert np.all(gpu["pbar_max"] < 1.0)  # every row is tied
    for c in (0, r - 1):  # the first and the last copy of every query and key
        rows = slice(c * n, (c + 1) * n)
        part = {key: val[:, :, rows] for key, val in gpu.items()}
        ref = P.oracle(small, mode, o_gpu=part["o"])
        ref["rs"] = r * ref["rs"]
        ref["lse"] = ref["lse"] + math.log(r)
        ref["m"] = A.select_shift(ref["rm"], ref["rs"], 2.0, mode)
        errs = P.compare(part, ref, exact_stats=(name == "tiestress"))
        print(f"{name} d={d} mode {mode} N={n * r} copy {c}:",
              {key: tuple(round(x, 5) for x in val) for key, val in errs.items()})

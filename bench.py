#!/usr/bin/env python
"""Benchmark: causal attention fwd+bwd TFLOP/s on B200, stabilised softmax.

One step = fa_fwd + fa_bwd (delta, main, dQ convert) on the GPT-2-small
attention workload (B8 H12 N1024 d64, causal, beta = 2), inputs resident in
HBM.  The inputs (50 MB) fit in the 126 MB L2, so L2 is flushed (a 256 MiB
write) before every timed step; the flush is outside the CUDA-event intervals.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload g2s|g2m|long|tiestress|tiny] [--mode 0|1|2]

The default workload (GPT-2-small attention, g2s) is the headline; the other
named workloads are the parity-test shapes and are timed the same way.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own copy of the
workload (independent (batch, head) problems, no collective on the data path:
weak scaling); the timed interval is the max over ranks.  `--impl reference`
times the CPU float64 oracle on a bounded sample of the same workload.

FLOP convention: forward 4*B*H*N^2*d, backward 2.5x forward, halved when
causal; total 7*B*H*N^2*d for causal.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd+bwd TFLOP/s (causal) and % of B200 dense BF16 peak, stabilised mode"
WORKLOAD = "g2s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ("bf16_numerics_b200/csrc/fa_ptx.cuh", "bf16_numerics_b200/csrc/fa_fwd.cuh",
                  "bf16_numerics_b200/csrc/fa_fwd_split.cuh",
                  "bf16_numerics_b200/csrc/fa_bwd.cuh", "bf16_numerics_b200/csrc/fa_bwd_pipe.cuh",
                  "bf16_numerics_b200/csrc/fa_bwd_pipe128.cuh", "bf16_numerics_b200/csrc/fa_lib.cu")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", type=int, default=1, help="0 standard shift, 1 stabilised shift, 2 with margin")
    ap.add_argument("--workload", default=WORKLOAD, help="workload name (workloads.CONFIGS)")
    ap.add_argument("--beta", type=float, default=2.0)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bounded oracle sample (seconds of CPU work)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu
    summary, if it was taken on the current kernel sources (matching source
    hash); else None.  Line format: kernel workload source_hash bytes N."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if (len(parts) >= 5 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload
                    and parts[2] == src):
                return float(parts[4])
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# --------------------------------------------------------------- oracle arm
def cpu_oracle_sample(w, mode, beta, seconds, first=None):
    """Time the float64 oracle fwd+bwd on (batch, head) pairs, in order and
    wrapping around to the first head, until about `seconds` of CPU work;
    returns (flops_done, elapsed, head evaluations, threads).  If `first` is a
    dict, the first head's results (o, dq, dk, dv) are stored in it."""
    from oracle import attention as A
    from threadpoolctl import threadpool_info

    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    per_head = w.flops_total() / len(pairs)
    done, t0 = 0, time.perf_counter()
    while True:
        sub = w.heads([pairs[done % len(pairs)]])
        f = A.attention_fwd(sub.q, sub.k, sub.v, sub.causal, mode, beta)
        g = A.attention_bwd(sub.q, sub.k, sub.v, sub.do, sub.causal, mode, beta, fwd=f)
        if first is not None and done == 0:
            first.update(o=f["o"], dq=g["dq"], dk=g["dk"], dv=g["dv"])
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    elapsed = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return per_head * done, elapsed, done, threads


def parity_readout(ref, gpu):
    """Max-abs error / max|ref| of head (0, 0) for each output: GPU against
    the float64 oracle chained forward -> backward."""
    import numpy as np

    out = {"head": "(b, h) = (0, 0)", "reference": "float64 oracle, its own O in the backward",
           "bar": 1e-2}
    for key in ("o", "dq", "dk", "dv"):
        r = np.asarray(ref[key], dtype=np.float64).reshape(-1)
        g_ = gpu[key][0, 0].float().cpu().numpy().astype(np.float64).reshape(-1)
        out[key] = float(np.abs(g_ - r).max() / max(np.abs(r).max(), 1e-30))
    return out


# ------------------------------------------------------------------ ranks
def rank_seed(rank: int, workload: str = WORKLOAD) -> int:
    """Seed of a rank's copy of the workload: same shapes on every rank (weak
    scaling), independent values."""
    import workloads

    return workloads.CONFIGS[workload][5] + rank


def rank_max(x: float, world: int, device=None) -> float:
    """Max of x over all ranks (x itself on one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


WORKLOAD_TEXT = {
    "g2s": ("GPT-2 small attention", "seeded synthetic N(0,1) Q,K,V,dO; key 0 duplicated, 10% of rows tied on it; "
                                     "V cols 0-7 mean -0.75"),
    "g2m": ("GPT-2 medium attention", "seeded synthetic Q,K ~ N(0,1.5^2), V,dO ~ N(0,1)"),
    "long": ("long-context attention", "seeded synthetic N(0,1); key 0 duplicated, 5% of rows tied on it"),
    "tiestress": ("tie-stress attention", "Q,K on the 1/8 grid, 25% of rows tied (rm > 0, < 0, == 0); "
                                          "V, dO dims 0-31 mean -0.5"),
    "tiny": ("tiny attention", "Q,K on the 1/8 grid; V cols 0-15 mean -1"),
}
MODE_TEXT = {0: "standard", 1: "stabilized", 2: "stabilized_margin"}


def launched_kernel_name(slot: str, d: int) -> str:
    """The name ncu shows for the kernel behind one of the library's timing
    slots (fa_timing_read), so that a bench line and an ncu summary match."""
    if slot == "fa_bwd_main_kernel":
        return "fa_bwd_main_pipe_kernel" if d == 64 else "fa_bwd_main_pipe128_kernel"
    if slot == "fa_fwd_kernel":
        return f"fa_fwd_split_kernel<{d}>" if d == 64 else f"fa_fwd_kernel<{d}>"
    return slot


def kernel_role(name: str) -> str:
    """Which step of the path a launched kernel (as launched_kernel_name
    reports it) performs."""
    if name.startswith("fa_fwd_"):
        return "fwd"
    if name.startswith("fa_bwd_main"):
        return "bwd_main"
    if name == "fa_bwd_delta_kernel":
        return "delta"
    if name == "fa_bwd_dq_convert_kernel":
        return "dq_convert"
    raise ValueError(f"unknown kernel {name}")


def kernel_bound(name: str) -> str:
    """The roofline that bounds a kernel: the forward and the backward main
    kernels are dense contractions; delta and the dQ conversion stream HBM."""
    return "tensor" if kernel_role(name) in ("fwd", "bwd_main") else "hbm"


def workload_config(w, mode, beta):
    what, inputs = WORKLOAD_TEXT.get(w.name, (w.name, "seeded synthetic"))
    return {"workload": f"{w.name}: {what} B{w.B} H{w.H} N{w.N} d{w.d} {'causal' if w.causal else 'non-causal'}, "
                        f"{MODE_TEXT[mode]} shift (beta={beta})",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "softmax_mode": MODE_TEXT[mode], "beta": beta,
            "l2": "flushed before every timed step (256 MiB write, then a 256 MiB read of another buffer; outside the timed intervals)",
            "inputs": inputs, "seed": w.seed}


def run_reference(args, rank, world):
    import workloads

    if rank != 0:
        return 0
    w = workloads.make(args.workload)
    per_step = min(1.0, 120.0 / max(1, args.steps + args.warmup))  # whole run bounded to ~2 min (>= 1 head/step)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, args.mode, args.beta, per_step)
    flops, secs, heads = 0.0, 0.0, 0
    threads = 1
    for _ in range(args.steps):
        f_, s_, h_, threads = cpu_oracle_sample(w, args.mode, args.beta, per_step)
        flops += f_
        secs += s_
        heads += h_
    value = flops / secs / 1e12
    sample = (f"{heads} (b,h) heads of {w.B * w.H} over {args.steps} steps, float64 NumPy oracle fwd+bwd, "
              f"throughput scaled per head")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.mode, args.beta),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import bf16_numerics_b200 as fa
    import workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.make(args.workload, seed=rank_seed(rank, args.workload))
    B, H, N, d = w.B, w.H, w.N, w.d
    mode, beta, causal = args.mode, args.beta, w.causal

    h_in = [torch.from_numpy(x).to(torch.bfloat16).pin_memory() for x in (w.q, w.k, w.v, w.do)]
    q, k, v, do = (t.to(dev) for t in h_in)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    stats = fa.RowStats(m=torch.empty(B, H, N, device=dev, dtype=torch.float32))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), device=dev, dtype=torch.uint8)
    flush = torch.empty(256 * 1024 * 1024, device=dev, dtype=torch.uint8)
    flush_read = torch.zeros(64 * 1024 * 1024, device=dev, dtype=torch.float32)

    def flush_l2():
        # write 256 MiB (evicts the inputs), then read another 256 MiB so the
        # dirty lines of the write are back in HBM before the timed interval
        flush.zero_()
        flush_read.sum()
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fa_fwd(q, k, v, o, lse, stats, causal, mode, beta, stream)
        fa.fa_bwd(q, k, v, o, do, lse, stats.m, dq, dk, dv, ws, causal, mode, beta, stream)

    for _ in range(max(3, args.warmup)):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)
    status, word = fa.fa_device_error()
    if status != 0:
        raise RuntimeError(f"device error word {word:#x} during warm-up")

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x for x in visible.split(",") if x.strip()]
    phys = int(ids[local_rank]) if len(ids) > local_rank and ids[local_rank].strip().isdigit() else local_rank
    sampler = ClockSampler(phys)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.2)
    for i in range(K):
        flush_l2()
        starts[i].record(stream)
        step()
        stops[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, stops)]
    total_ms_max = rank_max(sum(step_ms), world, dev)
    # per-kernel durations: a second timed pass with the library recording
    # CUDA events on the launching stream around each of its launches
    KR = min(K, 200)
    fa.fa_timing_enable(True)
    for i in range(KR):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)
    fa.fa_timing_enable(False)
    per_kernel = {launched_kernel_name(slot, d): v for slot, v in fa.fa_timing_read().items()}
    status, word = fa.fa_device_error()
    if status != 0:
        raise RuntimeError(f"device error word {word:#x} during timing")

    flops_step = w.flops_total()
    value = aggregate_tflops(world, flops_step, K, total_ms_max)

    # -------- end to end through the public API with host buffers
    # Every step copies its inputs from pinned host memory and its results
    # back, inside the timed interval.  Serial: copy in, compute, copy out on
    # one stream.  Pipelined (the reported value), as a training loop with a
    # prefetching loader runs: two device buffer sets alternate, and the inputs
    # of step i+1 go up on one copy stream and the results of step i-1 come
    # down on another while step i computes.
    E = args.e2e_steps
    h_out = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    h2d = sum(x.numel() * x.element_size() for x in h_in)
    d2h = sum(x.numel() * x.element_size() for x in h_out)

    def e2e_step():
        for hs, dt in zip(h_in, (q, k, v, do)):
            dt.copy_(hs, non_blocking=True)
        step()
        for hs, dt in zip(h_out, (o, dq, dk, dv)):
            hs.copy_(dt, non_blocking=True)

    def timed(fn, n, s_begin, s_end):
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_begin)
        fn(n)
        e1.record(s_end)
        torch.cuda.synchronize(dev)
        return rank_max(e0.elapsed_time(e1), world, dev)

    def serial(n):
        for _ in range(n):
            e2e_step()

    serial(3)
    e2e_serial = aggregate_tflops(world, flops_step, E, timed(serial, E, stream, stream))

    bufs = [dict(q=q, k=k, v=v, do=do, o=o, lse=lse, stats=stats, dq=dq, dk=dk, dv=dv, ws=ws),
            dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), do=torch.empty_like(do),
                 o=torch.empty_like(o), lse=torch.empty_like(lse), stats=fa.RowStats(m=torch.empty_like(stats.m)),
                 dq=torch.empty_like(dq), dk=torch.empty_like(dk), dv=torch.empty_like(dv), ws=torch.empty_like(ws))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n):
        for i in range(n):
            bb = bufs[i % 2]
            if i >= 2:
                s_in.wait_event(comp_done[i % 2])  # step i-2 has finished reading these inputs
            for hs, key in zip(h_in, ("q", "k", "v", "do")):
                with torch.cuda.stream(s_in):
                    bb[key].copy_(hs, non_blocking=True)
            in_done[i % 2].record(s_in)
            stream.wait_event(in_done[i % 2])
            if i >= 2:
                stream.wait_event(out_done[i % 2])  # step i-2's results have been copied out
            fa.fa_fwd(bb["q"], bb["k"], bb["v"], bb["o"], bb["lse"], bb["stats"], causal, mode, beta, stream)
            fa.fa_bwd(bb["q"], bb["k"], bb["v"], bb["o"], bb["do"], bb["lse"], bb["stats"].m, bb["dq"], bb["dk"],
                      bb["dv"], bb["ws"], causal, mode, beta, stream)
            comp_done[i % 2].record(stream)
            s_out.wait_event(comp_done[i % 2])
            for hs, key in zip(h_out, ("o", "dq", "dk", "dv")):
                with torch.cuda.stream(s_out):
                    hs.copy_(bb[key], non_blocking=True)
            out_done[i % 2].record(s_out)

    pipelined(3)
    e2e_value = aggregate_tflops(world, flops_step, E, timed(pipelined, E, s_in, s_out))
    status, word = fa.fa_device_error()
    if status != 0:
        raise RuntimeError(f"device error word {word:#x} during the end-to-end steps")

    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    # per-kernel roofline from the library's event records (launching stream)
    fwd_flops = w.flops_fwd()
    bwd_flops = 2.5 * fwd_flops
    rows = B * H * N
    delta_bytes = rows * d * 2 * 2 + rows * 4  # algorithmic: read O, dO; write delta (the dQ clear is overhead)
    dq_bytes = rows * d * 4 + rows * d * 2  # dQ convert: read the fp32 accumulator, write bf16
    kern = {}
    for name, (n_l, ms) in per_kernel.items():
        if n_l == 0:
            continue
        avg_s = ms / n_l * 1e-3
        work = {"fwd": fwd_flops, "bwd_main": bwd_flops, "delta": delta_bytes, "dq_convert": dq_bytes}[kernel_role(name)]
        if kernel_bound(name) == "tensor":
            kern[name] = {"bound": "tensor", "avg_us": avg_s * 1e6, "achieved": work / avg_s / 1e12,
                          "unit": "TFLOP/s", "frac": work / avg_s / 1e12 / peak_tf}
        else:
            kern[name] = {"bound": "hbm", "avg_us": avg_s * 1e6, "achieved": work / avg_s / 1e9,
                          "unit": "GB/s", "frac": work / avg_s / 1e9 / hbm}
        kern[name]["launches"] = n_l
    dominant = max(per_kernel, key=lambda nm: per_kernel[nm][1])
    dk_ = kern[dominant]
    traffic = recorded_traffic(dominant, args.workload)
    roofline = {"kernel": dominant, "bound": dk_["bound"], "achieved": dk_["achieved"],
                "peak": peak_tf if dk_["bound"] == "tensor" else hbm, "unit": dk_["unit"], "frac": dk_["frac"],
                "traffic": traffic, "peak_source": f"{peak_src} ({'bf16_tflops burst' if dk_['bound'] == 'tensor' else 'hbm_gbs'})"}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms_max / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, mode, beta),
            "pct_of_peak": 100.0 * value / (world * peak_tf),
            "pct_of_sustained_peak": 100.0 * value / (world * float(peaks.get("bf16_tflops_sustained", peak_tf))),
            "peak_source": peak_src,
            "roofline": roofline, "kernels": kern,
            "gpu_launches": K * sum(n for n, _ in per_kernel.values()) // KR,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": E, "outputs": "O, dQ, dK, dV copied back to pinned host memory",
                    "pipelining": "two device buffer sets; inputs of step i+1 (H2D) and results of step i-1 "
                                  "(D2H) move on two copy streams while step i computes",
                    "serial_value": e2e_serial},
            "clocks": clocks, "step_ms_p10_p50_p90": [float(np.percentile(step_ms, p)) for p in (10, 50, 90)]}
    if world == 1 and not args.no_cpu_baseline:
        first = {}
        flops_c, secs_c, heads_c, threads_c = cpu_oracle_sample(w, mode, beta, args.cpu_seconds, first)
        line["cpu_baseline"] = {"value": flops_c / secs_c / 1e12, "unit": "TFLOP/s", "cores": threads_c,
                                "kind": "oracle",
                                "sample": f"{heads_c} (b,h)-head fwd+bwd evaluations cycling over the {B * H} heads "
                                          f"of the same workload, float64 NumPy oracle, {secs_c:.1f} s"}
        # the oracle's first head against the GPU's outputs for it (the last
        # timed step's inputs are the workload's, so the outputs are too)
        line["parity"] = parity_readout(first, {"o": o, "dq": dq, "dk": dk, "dv": dv})
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world != 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

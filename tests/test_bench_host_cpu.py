"""Host-side logic of bench.py on the CPU: the per-workload DRAM traffic
record, the clock/throttle-reason parsing, the peaks fallback and the parity
readout."""

import os

import numpy as np

import bench


def test_traffic_record_is_keyed_by_kernel_workload_and_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# kernel workload source_hash unit bytes\n"
        "fa_bwd_main_pipe_kernel g2s abc123 bytes 1000\n"
        "fa_bwd_main_pipe128_kernel long abc123 bytes 5000\n"
        "fa_fwd_kernel<64> g2s oldhash bytes 7\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc123")
    assert bench.recorded_traffic("fa_bwd_main_pipe_kernel", "g2s") == 1000.0
    assert bench.recorded_traffic("fa_bwd_main_pipe128_kernel", "long") == 5000.0
    assert bench.recorded_traffic("fa_bwd_main_pipe_kernel", "tiestress") is None  # no capture for it
    assert bench.recorded_traffic("fa_fwd_kernel<64>", "g2s") is None  # taken on other sources


def test_traffic_record_missing_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("fa_bwd_main_pipe_kernel", "g2s") is None


def test_committed_traffic_lines_parse():
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles", "traffic.txt")
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        kernel, workload, src, unit, value = line.split()
        assert unit == "bytes" and float(value) > 0 and len(src) == 16
        assert workload in ("g2s", "g2m", "tiestress", "long", "tiny")


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.lines = lines
    return s


def test_clock_sampler_reports_median_and_active_reasons():
    lines = [
        "1965, 1965, 450.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 610.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    r = _sampler(lines).stop()
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 3 and r["power_w_max"] == 610.0


def test_clock_sampler_flags_slowdowns():
    lines = ["1200, 1965, 300.0, 0x8, Active, Not Active, Active, Not Active"]
    r = _sampler(lines).stop()
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_sampler_without_samples():
    assert _sampler([]).stop()["reasons"] == ["no samples"]


def test_peaks_fall_back_when_the_file_is_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback"
    assert peaks == bench.FALLBACK_PEAKS


def test_launched_kernel_names_follow_the_head_dimension():
    import bench

    assert bench.launched_kernel_name("fa_bwd_main_kernel", 64) == "fa_bwd_main_pipe_kernel"
    assert bench.launched_kernel_name("fa_bwd_main_kernel", 128) == "fa_bwd_main_pipe128_kernel"
    assert bench.launched_kernel_name("fa_fwd_kernel", 128) == "fa_fwd_kernel<128>"
    assert bench.launched_kernel_name("fa_fwd_kernel", 64) == "fa_fwd_split_kernel<64>"
    assert bench.launched_kernel_name("fa_bwd_delta_kernel", 64) == "fa_bwd_delta_kernel"


def test_every_launched_kernel_has_its_roofline():
    import bench

    for d in (64, 128):
        names = [bench.launched_kernel_name(slot, d) for slot in
                 ("fa_fwd_kernel", "fa_bwd_delta_kernel", "fa_bwd_main_kernel", "fa_bwd_dq_convert_kernel")]
        assert [bench.kernel_bound(n) for n in names] == ["tensor", "hbm", "tensor", "hbm"]
        assert [bench.kernel_role(n) for n in names] == ["fwd", "delta", "bwd_main", "dq_convert"]


def test_parity_readout_is_relative_max_abs_error_of_head_zero():
    """bench.py's parity field: max-abs error / max|ref| of head (0, 0) for O,
    dQ, dK, dV, the GPU side read through float32."""
    import torch

    rng = np.random.default_rng(3)
    ref = {key: rng.standard_normal((1, 1, 16, 8)) for key in ("o", "dq", "dk", "dv")}
    gpu = {key: torch.from_numpy(ref[key]).float() for key in ref}
    same = bench.parity_readout(ref, gpu)
    assert all(same[key] < 1e-6 for key in ("o", "dq", "dk", "dv"))
    assert same["bar"] == 1e-2
    bump = dict(gpu)
    bump["dk"] = gpu["dk"].clone()
    bump["dk"][0, 0, 3, 2] += 0.25 * float(np.abs(ref["dk"]).max())
    assert abs(bench.parity_readout(ref, bump)["dk"] - 0.25) < 1e-6

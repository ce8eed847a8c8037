"""Host-side helpers of bench.py on CPU: the DRAM-traffic record is used only
while every kernel source it lists still has the hash taken at capture time."""
import hashlib

import bench


def _record(tmp_path, files, shas, extra="dram_bytes_per_launch_avg: 123\n"):
    (tmp_path / "profiles").mkdir(exist_ok=True)
    (tmp_path / "profiles" / "r.txt").write_text(
        "# a capture summary\n"
        f"source_files: {', '.join(files)}\n"
        f"source_sha256: {', '.join(shas)}\n" + extra)


def test_traffic_record_current_then_stale(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "a.cuh").write_text("kernel a")
    (tmp_path / "b.cu").write_text("kernel b")
    shas = [hashlib.sha256(b"kernel a").hexdigest(), hashlib.sha256(b"kernel b").hexdigest()]
    _record(tmp_path, ["a.cuh", "b.cu"], shas)
    rec, state = bench.traffic_record("r.txt")
    assert state == "current" and rec["dram_bytes_per_launch_avg"] == "123"
    (tmp_path / "b.cu").write_text("kernel b, edited")
    rec, state = bench.traffic_record("r.txt")
    assert rec is None and state == "stale"


def test_traffic_record_missing_or_malformed(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("absent.txt") == (None, None)
    (tmp_path / "a.cuh").write_text("x")
    _record(tmp_path, ["a.cuh", "b.cu"], [hashlib.sha256(b"x").hexdigest()])  # count mismatch
    assert bench.traffic_record("r.txt") == (None, None)
    _record(tmp_path, ["gone.cuh"], ["0" * 64])  # listed source no longer exists
    assert bench.traffic_record("r.txt") == (None, None)


def test_decode_bytes_match_the_workload_sizes():
    """Packed codes + bf16 scales/biases + x + y, once each: 9.45 MB for
    4096x4096 and 33.07 MB for 14336x4096 at 4 bits, group 64, M = 1."""
    assert bench.decode_bytes(1, 4096, 4096, 4, 64) == 4096 * 4096 // 2 + 4096 * 64 * 4 + 2 * 4096 * 2
    assert round(bench.decode_bytes(1, 4096, 4096, 4, 64) / 1e6, 2) == 9.45
    assert round(bench.decode_bytes(1, 14336, 4096, 4, 64) / 1e6, 2) == 33.07
    # the two 14336-sized shapes move the same bytes (x and y swap sizes)
    assert bench.decode_bytes(1, 14336, 4096, 4, 64) == bench.decode_bytes(1, 4096, 14336, 4, 64)


def test_clock_sampler_decodes_reasons_with_a_fake_nvml(monkeypatch):
    """The sampler reads SM clocks and event-reason bits through NVML; a fake
    NVML module stands in for the GPU.  The fake offers getters only, so a
    call to any setter would raise: in the constructor that leaves the
    sampler disabled, in the sampling loop it drops the samples, and either
    fails an assertion below."""
    import itertools
    import sys
    import time
    import types

    import torch

    seq = itertools.cycle([(1965, 0x4), (1950, 0x0), (1900, 0x8)])
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
        nvmlDeviceGetHandleByPciBusId=lambda b: ("gpu", b),
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: cur[0][0],
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: cur[0][1],
    )
    cur = [next(seq)]

    def advance(*a, **k):
        cur[0] = next(seq)
        return False

    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(), raising=False)
    cs = bench.ClockSampler(0, period_s=0.001)
    assert cs.nv is fake and cs.max_mhz == 1965
    cs._stop.wait = advance  # step through the fake sequence once per sample
    with cs:
        time.sleep(0.05)
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965 and s["samples"] >= 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert 1900 <= s["sm_mhz"] <= 1965


def test_clock_sampler_without_nvml_reports_unavailable(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    cs = bench.ClockSampler(0)
    with cs:
        pass
    assert cs.summary()["reasons"] == ["unavailable"]


def test_gpu_arm_fails_loudly_without_a_gpu():
    """With no GPU the bench's own arm exits non-zero and prints no result
    line: there is no CPU path that could stand in for the kernels."""
    import os
    import subprocess
    import sys

    import pytest
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode != 0
    assert '"metric"' not in r.stdout

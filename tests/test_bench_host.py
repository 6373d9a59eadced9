"""Host logic of bench.py on CPU: the clock sampler's summary from a fake NVML
(read-only queries; throttle bits mapped to the reasons the timing rules name,
the median taken over samples under load) and from an nvidia-smi CSV, and the
recorded-traffic guard that reports null once a GEMM source changes."""
import hashlib
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _FakeNvml(types.SimpleNamespace):
    NVML_CLOCK_SM = 1

    def __init__(self, seq):
        super().__init__()
        self.seq = list(seq)
        self.i = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, u):
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, c):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, c):
        return self.seq[min(self.i, len(self.seq) - 1)][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        v = self.seq[min(self.i, len(self.seq) - 1)][1]
        self.i += 1
        return v


def test_nvml_summary_maps_reason_bits_and_takes_the_loaded_median(monkeypatch, tmp_path):
    fake = _FakeNvml([(1965, 0x0), (1950, 0x4), (210, 0x1), (1965, 0x8), (1965, 0x0)])
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", lambda self: (fake, "h"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    c = bench.ClockSampler(0)
    with c:
        while fake.i < 5:
            pass
    s = c.summary()
    assert s["source"] == "nvml" and s["sm_max_mhz"] == 1965.0 and s["samples"] >= 5
    assert s["sm_mhz"] == 1965.0  # the idle 210 MHz sample is not under load
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]  # 0x8 and 0x4; 0x1 (idle) is not a reason
    assert list(tmp_path.iterdir()) == []  # the samples stay in memory: nothing is written


def test_nvidia_smi_csv_summary(monkeypatch, tmp_path):
    c = bench.ClockSampler(0)
    c.path = str(tmp_path / "clocks.csv")
    with open(c.path, "w") as f:
        f.write("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 1965, 1965, 650.0, 0x0, Not Active, Not Active, Active, Not Active\n")
    c.proc = object()  # as if nvidia-smi had run
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert not os.path.exists(c.path)  # the temporary sample file is removed once read


def test_traffic_is_null_once_a_gemm_source_changes(monkeypatch, tmp_path):
    csrc = tmp_path / "indirect_expert_matmul_b200" / "csrc"
    csrc.mkdir(parents=True)
    digests = {}
    for name in bench.GATE_UP_TRAFFIC["sources_sha256"]:
        (csrc / name).write_bytes(name.encode())
        digests[name] = hashlib.sha256(name.encode()).hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.GATE_UP_TRAFFIC, "sources_sha256", digests)
    assert bench.gate_up_traffic() == bench.GATE_UP_TRAFFIC["bytes_per_launch"]
    (csrc / "gemm.cu").write_bytes(b"changed")
    assert bench.gate_up_traffic() is None


def test_cpu_baseline_survives_batches_with_fewer_experts_than_k(monkeypatch):
    # with 2 host cores a batch holds 2 slots, so fewer than k = 8 distinct experts
    monkeypatch.setattr(bench.os, "sched_getaffinity", lambda pid: {0, 1})
    r = bench.cpu_baseline(budget_s=0.01)
    assert r["value"] > 0 and r["cores"] == 2 and r["kind"] == "oracle"

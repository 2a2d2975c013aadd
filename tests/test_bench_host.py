"""Host-side logic of bench.py (CPU): the algorithmic byte counts the roofline
divides by, the kernel count per pass, the clock record and the rule that
reports committed DRAM traffic only for unchanged GEMV sources."""
import json
import os

import pytest

import bench
from synth import FULL, Q4_0, Q8_0


def test_pass_bytes_of_the_64_layer_stage():
    # packed weights: per layer gate + up [17408 x 5120] and down [5120 x 17408],
    # plus the mixer's in [10336 or 14336 x 5120] and out [5120 x 6144]; Q4_0 = 18 B / 32
    ffn = 3 * 17408 * 5120
    dn = ffn + 10336 * 5120 + 5120 * 6144
    at = ffn + 14336 * 5120 + 5120 * 6144
    assert bench.layer_bytes(FULL, Q4_0, 0) == dn * 18 // 32 == 197_867_520          # 197.9 MB
    assert bench.layer_bytes(FULL, Q4_0, 3) == at * 18 // 32 == 209_387_520          # 209.4 MB
    b = bench.pass_bytes(FULL, Q4_0, range(64), 4096)
    assert b["weights"] == (48 * dn + 16 * at) * 18 // 32 == 12_847_841_280          # 12.848 GB
    assert bench.pass_bytes(FULL, Q8_0, range(64), 4096)["weights"] == (48 * dn + 16 * at) * 34 // 32
    # KV: 16 attention layers read K and V rows 0..4096 (f16, 4 heads x 256)
    assert b["kv"] == 16 * 2 * 4 * 4097 * 256 * 2
    # DeltaNet state: 48 layers, f32 [48][128][128] read once and written once
    assert b["state"] == 48 * 48 * 128 * 128 * 4 * 2
    assert b["total"] == b["weights"] + b["kv"] + b["state"]


def test_launches_per_pass():
    # stage input, then per layer in-proj, mixer (DeltaNet step | attention
    # partials + combine), out-proj, gate/up, down
    assert bench.launches_per_pass(FULL, range(64)) == 1 + 48 * 5 + 16 * 6 == 337
    assert bench.launches_per_pass(FULL, range(0, 4)) == 1 + 3 * 5 + 6
    assert bench.launches_per_pass(FULL, range(64), persistent=True) == 1


class _FakeSmi:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def test_clock_record_median_max_and_reasons():
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi("\n".join([
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]))
    r = s.stop()
    assert r["sm_mhz"] == 1950 and r["sm_max_mhz"] == 1965 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler(0).stop()["reasons"] == ["clock sampling unavailable"]


def test_clock_record_from_nvml_samples():
    s = bench.ClockSampler(0)

    class _Done:
        def set(self):
            pass

    class _Thread:
        def join(self, timeout=None):
            pass

    s.thread, s.stop_ev, s.max_mhz = _Thread(), _Done(), 1965.0
    s.samples = [(1965.0, set()), (1440.0, {"sw_power_cap"}), (1950.0, set()), (1960.0, {"hw_slowdown"})]
    r = s.stop()
    assert r["sm_mhz"] == 1955.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 4
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_traffic_is_reported_only_for_the_sources_it_was_measured_on(monkeypatch):
    p = os.path.join(bench.ROOT, "profiles", "qgemv_dram.json")
    with open(p) as f:
        d = json.load(f)
    if d["sources_sha256"] == bench.kernel_sources_sha():
        assert bench.committed_traffic() == d["traffic_bytes_per_launch"]
    else:                                   # the GEMV changed since the capture: no figure
        assert bench.committed_traffic() is None
    # per launch, within a few percent of the algorithmic bytes (no re-reads)
    assert 1.0 <= d["traffic_bytes_per_launch"] / d["algorithmic_bytes_per_launch"] < 1.05
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: "0" * 64)
    assert bench.committed_traffic() is None

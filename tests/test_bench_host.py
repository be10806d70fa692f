"""bench.py host helpers that need no GPU: the clock-sample filter, the traffic records,
the step timer's event arithmetic and the projection report."""

import datetime
import os
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _line(ts, mhz, cap="Not Active"):
    return (f"{ts.strftime('%Y/%m/%d %H:%M:%S.%f')[:-3]}, 0, {mhz}, 1965, 700.00, 0x0, Not Active, Not Active, "
            f"Not Active, {cap}\n")


def test_clock_summary_keeps_only_the_timed_region():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    c = bench.ClockSampler(0)
    fd, c.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.write(_line(t0 - datetime.timedelta(seconds=1), 600))              # idle, before
        f.write(_line(t0 + datetime.timedelta(milliseconds=200), 1900, "Active"))
        f.write(_line(t0 + datetime.timedelta(milliseconds=400), 1800))
        f.write(_line(t0 + datetime.timedelta(seconds=3), 500))               # idle, after
    c.t0, c.t1 = t0, t0 + datetime.timedelta(milliseconds=500)
    s = c.summary()
    assert s["samples"] == 2 and s["in_timed_region"]
    assert s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_all_samples():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    c = bench.ClockSampler(0)
    fd, c.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.write(_line(t0 - datetime.timedelta(seconds=1), 1700))
    c.t0, c.t1 = t0, t0 + datetime.timedelta(milliseconds=5)
    s = c.summary()
    assert s["samples"] == 1 and not s["in_timed_region"] and s["sm_mhz"] == 1700


def test_profile_traffic_reads_the_record_of_the_current_source():
    from dsa_lightning_indexer_03_b200 import build as B
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    want = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            key, _, rest = line.rpartition(":")
            n, h = rest.split()[:2]
            want[key.strip()] = (float(n), h)
    for key, (n, h) in want.items():
        got = bench._profile_traffic(key)
        assert got == (n if h == B.source_hash() else None), key
    assert bench._profile_traffic("score_topk:no_such_workload") is None


def test_projection_report_counts_both_gemms_and_the_bytes_once():
    r = bench.projection_report(8192, 0.5, 1650.2, 6538.0)
    flops = 2 * 8192 * (1536 * 4096) + 2 * 8192 * (7168 * (128 + 32))
    assert r["flop"] == flops
    per_token = 7168 * 2 + 1536 * 2 + 32 * 128 * 2 + 128 * 2 + 32 * 4   # hidden, q_latent in; q, k, w out
    weights = (1536 * 4096 + 7168 * 160) * 2
    assert r["bytes"] == 8192 * per_token + weights
    assert abs(r["achieved_tflops"] - flops / 0.5e-3 / 1e12) < 0.01
    assert abs(r["frac_tensor"] - r["achieved_tflops"] / 1650.2) < 1e-3
    assert abs(r["achieved_gbs"] - r["bytes"] / 0.5e-3 / 1e9) < 0.01


def test_time_steps_splits_projection_and_topk(monkeypatch):
    """The events fn records split each step into projection and score + top-k."""
    clock = [0.0]

    class FakeEvent:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = clock[0]

        def elapsed_time(self, other):
            return other.t - self.t

    def fn(ev):
        clock[0] += 2.0          # projections
        ev[0].record()
        clock[0] += 5.0          # score + top-k
        ev[1].record()

    monkeypatch.setattr(bench.torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda: None)
    step, topk, proj = bench._time_steps(fn, 3, lambda: None)
    assert step == [7.0] * 3 and topk == [5.0] * 3 and proj == [2.0] * 3

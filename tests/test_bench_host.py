"""bench.py host helpers that need no GPU: the clock-sample filter."""

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

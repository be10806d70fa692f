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
    """The spans fn records split each step into projection and score + top-k time, summed
    over the calls of a step (the chunked prefill makes 16 of each)."""
    clock = [0.0]

    class FakeEvent:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = clock[0]

        def elapsed_time(self, other):
            return other.t - self.t

    def advance(dt):
        def f():
            clock[0] += dt
        return f

    def fn(spans):
        for _ in range(2):
            spans.span("project", advance(2.0))
            clock[0] += 0.5          # work between the spans (counted in the step only)
            spans.span("topk", advance(5.0))

    monkeypatch.setattr(bench.torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda: None)
    step, topk, proj = bench._time_steps(fn, 3, lambda: None)
    assert step == [15.0] * 3 and topk == [10.0] * 3 and proj == [4.0] * 3


def test_prefill_roofline_arithmetic():
    peaks = dict(bf16_tflops=1650.0, bf16_tflops_sustained=1400.0, source="measured")
    r = bench.prefill_roofline(8_590_000_128, 100.0, peaks, None)
    tflops = 8_590_000_128 * 8192 / 0.1 / 1e12
    assert abs(r["achieved"] - tflops) < 0.01
    assert abs(r["frac"] - tflops / 1650.0) < 1e-4      # short timed region: burst peak
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["gpairs_score_topk"] - 85.9) < 0.001
    # a timed region of seconds of back-to-back launches is held to the sustained peak
    r = bench.prefill_roofline(8_590_000_128, 100.0, peaks, None, timed_s=2.0)
    assert r["peak"] == 1400.0 and abs(r["frac"] - tflops / 1400.0) < 1e-4
    assert abs(r["frac_burst"] - tflops / 1650.0) < 1e-4 and "sustained" in r["peak_source"]
    # FP8 operands: the nominal 2x of the bf16 figure
    r = bench.prefill_roofline(8_590_000_128, 100.0, peaks, None, fp8=True, timed_s=0.1)
    assert r["peak"] == 3300.0


def test_headline_is_the_long_context_chunked_prefill():
    import workloads as W
    assert bench.HEADLINE == "chunked_128k"
    cfg = W.WORKLOADS[bench.HEADLINE]
    S = cfg["seq_len"]
    import torch
    assert W.causal_pairs(torch.arange(S, dtype=torch.int32)) == 8_590_000_128
    assert set(bench.ALL_WORKLOADS) == set(W.WORKLOADS)


def test_stratified_rows_cover_chunk_edges_and_the_topk_boundary():
    import torch

    import workloads as W
    S, C = 131072, 8192
    r = W.stratified_rows(torch.tensor([0, S]), 512, chunk=C, positions=torch.arange(S)).tolist()
    assert len(r) == 512 and r == sorted(set(r))
    for c in range(S // C):
        assert c * C in r and c * C + C - 1 in r
    for p in (2046, 2047, 2048, 2049):
        assert p in r
    # every 1/64 of the range holds a sampled row
    assert len({t * 64 // S for t in r}) == 64


def test_mla_inputs_are_seeded_distinct_selections_padded_with_minus_one():
    import torch
    import workloads as W
    a = W.make_mla(3, [5000, 100], [2, 3], n_heads=8, k_sel=256, pad=6)
    b = W.make_mla(3, [5000, 100], [2, 3], n_heads=8, k_sel=256, pad=6)
    assert torch.equal(a.idx, b.idx) and torch.equal(a.q.view(torch.int16), b.q.view(torch.int16))
    assert a.q.shape == (5, 8, 576) and a.kv.shape == (5100, 576) and a.idx.shape == (5, 256)
    assert a.cache_offsets.tolist() == [0, 5000, 5100] and a.q_seq_offsets.tolist() == [0, 2, 5]
    for t in range(5):
        L = 5000 if t < 2 else 100
        row = a.idx[t]
        n = min(256 - 6, L)
        assert torch.all(row[n:] == -1)
        sel = row[:n]
        assert torch.all((sel >= 0) & (sel < L)) and sel.unique().numel() == n


def test_mla_decode_record_bytes_and_flops():
    # the decode batch (64 queries x 96 heads x 2,048 rows): 2,048 rows x 1,152 B + q 96 x 1,152 B
    # + idx 8 KB + out 96 x 1,024 B + lse 384 B per query; 2 x 96 x 2,048 x 1,088 flop per query
    per_query = 2048 * 1152 + 96 * 1152 + 8192 + 96 * 1024 + 384
    assert bench.mla_bytes_flops(64, 96, 2048) == (64 * per_query, 64 * 2 * 96 * 2048 * 1088)
    assert bench.mla_bytes_flops(64, 96, 2048)[0] == 164_913_152

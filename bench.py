#!/usr/bin/env python3
"""Benchmark of the DSA lightning indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path over one batch: the projections
(dsa_indexer_project: q, and k|w with the key LayerNorm) and the score + top-2,048
(dsa_indexer_topk).  The headline workload is the long-context chunked prefill:
one 131,072-token sequence processed as 16 chunks of 8,192 queries, each chunk
projected and then scored against every causal prior key of the cache
(8,590,000,128 causal pairs per step).  The other four workloads (prefill_3k,
prefill_8k, prefill_2x32k_heavy, decode_64) are timed in the same run and reported
under "workloads", each with its own roofline.  Inputs are seeded synthetic tensors
resident in HBM; L2 is flushed (256 MB write) between timed steps, outside the
timed events.

With N > 1 (torchrun), every rank runs its own independent batch (weak scaling,
no collective on the data path); times are the max over ranks.  --impl reference
times the CPU oracle on bounded samples of the same workload.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "indexer score+top-2048 Gpairs/s (prefill), decode GB/s; % of roofline"
FLOP_PER_PAIR = 2 * 32 * 128           # one (query, key) pair: 32 heads x 128-dim dot products
L2_FLUSH_BYTES = 256 << 20
HEADLINE = "chunked_128k"
PREFILL_WORKLOADS = ["prefill_3k", "prefill_8k", "prefill_2x32k_heavy", "chunked_128k"]
ALL_WORKLOADS = PREFILL_WORKLOADS + ["decode_64"]

# kernels of this library launched by one call of each entry point (the timed region holds
# nothing else of ours): project = q GEMM + k|w GEMM with the LayerNorm epilogue;
# topk = prep + score kernel, plus the merge on the split-key path
LAUNCHES = {"project": 2, "topk": 2, "topk_split": 3, "sparse_mla": 1}

# sparse MLA over the selection ('Latent attention (MLA)' row): 96 heads, 576 cached values
# per token (512 latent + 64 rope), 2,048 selected tokens per query, scale 1/sqrt(192)
MLA_SCALE = 192 ** -0.5


# ------------------------------------------------------------------------------------------ helpers

def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def _profile_traffic(kernel_key: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summaries
    (profiles/traffic.txt lines 'key: bytes source_hash'), or None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    from dsa_lightning_indexer_03_b200 import build as B
    src_hash = B.source_hash()
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.rpartition(":")   # the key itself holds a colon (kernel:workload)
        parts = rest.split()
        if key.strip() == kernel_key and len(parts) >= 2 and parts[1] == src_hash:
            return float(parts[0])
    return None


def max_over_ranks(x, dist, device):
    """Max of a per-rank scalar over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units of all ranks per second, given the slowest rank's time for its units."""
    return units_per_rank * world / (ms * 1e-3)


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running; summary() keeps the
    samples taken between mark_start() and mark_end()."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.t0 = None
        self.t1 = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]),
                             {n for n, v in zip(names, f[6:10]) if v.lower().startswith("active")}))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        pad = datetime.timedelta(milliseconds=100)
        inside = [r for r in rows if self.t0 is not None and self.t1 is not None and self.t0 - pad <= r[0] <= self.t1 + pad]
        use = inside or rows
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(set().union(*(r[3] for r in use))), "samples": len(use),
                "in_timed_region": bool(inside)}


def _flush_l2(buf):
    buf.add_(1)


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class Spans(list):
    """CUDA event spans recorded inside one step: (kind, start event, end event)."""

    def span(self, kind, f):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        f()
        e.record()
        self.append((kind, s, e))


def _time_steps(fn, steps, flush):
    """Per-step CUDA events on the current stream (L2 flushed between steps, outside the
    events).  fn(spans) runs one step and records its projection and score + top-k calls
    as spans.  Returns per-step lists: step ms, score + top-k ms, projection ms."""
    out = []
    for _ in range(steps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        spans = Spans()
        e0.record()
        fn(spans)
        e1.record()
        out.append((e0, e1, spans))
    torch.cuda.synchronize()
    step = [a.elapsed_time(b) for a, b, _ in out]
    topk = [sum(s.elapsed_time(e) for k, s, e in sp if k == "topk") for _, _, sp in out]
    proj = [sum(s.elapsed_time(e) for k, s, e in sp if k == "project") for _, _, sp in out]
    return step, topk, proj


def projection_report(T, ms, peak_tflops, hbm_gbs):
    """Throughput of dsa_indexer_project over T tokens in ms: the q GEMM (1,536 -> 4,096)
    and the k|w GEMM (7,168 -> 128 + 32) with its LayerNorm epilogue, run concurrently.
    Algorithmic flops are the two GEMMs'; algorithmic bytes are the activations read
    once, the weights read once and q, k, w written once."""
    flops = 2 * T * (1536 * 4096 + 7168 * 160)
    nbytes = (T * (7168 * 2 + 1536 * 2 + 4096 * 2 + 128 * 2 + 32 * 4)
              + (1536 * 4096 + 7168 * 160) * 2)
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 4), "tokens": T, "flop": flops, "bytes": nbytes,
            "achieved_tflops": round(tflops, 2), "frac_tensor": round(tflops / peak_tflops, 4),
            "achieved_gbs": round(gbs, 2), "frac_hbm": round(gbs / hbm_gbs, 4)}


LONG_TIMED_S = 1.0   # a timed region at least this long runs the kernels back to back for seconds


def tensor_peak(peaks, timed_s, fp8=False):
    """The bf16 tensor peak a kernel is held to: the burst figure when its timed region is short,
    the sustained one (the same GEMM run back to back for seconds, under the power cap) when the
    timed region lasts LONG_TIMED_S or more.  FP8 operands: times the nominal fp8 / bf16 ratio 2.
    Returns (peak TFLOP/s, description)."""
    long_run = timed_s >= LONG_TIMED_S and "bf16_tflops_sustained" in peaks
    peak = (peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]) * (2 if fp8 else 1)
    what = (f"sustained bf16 (timed region {timed_s:.1f} s, back to back)" if long_run
            else f"burst bf16 (timed region {timed_s:.2f} s)")
    src = "of measured" if peaks["source"] == "measured" else "of fallback"
    return peak, f"{peaks['source']} {what}" + (" x 2 (fp8)" if fp8 else "") + f" ({src})"


def prefill_roofline(pairs, topk_ms, peaks, traffic, fp8=False, timed_s=0.0):
    """Roofline of the score + top-k over a prefill workload: pairs x 8,192 flop over the
    summed dsa_indexer_topk time, against the measured bf16 peak that tensor_peak picks for
    the length of the timed region; frac_burst is the fraction of the burst peak either way."""
    tflops = pairs * FLOP_PER_PAIR / (topk_ms * 1e-3) / 1e12
    peak, source = tensor_peak(peaks, timed_s, fp8)
    burst = peaks["bf16_tflops"] * (2 if fp8 else 1)
    return {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(tflops / peak, 4), "frac_burst": round(tflops / burst, 4), "traffic": traffic,
            "kernel": "score_topk (dsa_indexer_topk: prep + score)", "ms_per_launch": None,
            "ms_topk_per_step": round(topk_ms, 4), "gpairs_score_topk": round(pairs / (topk_ms * 1e-3) / 1e9, 3),
            "peak_source": source}


# ------------------------------------------------------------------------------------------ GPU arm: workloads

def _make_indexer(d, wts, device, max_tokens):
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    return d.Indexer(to(wts.W_q), to(wts.W_k), to(wts.W_w), to(wts.gamma), to(wts.beta), max_tokens=max_tokens)


def setup_prefill(d, name, seed_offset, device, fp8=False):
    """Inputs of a prefill workload, resident on the device.  A prefill job is a list of
    calls ("chunks"): one call for the single-shot prefills, 16 calls of 8,192 queries for
    the chunked long-context prefill, each scoring against the keys of every earlier chunk."""
    cfg = W.WORKLOADS[name]
    wts = W.make_weights(cfg["weight_seed"])
    seed = cfg["act_seed"] + seed_offset
    if cfg["kind"] == "chunked":
        S, C = cfg["seq_len"], cfg["chunk"]
        parts = [W.make_prefill(seed, [C], start_positions=[c * C], cache_lens=[S], sub=c) for c in range(S // C)]
        hidden = torch.cat([p.hidden for p in parts])
        q_latent = torch.cat([p.q_latent for p in parts])
        positions = torch.cat([p.positions for p in parts])
        qoffs = [torch.tensor([0, C], dtype=torch.int32) for _ in parts]
        coff = torch.tensor([0, S], dtype=torch.int64)
        bounds = [(c * C, (c + 1) * C) for c in range(S // C)]
        heavy = None
        seq_offsets = torch.tensor([0, S], dtype=torch.int32)
    else:
        batch = W.make_prefill(seed, cfg["seq_lens"])
        hidden, q_latent, positions = batch.hidden, batch.q_latent, batch.positions
        T = hidden.shape[0]
        qoffs = [batch.q_seq_offsets]
        coff = batch.cache_offsets
        bounds = [(0, T)]
        heavy = W.heavy_hitter_rows(seed, coff, cfg["heavy_frac"]) if "heavy_frac" in cfg else None
        seq_offsets = batch.q_seq_offsets
    T = hidden.shape[0]
    chunk_T = max(b - a for a, b in bounds)
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    st = dict(name=name, T=T, bounds=bounds, ix=_make_indexer(d, wts, device, max(chunk_T, 256)),
              host=dict(hidden=hidden, q_latent=q_latent, positions=positions, qoffs=qoffs, coff=coff),
              hidden=to(hidden), q_latent=to(q_latent), positions=to(positions),
              qoffs=[to(q) for q in qoffs], coff=to(coff), seq_offsets=seq_offsets,
              heavy=None if heavy is None else to(heavy),
              cache=torch.zeros((int(coff[-1]), 128), dtype=torch.bfloat16, device=device),
              q=torch.empty((T, 32, 128), dtype=torch.bfloat16, device=device),
              w=torch.empty((T, 32), dtype=torch.float32, device=device),
              idx=torch.empty((T, 2048), dtype=torch.int32, device=device),
              score=torch.empty((T, 2048), dtype=torch.float32, device=device),
              pairs=W.causal_pairs(positions), weights=wts, fp8=fp8)
    if fp8:
        rows = int(coff[-1])
        st["cache"] = torch.zeros((rows, 128), dtype=torch.uint8, device=device)
        st["kscale"] = torch.zeros((rows,), dtype=torch.float32, device=device)
        st["q"] = torch.empty((T, 32, 128), dtype=torch.uint8, device=device)
        st["qscale"] = torch.empty((T, 32), dtype=torch.float32, device=device)
    return st


def prefill_step(st, spans):
    """One pass of the hot path over the whole workload: per call, the projections (which
    write the call's keys into the cache) and then the score + top-k."""
    ix = st["ix"]
    if st["fp8"]:
        for (a0, a1), qoff in zip(st["bounds"], st["qoffs"]):
            spans.span("project", lambda: ix.project_fp8(
                st["hidden"][a0:a1], st["q_latent"][a0:a1], st["positions"][a0:a1], qoff, st["cache"], st["kscale"],
                st["coff"], q_out=st["q"][a0:a1], q_scale=st["qscale"][a0:a1], w_out=st["w"][a0:a1]))
            spans.span("topk", lambda: ix.topk_fp8(
                st["q"][a0:a1], st["qscale"][a0:a1], st["w"][a0:a1], st["positions"][a0:a1], qoff, st["cache"],
                st["kscale"], st["coff"], idx_out=st["idx"][a0:a1], score_out=st["score"][a0:a1]))
        return
    for (a0, a1), qoff in zip(st["bounds"], st["qoffs"]):
        spans.span("project", lambda: ix.project(st["hidden"][a0:a1], st["q_latent"][a0:a1],
                                                 st["positions"][a0:a1], qoff, st["cache"], st["coff"],
                                                 q_out=st["q"][a0:a1], w_out=st["w"][a0:a1]))
        if st["heavy"] is not None:
            # the workload's 1 % heavy-hitter key rows (x4, exact in bf16), applied to the
            # freshly written cache before scoring; an input-preparation step, outside the spans
            st["cache"][st["heavy"]] *= 4
        spans.span("topk", lambda: ix.topk(st["q"][a0:a1], st["w"][a0:a1], st["positions"][a0:a1], qoff,
                                           st["cache"], st["coff"], idx_out=st["idx"][a0:a1],
                                           score_out=st["score"][a0:a1]))


def setup_decode(d, seed_offset, device, fp8=False):
    cfg = W.WORKLOADS["decode_64"]
    wts = W.make_weights(cfg["weight_seed"])
    lengths = W.decode_lengths(cfg["act_seed"] + seed_offset, cfg["batch"], cfg["L_min"], cfg["L_max"])
    batch = W.make_decode(cfg["act_seed"] + seed_offset, lengths=torch.ones_like(lengths))  # new tokens only
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    ix = _make_indexer(d, wts, device, 256)
    B = cfg["batch"]
    total = int(lengths.sum())
    coff = torch.zeros(B + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(lengths, 0)
    # cached keys: LayerNorm (through the library) of N(0,1) pre-norm rows drawn on the device
    gd = torch.Generator(device=device).manual_seed(2000 + seed_offset)
    cache = torch.empty((total, 128), dtype=torch.bfloat16, device=device)
    step = 1 << 20
    for s in range(0, total, step):
        n = min(step, total - s)
        raw = torch.randn((n, 128), generator=gd, device=device, dtype=torch.float32)
        ix.key_norm(raw, out=cache[s:s + n])
    torch.cuda.synchronize()
    positions = (lengths - 1).to(torch.int32)
    st = dict(name="decode_64", ix=ix, T=B, hidden=to(batch.hidden), q_latent=to(batch.q_latent),
              positions=to(positions), qoff=to(torch.arange(B + 1, dtype=torch.int32)), coff=to(coff), cache=cache,
              q=torch.empty((B, 32, 128), dtype=torch.bfloat16, device=device),
              w=torch.empty((B, 32), dtype=torch.float32, device=device),
              idx=torch.empty((B, 2048), dtype=torch.int32, device=device),
              score=torch.empty((B, 2048), dtype=torch.float32, device=device),
              total_keys=total, lengths=lengths)
    st["fp8"] = fp8
    if fp8:
        # the FP8 cache of the same keys: e4m3 codes and one scale per row
        st["cache"], st["kscale"] = ix.quantize_keys_fp8(cache)
        del cache
        st["q"] = torch.empty((B, 32, 128), dtype=torch.uint8, device=device)
        st["qscale"] = torch.empty((B, 32), dtype=torch.float32, device=device)
        torch.cuda.synchronize()
    # algorithmic bytes of the score + top-k: every cached key once (with its scale for FP8),
    # q (and its head scales) and w once, indices + scores out
    if fp8:
        st["bytes"] = total * (128 + 4) + B * (32 * 128 + 32 * 4 + 32 * 4) + B * 2048 * (4 + 4)
    else:
        st["bytes"] = total * 128 * 2 + B * (32 * 128 * 2 + 32 * 4) + B * 2048 * (4 + 4)
    return st


def decode_step(ds, spans):
    ix = ds["ix"]
    if ds["fp8"]:
        spans.span("project", lambda: ix.project_fp8(ds["hidden"], ds["q_latent"], ds["positions"], ds["qoff"],
                                                     ds["cache"], ds["kscale"], ds["coff"], q_out=ds["q"],
                                                     q_scale=ds["qscale"], w_out=ds["w"]))
        spans.span("topk", lambda: ix.topk_fp8(ds["q"], ds["qscale"], ds["w"], ds["positions"], ds["qoff"],
                                               ds["cache"], ds["kscale"], ds["coff"], idx_out=ds["idx"],
                                               score_out=ds["score"]))
        return
    spans.span("project", lambda: ix.project(ds["hidden"], ds["q_latent"], ds["positions"], ds["qoff"], ds["cache"],
                                             ds["coff"], q_out=ds["q"], w_out=ds["w"]))
    spans.span("topk", lambda: ix.topk(ds["q"], ds["w"], ds["positions"], ds["qoff"], ds["cache"], ds["coff"],
                                       idx_out=ds["idx"], score_out=ds["score"]))


def e2e_prefill(st, steps):
    """The same workload through the public API with host buffers: every step copies each
    call's inputs in from pinned host memory (on an H2D stream, all calls queued at once so
    that the copies run ahead of the compute) and each call's indices out (on a D2H stream,
    queued behind that call), so that call c's indices return while call c+1 is scored and
    later inputs arrive.  Returns (ms per step, H2D bytes, D2H bytes)."""
    h = st["host"]
    ix = st["ix"]
    T = st["T"]
    pin = {k: h[k].pin_memory() for k in ("hidden", "q_latent", "positions", "coff")}
    pin_qoffs = [q.pin_memory() for q in h["qoffs"]]
    out = torch.empty((T, 2048), dtype=torch.int32).pin_memory()
    bi = sum(t.numel() * t.element_size() for t in pin.values()) + sum(q.numel() * 4 for q in pin_qoffs)
    bo = out.numel() * out.element_size()
    dev = st["hidden"].device
    h2d = torch.cuda.Stream(device=dev)
    d2h = torch.cuda.Stream(device=dev)
    main = torch.cuda.current_stream(dev)
    ts = []
    for _ in range(steps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        h2d.wait_stream(main)
        d2h.wait_stream(main)
        arrived = []
        with torch.cuda.stream(h2d):
            st["coff"].copy_(pin["coff"], non_blocking=True)
            for (a0, a1), qd, qh in zip(st["bounds"], st["qoffs"], pin_qoffs):
                qd.copy_(qh, non_blocking=True)
                st["hidden"][a0:a1].copy_(pin["hidden"][a0:a1], non_blocking=True)
                st["q_latent"][a0:a1].copy_(pin["q_latent"][a0:a1], non_blocking=True)
                st["positions"][a0:a1].copy_(pin["positions"][a0:a1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(h2d)
                arrived.append(ev)
        for ((a0, a1), qoff), ev_in in zip(zip(st["bounds"], st["qoffs"]), arrived):
            main.wait_event(ev_in)
            ix.project(st["hidden"][a0:a1], st["q_latent"][a0:a1], st["positions"][a0:a1], qoff, st["cache"],
                       st["coff"], q_out=st["q"][a0:a1], w_out=st["w"][a0:a1])
            if st["heavy"] is not None:
                st["cache"][st["heavy"]] *= 4
            ix.topk(st["q"][a0:a1], st["w"][a0:a1], st["positions"][a0:a1], qoff, st["cache"], st["coff"],
                    idx_out=st["idx"][a0:a1], score_out=st["score"][a0:a1])
            done = torch.cuda.Event()
            done.record(main)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                out[a0:a1].copy_(st["idx"][a0:a1], non_blocking=True)
        main.wait_stream(d2h)
        e1.record(main)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.mean(ts), bi, bo


def run_prefill(d, name, rank, device, steps, warmup, flush, peaks, mx, clk=None, fp8=False):
    st = setup_prefill(d, name, rank, device, fp8)
    fn = lambda spans: prefill_step(st, spans)  # noqa: E731
    _time_steps(fn, warmup, flush)
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark_start()
    step_ms, topk_ms, proj_ms = _time_steps(fn, steps, flush)
    if clk is not None:
        clk.mark_end()
    ms = mx(statistics.mean(step_ms))
    topk_avg = mx(statistics.mean(topk_ms))
    proj_avg = mx(statistics.mean(proj_ms))
    timed_s = mx(sum(step_ms)) * 1e-3
    err = st["ix"].device_error()
    n_calls = len(st["bounds"])
    rec = {"workload": name + ("_fp8" if fp8 else ""), "metric": "indexer score+top-2048 Gpairs/s (prefill)",
           "value": None, "unit": "Gpairs/s", "ms_per_step": round(ms, 4), "causal_pairs": st["pairs"],
           "tokens": st["T"], "calls_per_step": n_calls,
           "roofline": prefill_roofline(st["pairs"], topk_avg, peaks,
                                        _profile_traffic(f"score_topk:{name}" + ("_fp8" if fp8 else "")), fp8, timed_s),
           "projections": projection_report(st["T"], proj_avg, tensor_peak(peaks, timed_s)[0], peaks["hbm_gbs"]),
           "device_error": err, "gpu_launches_per_step": n_calls * (LAUNCHES["project"] + LAUNCHES["topk"])}
    rec["roofline"]["ms_per_launch"] = round(topk_avg / n_calls, 4)
    return st, rec, ms


def run_decode(d, rank, device, steps, warmup, flush, peaks, mx, fp8=False):
    ds = setup_decode(d, rank, device, fp8)
    fn = lambda spans: decode_step(ds, spans)  # noqa: E731
    _time_steps(fn, warmup, flush)
    dstep, dtopk, dproj = _time_steps(fn, steps, flush)
    dms = mx(statistics.mean(dtopk))
    dstep_ms = mx(statistics.mean(dstep))
    gbs = ds["bytes"] / (dms * 1e-3) / 1e9
    rec = {"workload": "decode_64" + ("_fp8" if fp8 else ""), "metric": "decode GB/s", "value": None, "unit": "GB/s",
           "keys_per_s": round(ds["total_keys"] / (dms * 1e-3) / 1e9, 3),
           "ms_score_topk": round(dms, 4), "ms_per_step": round(dstep_ms, 4), "ms_project": round(
               mx(statistics.mean(dproj)), 4),
           "keys_scanned": ds["total_keys"], "algorithmic_bytes": ds["bytes"],
           "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(gbs / peaks["hbm_gbs"], 4),
                        "traffic": _profile_traffic("score_topk:decode_64" + ("_fp8" if fp8 else "")),
                        "kernel": "score_topk split-key + merge (dsa_indexer_topk)", "ms_per_launch": round(dms, 4),
                        "peak_source": peaks["source"] + " HBM copy"},
           "device_error": ds["ix"].device_error(),
           "gpu_launches_per_step": LAUNCHES["project"] + LAUNCHES["topk_split"]}
    return ds, rec, gbs


def mla_bytes_flops(T, H, k):
    """Algorithmic bytes of a sparse MLA call (every selected 1,152-byte row once, q, the index
    rows, out and lse) and its useful flops (q . row over 576 values and p . latent over 512,
    per head and selected token)."""
    return (T * k * 576 * 2 + T * H * 576 * 2 + T * k * 4 + T * H * (512 * 2 + 4),
            2 * T * H * k * (576 + 512))


def setup_mla_decode(seed_offset, device, small=False):
    """The decode step's sparse MLA: 64 sequences of 16,384..131,072 cached 576-value rows,
    one query of 96 heads each, 2,048 selected positions per query (distinct, uniform over
    the sequence: the access pattern of an unsorted top-k row).  small: sequences of 2,048
    rows (every row selected once, in random order; a 151 MB cache for profiler captures)."""
    cfg = W.WORKLOADS["decode_64"]
    lengths = W.decode_lengths(cfg["act_seed"] + seed_offset, cfg["batch"], cfg["L_min"], cfg["L_max"])
    if small:
        lengths = torch.full_like(lengths, 2048)
    b = W.make_mla(cfg["act_seed"] + seed_offset, lengths.tolist(), [1] * cfg["batch"], device=str(device))
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    T, H, k = b.q.shape[0], b.q.shape[1], b.idx.shape[1]
    ms = dict(q=to(b.q), kv=b.kv, coff=to(b.cache_offsets), qoff=to(b.q_seq_offsets), idx=to(b.idx),
              out=torch.empty((T, H, 512), dtype=torch.bfloat16, device=device),
              lse=torch.empty((T, H), dtype=torch.float32, device=device), T=T, H=H, k=k)
    ms["bytes"], ms["flops"] = mla_bytes_flops(T, H, k)
    torch.cuda.synchronize()
    return ms


def mla_call(ix, ms):
    ix.sparse_mla(ms["q"], ms["kv"], ms["coff"], ms["qoff"], ms["idx"], MLA_SCALE, out=ms["out"], lse=ms["lse"])


def run_mla_decode(d, ix, rank, device, steps, warmup, flush, peaks, mx):
    ms = setup_mla_decode(rank, device)
    fn = lambda spans: spans.span("topk", lambda: mla_call(ix, ms))  # noqa: E731
    _time_steps(fn, warmup, flush)
    _, t, _ = _time_steps(fn, steps, flush)
    dms = mx(statistics.mean(t))
    gbs = ms["bytes"] / (dms * 1e-3) / 1e9
    rec = {"workload": "sparse_mla_decode_64", "metric": "sparse MLA decode GB/s", "value": None, "unit": "GB/s",
           "queries": ms["T"], "heads": ms["H"], "selected": ms["k"], "ms_per_step": round(dms, 4),
           "tflops": round(ms["flops"] / (dms * 1e-3) / 1e12, 2), "algorithmic_bytes": ms["bytes"],
           "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": _profile_traffic("sparse_mla:decode_64"),
                        "kernel": "sparse_mla_kernel (dsa_indexer_sparse_mla)", "ms_per_launch": round(dms, 4),
                        "peak_source": peaks["source"] + " HBM copy"},
           "device_error": ix.device_error(), "gpu_launches_per_step": LAUNCHES["sparse_mla"]}
    return ms, rec, gbs


def gpu_arm(args, rank, world, local_rank, dist):
    import dsa_lightning_indexer_03_b200 as d
    from dsa_lightning_indexer_03_b200 import build as B
    B.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    peaks = _peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush = lambda: _flush_l2(flush_buf)  # noqa: E731

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def mx(x):
        return max_over_ranks(x, dist, device)

    # ---------------- headline: every rank runs the same sequence of timed sections
    barrier()
    with ClockSampler(device.index) as clk:
        st, head, ms = run_prefill(d, args.workload, rank, device, args.steps, args.warmup, flush, peaks, mx, clk)
    barrier()
    clocks = clk.summary()
    value = whole_job_rate(st["pairs"], world, ms) / 1e9
    head["value"] = round(value, 3)
    e2e_ms, bi, bo = e2e_prefill(st, max(2, min(args.steps, 5)))
    e2e_ms = mx(e2e_ms)
    cfg = W.WORKLOADS[args.workload]
    del st
    torch.cuda.empty_cache()

    # ---------------- the other workloads, each with its own roofline
    subs = {}
    if not args.headline_only:
        for name in PREFILL_WORKLOADS:
            if name == args.workload:
                continue
            few = name in ("prefill_2x32k_heavy", "chunked_128k")
            n = args.steps if few else max(args.steps, 100)
            s2, rec, ms2 = run_prefill(d, name, rank, device, n, args.warmup, flush, peaks, mx)
            rec["value"] = round(whole_job_rate(s2["pairs"], world, ms2) / 1e9, 3)
            rec["steps"] = n
            subs[name] = rec
            del s2
            torch.cuda.empty_cache()
        n = max(args.steps, 100)
        for fp8 in (False, True):
            ds, rec, gbs = run_decode(d, rank, device, n, args.warmup, flush, peaks, mx, fp8)
            rec["value"] = round(gbs * world, 2)
            rec["steps"] = n
            subs[rec["workload"]] = rec
            del ds
            torch.cuda.empty_cache()
        # the consumer of the selection: sparse MLA attention of the decode batch
        ix = _make_indexer(d, W.make_weights(W.WORKLOADS["decode_64"]["weight_seed"], hidden_dim=256,
                                             q_latent_dim=128), device, 256)
        ms, rec, gbs = run_mla_decode(d, ix, rank, device, n, args.warmup, flush, peaks, mx)
        rec["value"] = round(gbs * world, 2)
        rec["steps"] = n
        subs[rec["workload"]] = rec
        del ms, ix
        torch.cuda.empty_cache()
        # the FP8 cache on the 8,192-token prefill (FP8 tensor-core scoring)
        s2, rec, ms2 = run_prefill(d, "prefill_8k", rank, device, n, args.warmup, flush, peaks, mx, fp8=True)
        rec["value"] = round(whole_job_rate(s2["pairs"], world, ms2) / 1e9, 3)
        rec["steps"] = n
        subs[rec["workload"]] = rec
        del s2
        torch.cuda.empty_cache()

    launches = head["gpu_launches_per_step"] * args.steps
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "Gpairs/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) random-init weights)",
        "config": {"workload": args.workload,
                   "batch": 1 if cfg["kind"] == "chunked" else len(cfg["seq_lens"]),
                   "seq_len": cfg["seq_len"] if cfg["kind"] == "chunked" else cfg["seq_lens"][0],
                   "chunk": cfg.get("chunk"), "calls_per_step": head["calls_per_step"],
                   "heads": 32, "head_dim": 128, "top_k": 2048, "causal_pairs_per_gpu": head["causal_pairs"],
                   "parallelism": f"independent replicas x{world}",
                   "l2": "flushed between timed steps (256 MB write); inputs larger than L2"},
        "roofline": head["roofline"],
        "e2e": {"value": round(whole_job_rate(head["causal_pairs"], world, e2e_ms) / 1e9, 3), "unit": "Gpairs/s",
                "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(e2e_ms, 4)},
        "projections": head["projections"],
        "clocks": clocks,
        "gpu_launches": launches,
        "device_error": head["device_error"],
    }
    if subs:
        line["workloads"] = subs
    return line


# ------------------------------------------------------------------------------------------ CPU oracle

def _oracle_weights(wts):
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    return f(wts.W_q), f(wts.W_k), f(wts.W_w), f(wts.gamma), f(wts.beta)


def cpu_oracle_workload(name, n_rows=512, proj_tokens=256, seed=0, full=None):
    """The oracle as it stands, timed on the workload: its projection (seconds per token,
    from `proj_tokens` tokens or every token) and its score + top-k (seconds per causal
    pair, from every query row or a stratified sample of `n_rows`: the first and last row
    of every sequence and chunk, the rows at positions 2,046..2,049, one seeded row per
    equal stratum), extrapolated to the whole workload where sampled.  The score step's
    cost does not depend on the key values, so sampled runs score against the oracle's
    LayerNorm of N(0,1) pre-norm rows (the keys' distribution) instead of projecting every
    key.  Returns (value, unit, description, seconds spent)."""
    import numpy as np

    import oracle
    cfg = W.WORKLOADS[name]
    wts = W.make_weights(cfg["weight_seed"])
    Wq, Wk, Ww, g, b = _oracle_weights(wts)
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    spent = 0.0
    if cfg["kind"] == "decode":
        lengths = W.decode_lengths(cfg["act_seed"], cfg["batch"], cfg["L_min"], cfg["L_max"])
        batch = W.make_decode(cfg["act_seed"], lengths=torch.ones_like(lengths))
        t0 = time.perf_counter()
        q, k_new, w = oracle.project(f(batch.hidden), f(batch.q_latent), Wq, Wk, Ww, g, b)
        t_proj = time.perf_counter() - t0
        t_norm = 0.0
        t_topk = 0.0
        for bi, L in enumerate(lengths.tolist()):   # one sequence's cache at a time
            raw = W.make_decode(cfg["act_seed"] + 1000 + bi, lengths=[L]).raw_keys
            t0 = time.perf_counter()
            keys = oracle.key_norm(raw.numpy().astype(np.float64), g, b)
            keys[L - 1] = k_new[bi]
            t1 = time.perf_counter()
            oracle.topk(q[bi:bi + 1], w[bi:bi + 1], np.array([L - 1]), np.array([0, 1]), keys, np.array([0, L]))
            t_topk += time.perf_counter() - t1
            t_norm += t1 - t0
        total = int(lengths.sum())
        nbytes = total * 128 * 2 + len(lengths) * (32 * 128 * 2 + 32 * 4) + len(lengths) * 2048 * 8
        spent = t_proj + t_norm + t_topk
        gbs = nbytes / (t_proj + t_topk) / 1e9
        desc = (f"decode_64 in full: projection of the 64 new tokens ({t_proj:.2f} s) and score+top-k of the 64 "
                f"queries over all {total} cached keys ({t_topk:.2f} s; the cache's LayerNorm, {t_norm:.1f} s, is "
                f"input preparation and not counted); algorithmic bytes {nbytes} as for the GPU")
        return gbs, "GB/s", desc, spent
    if cfg["kind"] == "chunked":
        S, C = cfg["seq_len"], cfg["chunk"]
        positions = torch.arange(S, dtype=torch.int32)
        qoff = torch.tensor([0, S], dtype=torch.int32)
        coff = np.array([0, S])
        chunk = C
        tok = W.make_prefill(cfg["act_seed"], [proj_tokens], start_positions=[S - proj_tokens], cache_lens=[S],
                             sub=S // C - 1)
        hid_s, qlat_s = tok.hidden, tok.q_latent
    else:
        batch = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
        positions, qoff = batch.positions, batch.q_seq_offsets
        coff = batch.cache_offsets.numpy()
        chunk = None
        hid_s, qlat_s = batch.hidden, batch.q_latent
    T = positions.numel()
    full = (T <= 8192) if full is None else full
    if full:
        rows = np.arange(T)
        n_tok = T
    else:
        rows = W.stratified_rows(qoff, n_rows, seed=seed, chunk=chunk, positions=positions).numpy()
        n_tok = min(proj_tokens, hid_s.shape[0])
    t0 = time.perf_counter()
    q_s, k_s, w_s = oracle.project(f(hid_s[:n_tok]), f(qlat_s[:n_tok]), Wq, Wk, Ww, g, b)
    t_proj_tok = (time.perf_counter() - t0) / n_tok
    spent += t_proj_tok * n_tok
    seq = oracle.sequence_of(qoff.numpy(), T)
    if full:
        keys = k_s
        qq, ww, pos_r = q_s, w_s, positions.numpy()
        qoff_r = qoff.numpy()
        if "heavy_frac" in cfg:
            keys = keys.copy()
            keys[W.heavy_hitter_rows(cfg["act_seed"], batch.cache_offsets, cfg["heavy_frac"]).numpy()] *= 4
    else:
        rows_cache = int(coff[-1])
        keys = oracle.key_norm(W.make_decode(cfg["act_seed"], lengths=[rows_cache]).raw_keys.numpy()
                               .astype(np.float64), g, b)
        if "heavy_frac" in cfg:
            keys[W.heavy_hitter_rows(cfg["act_seed"], batch.cache_offsets, cfg["heavy_frac"]).numpy()] *= 4
        # the sampled rows as a batch of their own: q, w from the oracle's projection of the
        # sampled tokens (reused cyclically), each row in its own sequence's key range
        qq = q_s[np.arange(len(rows)) % n_tok]
        ww = w_s[np.arange(len(rows)) % n_tok]
        pos_r = positions.numpy()[rows]
        qoff_r = np.zeros(len(coff), np.int64)
        qoff_r[1:] = np.cumsum(np.bincount(seq[rows], minlength=len(coff) - 1))
    t0 = time.perf_counter()
    oracle.topk(qq, ww, pos_r, qoff_r, keys, coff)
    t_topk = time.perf_counter() - t0
    spent += t_topk
    pairs_s = int((positions.numpy()[rows].astype(np.int64) + 1).sum())
    total_pairs = W.causal_pairs(positions)
    t_full = T * t_proj_tok + total_pairs * (t_topk / pairs_s)
    if full:
        desc = (f"{name} in full: projection of all {T} tokens ({t_proj_tok * T:.1f} s) and score+top-k of all {T} "
                f"query rows ({total_pairs} causal pairs, {t_topk:.1f} s)")
    else:
        desc = (f"{name}: projection of {n_tok} tokens ({t_proj_tok * 1e3:.2f} ms/token) and score+top-k of "
                f"{len(rows)} stratified query rows (first/last row of every sequence and chunk, positions "
                f"2046-2049, one seeded row per stratum; {pairs_s} causal pairs, {t_topk:.1f} s), extrapolated to "
                f"all {T} tokens / {total_pairs} pairs ({t_full:.0f} s)")
    return total_pairs / t_full / 1e9, "Gpairs/s", desc, spent


def cpu_baselines(headline, all_workloads=True):
    """cpu_baseline of the headline workload and of every other one (rank 0, N=1 only)."""
    cores = _cpu_threads()
    out = {}
    names = [headline] + ([n for n in ALL_WORKLOADS if n != headline] if all_workloads else [])
    for name in names:
        v, unit, desc, spent = cpu_oracle_workload(name)
        out[name] = {"value": float(f"{v:.6g}"), "unit": unit, "cores": cores, "kind": "oracle",
                     "sample": desc + f"; one process, numpy BLAS on {cores} threads for the matmuls"}
        print(f"cpu_baseline {name}: {v:.4g} {unit} ({spent:.1f} s)", file=sys.stderr, flush=True)
    return out


def reference_arm(args):
    """The reference arm: the oracle as it stands on bounded samples of the headline workload
    (each step: 16 stratified query rows and the projection of 16 tokens, seeded by the step)."""
    vals = []
    desc = ""
    for i in range(min(args.warmup, 1)):
        cpu_oracle_workload(args.workload, n_rows=4, proj_tokens=4, seed=10_000 + i, full=False)
    wall = 0.0
    for i in range(args.steps):
        v, unit, desc, spent = cpu_oracle_workload(args.workload, n_rows=16, proj_tokens=16, seed=i, full=False)
        vals.append(v)
        wall += spent
    value = statistics.mean(vals)
    cores = _cpu_threads()
    cfg = W.WORKLOADS[args.workload]
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": float(f"{value:.6g}"),
        "unit": "Gpairs/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(wall / max(args.steps, 1) * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload,
                   "batch": 1 if cfg["kind"] == "chunked" else len(cfg.get("seq_lens", [1])),
                   "seq_len": cfg.get("seq_len") or cfg["seq_lens"][0], "top_k": 2048},
        "cpu_baseline": {"value": float(f"{value:.6g}"), "unit": "Gpairs/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}; one process, numpy BLAS on {cores} threads"},
        "e2e": {"value": float(f"{value:.6g}"), "unit": "Gpairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------------------ profiling driver

def profile_call(d, spec, repeats):
    """A small case for ncu captures: one dsa_indexer_topk call of a workload, repeated.
    spec is WORKLOAD[:CALL]; for the chunked prefill the cache is filled by projecting the
    chunks up to CALL one at a time, so the device holds one chunk's tensors, the key
    cache and the workspace (well under 1 GB); CALL "all" runs every chunk's call.  Prints the call's CUDA-event times."""
    name, _, call = spec.partition(":")
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if name == "project":
        # the projections of one workload's first call (dsa_indexer_project), timed alone
        st = setup_prefill(d, call, 0, device)
        (a0, a1), qoff = st["bounds"][0], st["qoffs"][0]
        ix = st["ix"]
        for i in range(repeats + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ix.project(st["hidden"][a0:a1], st["q_latent"][a0:a1], st["positions"][a0:a1], qoff, st["cache"],
                       st["coff"], q_out=st["q"][a0:a1], w_out=st["w"][a0:a1])
            e1.record()
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            r = projection_report(a1 - a0, ms, 1646.6, 6551.7)
            print(f"{spec} call {i}: {ms:.4f} ms, {r['achieved_gbs']:.1f} GB/s, {r['achieved_tflops']:.1f} TFLOP/s",
                  flush=True)
        assert ix.device_error() == d.DSA_OK
        return
    if name in ("decode_64", "decode_64_fp8"):
        fp8 = name.endswith("_fp8")
        ds = setup_decode(d, 0, device, fp8)
        spans = Spans()
        decode_step(ds, spans)      # the projections write the new keys; then time the calls
        torch.cuda.synchronize()
        for i in range(repeats):
            spans = Spans()
            decode_step(ds, spans)
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for k, a, b in spans if k == "topk")
            print(f"{spec} call {i}: {ms:.4f} ms, {ds['bytes'] / ms / 1e6:.1f} GB/s, 0 TFLOP/s", flush=True)
        assert ds["ix"].device_error() == d.DSA_OK
        return
    if name in ("sparse_mla_decode_64", "sparse_mla_small"):
        ix = _make_indexer(d, W.make_weights(0, hidden_dim=256, q_latent_dim=128), device, 256)
        ms = setup_mla_decode(0, device, small=name == "sparse_mla_small")
        for i in range(repeats):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mla_call(ix, ms)
            e1.record()
            e1.synchronize()
            t = e0.elapsed_time(e1)
            print(f"{spec} call {i}: {t:.4f} ms, {ms['bytes'] / t / 1e6:.1f} GB/s, "
                  f"{ms['flops'] / t / 1e9:.1f} TFLOP/s", flush=True)
        assert ix.device_error() == d.DSA_OK
        return
    cfg = W.WORKLOADS[name]
    wts = W.make_weights(cfg["weight_seed"])
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    def run_calls(label, ix, q, w, pos, qoff, cache, coff, pairs):
        idx = torch.empty((q.shape[0], 2048), dtype=torch.int32, device=device)
        sc = torch.empty((q.shape[0], 2048), dtype=torch.float32, device=device)
        torch.cuda.synchronize()
        for i in range(repeats):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ix.topk(q, w, pos, qoff, cache, coff, idx_out=idx, score_out=sc)
            e1.record()
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            print(f"{label} call {i}: {ms:.4f} ms, {pairs / ms / 1e6:.2f} Gpairs/s, "
                  f"{pairs * FLOP_PER_PAIR / ms / 1e9:.1f} TFLOP/s", flush=True)
        assert ix.device_error() == d.DSA_OK

    if cfg["kind"] == "chunked":
        # CALL = one chunk's call (the earlier chunks only fill the cache), or "all": every
        # chunk's call in order, each right after its chunk was projected
        S, C = cfg["seq_len"], cfg["chunk"]
        every = call == "all"
        c_last = S // C - 1 if (every or not call) else int(call)
        ix = _make_indexer(d, wts, device, C)
        cache = torch.zeros((S, 128), dtype=torch.bfloat16, device=device)
        coff = to(torch.tensor([0, S], dtype=torch.int64))
        qoff = to(torch.tensor([0, C], dtype=torch.int32))
        for c in range(c_last + 1):
            b = W.make_prefill(cfg["act_seed"], [C], start_positions=[c * C], cache_lens=[S], sub=c)
            pos = to(b.positions)
            q, w = ix.project(to(b.hidden), to(b.q_latent), pos, qoff, cache, coff)
            if every:
                run_calls(f"{name}:{c}", ix, q, w, pos, qoff, cache, coff, W.causal_pairs(b.positions))
        if every:
            return
        pairs = W.causal_pairs(b.positions)
    else:
        b = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
        ix = _make_indexer(d, wts, device, max(b.hidden.shape[0], 256))
        cache = torch.zeros((int(b.cache_offsets[-1]), 128), dtype=torch.bfloat16, device=device)
        pos, qoff, coff = to(b.positions), to(b.q_seq_offsets), to(b.cache_offsets)
        q, w = ix.project(to(b.hidden), to(b.q_latent), pos, qoff, cache, coff)
        if "heavy_frac" in cfg:
            cache[to(W.heavy_hitter_rows(cfg["act_seed"], b.cache_offsets, cfg["heavy_frac"]))] *= 4
        pairs = W.causal_pairs(b.positions)
    run_calls(spec, ix, q, w, pos, qoff, cache, coff, pairs)


# ------------------------------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=HEADLINE, choices=PREFILL_WORKLOADS)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads' records")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-call", default=None, metavar="WORKLOAD[:CALL]",
                    help="only run one score + top-k call of a workload --steps times (for ncu captures)")
    args = ap.parse_args()
    if args.profile_call:
        import dsa_lightning_indexer_03_b200 as d
        from dsa_lightning_indexer_03_b200 import build as B
        B.build()
        profile_call(d, args.profile_call, args.steps)
        return
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return

    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    line = gpu_arm(args, rank, world, local_rank, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baselines(args.workload, all_workloads=not args.headline_only)
        line["cpu_baseline"] = cb[args.workload]
        for name, rec in line.get("workloads", {}).items():
            if name in cb:
                rec["cpu_baseline"] = cb[name]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

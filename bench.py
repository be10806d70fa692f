#!/usr/bin/env python3
"""Benchmark of the DSA lightning indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the hot path over one batch: the projections
(dsa_indexer_project) and the score + top-2,048 (dsa_indexer_topk).  The
headline workload is the 8,192-token single-sequence prefill; the decode step
(64 sequences, caches of 16K..128K tokens) is measured in the same run and
reported under "decode"; the projections' share of the prefill step, timed by the
same events, under "projections".  Inputs are seeded synthetic tensors resident in HBM;
L2 is flushed (256 MB write) between timed steps, outside the timed events.

With N > 1 (torchrun), every rank runs its own independent batch (weak
scaling, no collective on the data path); times are the max over ranks.
--impl reference times the CPU oracle on a bounded sample of the same workload.
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


# ------------------------------------------------------------------------------------------ GPU arm

def _setup_prefill(d, name, seed_offset, device):
    cfg = W.WORKLOADS[name]
    wts = W.make_weights(cfg["weight_seed"])
    batch = W.make_prefill(cfg["act_seed"] + seed_offset, cfg["seq_lens"])
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    ix = d.Indexer(to(wts.W_q), to(wts.W_k), to(wts.W_w), to(wts.gamma), to(wts.beta),
                   max_tokens=max(batch.hidden.shape[0], 256))
    T = batch.hidden.shape[0]
    rows = int(batch.cache_offsets[-1])
    st = dict(ix=ix, T=T, host=batch,
              hidden=to(batch.hidden), q_latent=to(batch.q_latent), positions=to(batch.positions),
              qoff=to(batch.q_seq_offsets), coff=to(batch.cache_offsets),
              cache=torch.zeros((rows, 128), dtype=torch.bfloat16, device=device),
              q=torch.empty((T, 32, 128), dtype=torch.bfloat16, device=device),
              w=torch.empty((T, 32), dtype=torch.float32, device=device),
              idx=torch.empty((T, 2048), dtype=torch.int32, device=device),
              score=torch.empty((T, 2048), dtype=torch.float32, device=device),
              pairs=W.causal_pairs(batch.positions))
    return st


def _prefill_step(st, ev=None):
    ix = st["ix"]
    ix.project(st["hidden"], st["q_latent"], st["positions"], st["qoff"], st["cache"], st["coff"],
               q_out=st["q"], w_out=st["w"])
    if ev is not None:
        ev[0].record()
    ix.topk(st["q"], st["w"], st["positions"], st["qoff"], st["cache"], st["coff"], idx_out=st["idx"],
            score_out=st["score"])
    if ev is not None:
        ev[1].record()


def _setup_decode(d, seed_offset, device):
    cfg = W.WORKLOADS["decode_64"]
    wts = W.make_weights(cfg["weight_seed"])
    lengths = W.decode_lengths(cfg["act_seed"] + seed_offset, cfg["batch"], cfg["L_min"], cfg["L_max"])
    batch = W.make_decode(cfg["act_seed"] + seed_offset, lengths=torch.ones_like(lengths))  # new tokens only
    to = lambda t: t.to(device).contiguous()  # noqa: E731
    ix = d.Indexer(to(wts.W_q), to(wts.W_k), to(wts.W_w), to(wts.gamma), to(wts.beta), max_tokens=256)
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
    st = dict(ix=ix, T=B, hidden=to(batch.hidden), q_latent=to(batch.q_latent), positions=to(positions),
              qoff=to(torch.arange(B + 1, dtype=torch.int32)), coff=to(coff), cache=cache,
              q=torch.empty((B, 32, 128), dtype=torch.bfloat16, device=device),
              w=torch.empty((B, 32), dtype=torch.float32, device=device),
              idx=torch.empty((B, 2048), dtype=torch.int32, device=device),
              score=torch.empty((B, 2048), dtype=torch.float32, device=device),
              total_keys=total)
    # algorithmic bytes of the score + top-k: every cached key once, q/w once, indices+scores out
    st["bytes"] = total * 128 * 2 + B * (32 * 128 * 2 + 32 * 4) + B * 2048 * (4 + 4)
    return st


def _time_steps(fn, steps, flush):
    """Per-step CUDA events (L2 flushed between steps, outside the events); fn records
    its two events around the score + top-k, after the projections.  Returns the step,
    score + top-k and projection ms lists."""
    outer = []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        fn((e[1], e[2]))
        e[3].record()
        outer.append(e)
    torch.cuda.synchronize()
    return ([a[0].elapsed_time(a[3]) for a in outer], [a[1].elapsed_time(a[2]) for a in outer],
            [a[0].elapsed_time(a[1]) for a in outer])


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


def _e2e_prefill(st, steps, n_chunks=4):
    """Same metric through the public API with host buffers: every step copies the inputs in
    from pinned host memory and the indices out, in n_chunks chunks of query tokens on a copy
    stream, so that chunk c+1's inputs travel while chunk c is projected and scored (the
    chunked-prefill use of the API: each chunk's queries see the keys of every earlier chunk,
    already in the cache).  Returns (ms per step, H2D bytes, D2H bytes)."""
    h = st["host"]
    ix = st["ix"]
    T = st["T"]
    if len(h.q_seq_offsets) != 2:      # one sequence; otherwise copy and compute in one piece
        n_chunks = 1
    pin = {k: getattr(h, k).pin_memory() for k in ("hidden", "q_latent", "positions", "q_seq_offsets",
                                                    "cache_offsets")}
    out = torch.empty((T, 2048), dtype=torch.int32).pin_memory()
    bi = sum(t.numel() * t.element_size() for t in pin.values())
    bo = out.numel() * out.element_size()
    bounds = [T * c // n_chunks for c in range(n_chunks + 1)]
    dev = st["hidden"].device
    qoffs = [torch.tensor([0, bounds[c + 1] - bounds[c]], dtype=torch.int32, device=dev) for c in range(n_chunks)]
    copy = torch.cuda.Stream(device=dev)
    main = torch.cuda.current_stream(dev)
    ts = []
    for _ in range(steps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        copy.wait_stream(main)
        with torch.cuda.stream(copy):
            st["coff"].copy_(pin["cache_offsets"], non_blocking=True)
            st["qoff"].copy_(pin["q_seq_offsets"], non_blocking=True)
        arrived, done = [], []
        for c in range(n_chunks):
            a0, a1 = bounds[c], bounds[c + 1]
            with torch.cuda.stream(copy):
                st["hidden"][a0:a1].copy_(pin["hidden"][a0:a1], non_blocking=True)
                st["q_latent"][a0:a1].copy_(pin["q_latent"][a0:a1], non_blocking=True)
                st["positions"][a0:a1].copy_(pin["positions"][a0:a1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
                arrived.append(ev)
        for c in range(n_chunks):
            a0, a1 = bounds[c], bounds[c + 1]
            main.wait_event(arrived[c])
            qoff = st["qoff"] if n_chunks == 1 else qoffs[c]
            ix.project(st["hidden"][a0:a1], st["q_latent"][a0:a1], st["positions"][a0:a1], qoff, st["cache"],
                       st["coff"], q_out=st["q"][a0:a1], w_out=st["w"][a0:a1])
            ix.topk(st["q"][a0:a1], st["w"][a0:a1], st["positions"][a0:a1], qoff, st["cache"], st["coff"],
                    idx_out=st["idx"][a0:a1], score_out=st["score"][a0:a1])
            ev = torch.cuda.Event()
            ev.record(main)
            done.append(ev)
        with torch.cuda.stream(copy):
            for c in range(n_chunks):
                copy.wait_event(done[c])
                out[bounds[c]:bounds[c + 1]].copy_(st["idx"][bounds[c]:bounds[c + 1]], non_blocking=True)
        main.wait_stream(copy)
        e1.record(main)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.mean(ts), bi, bo


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

    # ---------------- prefill (headline)
    st = _setup_prefill(d, args.workload, rank, device)
    fn = lambda ev: _prefill_step(st, ev)  # noqa: E731
    _time_steps(fn, args.warmup, flush)
    barrier()
    with ClockSampler(device.index) as clk:
        clk.mark_start()
        step_ms, topk_ms, proj_ms = _time_steps(fn, args.steps, flush)
        clk.mark_end()
    barrier()
    clocks = clk.summary()
    ms = mx(statistics.mean(step_ms))
    topk_avg = mx(statistics.mean(topk_ms))
    proj_avg = mx(statistics.mean(proj_ms))
    pairs = st["pairs"]
    st_tokens = st["hidden"].shape[0]
    value = whole_job_rate(pairs, world, ms) / 1e9
    achieved_tflops = pairs * FLOP_PER_PAIR / (topk_avg * 1e-3) / 1e12
    traffic = _profile_traffic(f"score_topk:{args.workload}")
    e2e_ms, bi, bo = _e2e_prefill(st, max(2, min(args.steps, 5)))
    e2e_ms = mx(e2e_ms)
    st["ix"].device_error()

    # ---------------- decode (second half of the metric)
    dec = None
    if not args.skip_decode:
        del st
        torch.cuda.empty_cache()
        ds = _setup_decode(d, rank, device)

        def dfn(ev):
            ix = ds["ix"]
            ix.project(ds["hidden"], ds["q_latent"], ds["positions"], ds["qoff"], ds["cache"], ds["coff"],
                       q_out=ds["q"], w_out=ds["w"])
            if ev is not None:
                ev[0].record()
            ix.topk(ds["q"], ds["w"], ds["positions"], ds["qoff"], ds["cache"], ds["coff"], idx_out=ds["idx"],
                    score_out=ds["score"])
            if ev is not None:
                ev[1].record()

        _time_steps(dfn, args.warmup, flush)
        barrier()
        dstep, dtopk, _ = _time_steps(dfn, args.steps, flush)
        barrier()
        dms = mx(statistics.mean(dtopk))
        dstep_ms = mx(statistics.mean(dstep))
        gbs = ds["bytes"] / (dms * 1e-3) / 1e9
        dec = {"workload": "decode_64", "metric": "decode GB/s", "value": round(gbs * world, 2), "unit": "GB/s",
               "ms_score_topk": round(dms, 4), "ms_per_step": round(dstep_ms, 4),
               "keys_scanned": ds["total_keys"], "algorithmic_bytes": ds["bytes"],
               "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": round(gbs / peaks["hbm_gbs"], 4),
                            "traffic": _profile_traffic("score_topk:decode_64")}}
        ds["ix"].device_error()

    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "Gpairs/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) random-init weights)",
        "config": {"workload": args.workload, "batch": len(W.WORKLOADS[args.workload]["seq_lens"]),
                   "seq_len": W.WORKLOADS[args.workload]["seq_lens"][0], "heads": 32, "head_dim": 128,
                   "top_k": 2048, "causal_pairs_per_gpu": pairs, "parallelism": f"independent replicas x{world}",
                   "l2": "flushed between timed steps (256 MB write)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved_tflops, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved_tflops / peaks["bf16_tflops"], 4),
                     "traffic": traffic, "kernel": "score_topk (dsa_indexer_topk: prep + score)",
                     "ms_per_launch": round(topk_avg, 4), "peak_source": peaks["source"] + " burst bf16"},
        "e2e": {"value": round(whole_job_rate(pairs, world, e2e_ms) / 1e9, 3), "unit": "Gpairs/s",
                "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(e2e_ms, 4)},
        "projections": projection_report(st_tokens, proj_avg, peaks["bf16_tflops"], peaks["hbm_gbs"]),
        "clocks": clocks,
        "gpu_launches": args.steps * 4,
    }
    if dec is not None:
        line["decode"] = dec
    return line


# ------------------------------------------------------------------------------------------ CPU oracle arm

def cpu_oracle_sample(name, proj_tokens=256, n_rows=12, seed=0):
    """The oracle as it stands, on bounded samples of the workload: its projection
    of `proj_tokens` tokens (seconds per token) and its score + top-k of `n_rows`
    query rows spread over the positions (seconds per causal pair), extrapolated
    to the whole workload.  Returns (Gpairs/s, description, seconds spent)."""
    import numpy as np

    import oracle
    cfg = W.WORKLOADS[name]
    wts = W.make_weights(cfg["weight_seed"])
    batch = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
    T = batch.hidden.shape[0]
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    Wq, Wk, Ww, g, b = f(wts.W_q), f(wts.W_k), f(wts.W_w), f(wts.gamma), f(wts.beta)
    hid = f(batch.hidden[:proj_tokens])
    qlat = f(batch.q_latent[:proj_tokens])
    t0 = time.perf_counter()
    oracle.project(hid, qlat, Wq, Wk, Ww, g, b)
    t_proj = (time.perf_counter() - t0) / proj_tokens
    # score + top-k rows: keys = the oracle's key norm of seeded pre-norm rows (the
    # workload's key distribution), q / w of the sampled rows from the oracle projection
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(np.arange(T // 2, T), size=n_rows, replace=False))
    raw = W.make_decode(cfg["act_seed"], lengths=[T]).raw_keys
    keys = oracle.key_norm(raw.to(torch.float64).numpy(), g, b)
    q, _, w = oracle.project(f(batch.hidden[rows]), f(batch.q_latent[rows]), Wq, Wk, Ww, g, b)
    qq = np.zeros((T, 32, 128))
    ww = np.zeros((T, 32))
    qq[rows] = q
    ww[rows] = w
    t0 = time.perf_counter()
    oracle.topk(qq, ww, batch.positions.numpy(), batch.q_seq_offsets.numpy(), keys, np.array([0, T]), rows=rows)
    t_topk = time.perf_counter() - t0
    pairs_s = int((batch.positions[rows].to(torch.int64) + 1).sum())
    total_pairs = W.causal_pairs(batch.positions)
    t_full = T * t_proj + total_pairs * (t_topk / pairs_s)
    desc = (f"{name}: projection of {proj_tokens} tokens ({t_proj * 1e3:.2f} ms/token) and score+top-k of "
            f"{n_rows} query rows ({pairs_s} causal pairs, {t_topk:.2f} s), extrapolated to all {T} tokens "
            f"/ {total_pairs} pairs ({t_full:.0f} s)")
    return total_pairs / t_full / 1e9, desc, t_proj * proj_tokens + t_topk


def reference_arm(args):
    vals = []
    desc = ""
    for _ in range(min(args.warmup, 1)):
        cpu_oracle_sample(args.workload, proj_tokens=32, n_rows=2)
    wall = 0.0
    for i in range(args.steps):
        v, desc, spent = cpu_oracle_sample(args.workload, seed=i)
        vals.append(v)
        wall += spent
    value = statistics.mean(vals)
    cores = _cpu_threads()
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
        "config": {"workload": args.workload, "batch": len(W.WORKLOADS[args.workload]["seq_lens"]),
                   "seq_len": W.WORKLOADS[args.workload]["seq_lens"][0], "top_k": 2048},
        "cpu_baseline": {"value": float(f"{value:.6g}"), "unit": "Gpairs/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": float(f"{value:.6g}"), "unit": "Gpairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_8k", choices=["prefill_3k", "prefill_8k", "prefill_2x32k_heavy"])
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
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
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    line = gpu_arm(args, rank, world, local_rank, dist)
    if rank == 0 and not args.no_cpu_baseline:
        v, desc, _ = cpu_oracle_sample(args.workload)
        line["cpu_baseline"] = {"value": float(f"{v:.6g}"), "unit": "Gpairs/s", "cores": _cpu_threads(), "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

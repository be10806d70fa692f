"""Parity at the full workload sizes, in the launch configuration the benchmark times
(dsa_indexer_project then dsa_indexer_topk with default flags): every output row is
checked for the properties that hold at any size (indices inside the causal prefix,
no duplicates, exact padding, valid entries first), and sampled rows are compared
with the oracle, which scores them one by one.

The oracle takes the queries, weights and keys either from the raw inputs (end to
end, prefill_8k) or from the GPU's own projections after those have been checked on
sampled tokens (the larger workloads, where projecting every token in float64 would
take minutes)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import assert_proj_close, check_topk, f64, oracle_project

pytestmark = pytest.mark.gpu

TOP_K = 2048


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dsa_lightning_indexer_03_b200 import build
    build.build()
    import dsa_lightning_indexer_03_b200 as d
    return d


def _cuda(t):
    return t.to("cuda").contiguous()


def _indexer(d, wts, max_tokens):
    return d.Indexer(_cuda(wts.W_q), _cuda(wts.W_k), _cuda(wts.W_w), _cuda(wts.gamma), _cuda(wts.beta),
                     max_tokens=max_tokens)


def check_rows_valid(idx: torch.Tensor, positions: torch.Tensor):
    """Properties of every row that hold at any size (bit-exact)."""
    pos = positions.to(torch.int64).unsqueeze(1)
    n_valid = torch.clamp(pos + 1, max=TOP_K).squeeze(1)
    valid = idx >= 0
    assert torch.equal(valid.sum(1), n_valid), "number of valid entries per row"
    col = torch.arange(TOP_K, device=idx.device).unsqueeze(0)
    assert torch.equal(valid, col < n_valid.unsqueeze(1)), "valid entries must come first"
    assert bool(((idx <= pos) | ~valid).all()), "index outside the causal prefix"
    short = (pos.squeeze(1) + 1) <= TOP_K
    if bool(short.any()):
        rows = idx[short]
        exp = torch.where(col < n_valid[short].unsqueeze(1), col, torch.full_like(col, -1))
        assert torch.equal(rows.to(torch.int64), exp.expand_as(rows)), "short-prefix rows must be [0..p, -1...]"
    srt = torch.sort(idx, dim=1).values
    dup = (srt[:, 1:] == srt[:, :-1]) & (srt[:, 1:] >= 0)
    assert not bool(dup.any()), "duplicate index in a row"


def oracle_rows(q_rows, w_rows, pos_rows, seq_rows, keys_f64, cache_offsets):
    """Oracle top-k of sampled rows (sorted by sequence) against a float64 key cache."""
    seq_rows = np.asarray(seq_rows, np.int64)
    B = len(cache_offsets) - 1
    qoff = np.zeros(B + 1, np.int64)
    qoff[1:] = np.cumsum(np.bincount(seq_rows, minlength=B))
    return oracle.topk(q_rows, w_rows, pos_rows, qoff, keys_f64, cache_offsets, TOP_K,
                       keep_scores=True)


def sample_rows(T, n, must=()):
    rng = np.random.default_rng(12345 + T)
    rows = np.unique(np.concatenate([rng.choice(T, size=min(n, T), replace=False), np.asarray(must, np.int64)]))
    return rows[(rows >= 0) & (rows < T)]


def test_prefill_8k_end_to_end(dsa):
    cfg = W.WORKLOADS["prefill_8k"]
    wts = W.make_weights(cfg["weight_seed"])
    batch = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
    T = batch.hidden.shape[0]
    ix = _indexer(dsa, wts, T)
    cache = torch.zeros((int(batch.cache_offsets[-1]), 128), dtype=torch.bfloat16, device="cuda")
    pos, qoff, coff = _cuda(batch.positions), _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, cache, coff)
    idx, sc = ix.topk(q, w, pos, qoff, cache, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    check_rows_valid(idx, pos)
    keys = oracle.project_keys(f64(batch.hidden), f64(wts.W_k), f64(wts.gamma), f64(wts.beta))
    assert_proj_close(f64(cache), keys, "k")
    rows = W.stratified_rows(batch.q_seq_offsets, 256, seed=1, positions=batch.positions).numpy()
    oq, _, ow = oracle_project(wts, batch.hidden[rows], batch.q_latent[rows])
    assert_proj_close(f64(q[rows]).reshape(len(rows), -1), oq.reshape(len(rows), -1), "q")
    assert_proj_close(f64(w[rows]), ow, "w")
    _, _, I, A = oracle_rows(oq, ow, batch.positions.numpy()[rows], np.zeros(len(rows)), keys,
                             batch.cache_offsets.numpy())
    recall, _ = check_topk(idx[rows].cpu().numpy(), sc[rows].cpu().numpy(), rows, batch.positions.numpy()[rows],
                           I, A)
    print(f"prefill_8k end to end: {len(rows)} stratified rows against the oracle, recall {recall:.6f}")


def test_prefill_2x32k_heavy(dsa):
    cfg = W.WORKLOADS["prefill_2x32k_heavy"]
    wts = W.make_weights(cfg["weight_seed"])
    batch = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
    T = batch.hidden.shape[0]
    ix = _indexer(dsa, wts, T)
    cache = torch.zeros((int(batch.cache_offsets[-1]), 128), dtype=torch.bfloat16, device="cuda")
    pos, qoff, coff = _cuda(batch.positions), _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, cache, coff)
    heavy = W.heavy_hitter_rows(cfg["act_seed"], batch.cache_offsets)
    cache[_cuda(heavy)] *= 4   # exact in bf16
    idx, sc = ix.topk(q, w, pos, qoff, cache, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    check_rows_valid(idx, pos)
    strat = W.stratified_rows(batch.q_seq_offsets, 128, seed=2, positions=batch.positions).numpy()
    # and 128 rows whose selection holds heavy-hitter keys (the x4 rows)
    seq_all = oracle.sequence_of(batch.q_seq_offsets.numpy(), T)
    heavy_pos = torch.zeros(int(batch.cache_offsets[-1]), dtype=torch.bool, device="cuda")
    heavy_pos[_cuda(heavy)] = True
    base = _cuda(batch.cache_offsets[torch.as_tensor(seq_all)]).unsqueeze(1)
    sel_rows = (idx.to(torch.int64) + base).clamp(min=0)
    has_heavy = (heavy_pos[sel_rows] & (idx >= 0)).any(1).cpu().numpy()
    cand = np.setdiff1d(np.nonzero(has_heavy)[0], strat)
    rng = np.random.default_rng(3)
    hh = rng.choice(cand, size=min(128, len(cand)), replace=False)
    rows = np.unique(np.concatenate([strat, hh]))
    assert len(hh) == 128, "at least 128 queries select heavy-hitter keys"
    oq, ok_, ow = oracle_project(wts, batch.hidden[rows], batch.q_latent[rows])
    # projections of the sampled tokens (their key rows, before the heavy-hitter scaling)
    kr = f64(cache[_cuda(torch.as_tensor(rows))])
    scale = np.where(np.isin(rows, heavy.numpy()), 4.0, 1.0)[:, None]
    assert_proj_close(kr / scale, ok_, "k")
    assert_proj_close(f64(q[rows]).reshape(len(rows), -1), oq.reshape(len(rows), -1), "q")
    assert_proj_close(f64(w[rows]), ow, "w")
    # selection of the sampled rows, oracle-fed with the GPU's keys (checked above) and q, w
    seq = oracle.sequence_of(batch.q_seq_offsets.numpy(), T)[rows]
    _, _, I, A = oracle_rows(f64(q[rows]), f64(w[rows]), batch.positions.numpy()[rows], seq, f64(cache),
                             batch.cache_offsets.numpy())
    recall, _ = check_topk(idx[rows].cpu().numpy(), sc[rows].cpu().numpy(), rows, batch.positions.numpy()[rows],
                           I, A)
    print(f"prefill_2x32k_heavy: {len(rows)} rows ({len(hh)} selecting heavy hitters) against the oracle, "
          f"recall {recall:.6f}")


def test_decode_64(dsa):
    cfg = W.WORKLOADS["decode_64"]
    wts = W.make_weights(cfg["weight_seed"])
    lengths = W.decode_lengths(cfg["act_seed"], cfg["batch"], cfg["L_min"], cfg["L_max"])
    batch = W.make_decode(cfg["act_seed"], lengths=torch.ones_like(lengths))   # the 64 new tokens' inputs
    B = cfg["batch"]
    total = int(lengths.sum())
    coff = torch.zeros(B + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(lengths, 0)
    ix = _indexer(dsa, wts, 256)
    gd = torch.Generator(device="cuda").manual_seed(2000)
    cache = torch.empty((total, 128), dtype=torch.bfloat16, device="cuda")
    raw_sample = {}
    step = 1 << 20
    check_at = sample_rows(total, 64)
    for s0 in range(0, total, step):
        n = min(step, total - s0)
        raw = torch.randn((n, 128), generator=gd, device="cuda", dtype=torch.float32)
        ix.key_norm(raw, out=cache[s0:s0 + n])
        sel = check_at[(check_at >= s0) & (check_at < s0 + n)]
        if len(sel):
            raw_sample.update(zip(sel.tolist(), raw[_cuda(torch.as_tensor(sel - s0))].cpu()))
    positions = (lengths - 1).to(torch.int32)
    qoff = torch.arange(B + 1, dtype=torch.int32)
    # the new tokens' own keys go to the last row of each cache, as project writes them
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), _cuda(positions), _cuda(qoff), cache, _cuda(coff))
    idx, sc = ix.topk(q, w, _cuda(positions), _cuda(qoff), cache, _cuda(coff))
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    check_rows_valid(idx, _cuda(positions))
    last = (coff[1:] - 1).numpy()
    kr = np.stack([raw_sample[r].numpy() for r in check_at if r not in set(last.tolist())])
    rows_k = np.array([r for r in check_at if r not in set(last.tolist())])
    assert_proj_close(f64(cache[_cuda(torch.as_tensor(rows_k))]),
                      oracle.key_norm(kr.astype(np.float64), f64(wts.gamma), f64(wts.beta)), "cached k")
    oq, ok_, ow = oracle_project(wts, batch.hidden, batch.q_latent)
    assert_proj_close(f64(q).reshape(B, -1), oq.reshape(B, -1), "q")
    assert_proj_close(f64(w), ow, "w")
    assert_proj_close(f64(cache[_cuda(torch.as_tensor(last))]), ok_, "new k")
    rows = np.arange(B)
    I, A = [], []
    for b in rows:   # one sequence's cache at a time (the whole cache in float64 would be ~5 GB)
        lo, hi = int(coff[b]), int(coff[b + 1])
        _, _, Ib, Ab = oracle_rows(f64(q[b:b + 1]), f64(w[b:b + 1]), positions.numpy()[b:b + 1], [0],
                                   f64(cache[lo:hi]), np.array([0, hi - lo]))
        I += Ib
        A += Ab
    recall, _ = check_topk(idx[rows].cpu().numpy(), sc[rows].cpu().numpy(), rows, positions.numpy()[rows], I, A)
    print(f"decode_64: all {B} rows against the oracle, recall {recall:.6f}")


def test_chunked_128k(dsa):
    cfg = W.WORKLOADS["chunked_128k"]
    wts = W.make_weights(cfg["weight_seed"])
    S, C = cfg["seq_len"], cfg["chunk"]
    ix = _indexer(dsa, wts, C)
    cache = torch.zeros((S, 128), dtype=torch.bfloat16, device="cuda")
    coff = _cuda(torch.tensor([0, S], dtype=torch.int64))
    qoff = _cuda(torch.tensor([0, C], dtype=torch.int32))
    keep = {}
    for c in range(S // C):
        batch = W.make_prefill(cfg["act_seed"], [C], start_positions=[c * C], cache_lens=[S], sub=c)
        pos = _cuda(batch.positions)
        q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, cache, coff)
        idx, sc = ix.topk(q, w, pos, qoff, cache, coff)
        torch.cuda.synchronize()
        assert ix.device_error() == dsa.DSA_OK
        check_rows_valid(idx, pos)
        rows = W.stratified_rows(torch.tensor([0, C]), 32, seed=100 + c, positions=batch.positions).numpy()
        keep[c] = (batch, rows, q[rows].cpu(), w[rows].cpu(), idx[rows].cpu(), sc[rows].cpu())
    keys = f64(cache)
    n_rows, recalls = 0, []
    for c, (batch, rows, qs, ws, ids, scs) in keep.items():
        assert 0 in rows and C - 1 in rows and len(rows) >= 32
        oq, ok_, ow = oracle_project(wts, batch.hidden[rows], batch.q_latent[rows])
        assert_proj_close(f64(qs).reshape(len(rows), -1), oq.reshape(len(rows), -1), f"chunk {c} q")
        assert_proj_close(f64(ws), ow, f"chunk {c} w")
        assert_proj_close(f64(cache[_cuda(torch.as_tensor(c * C + rows))]), ok_, f"chunk {c} k")
        pos_rows = batch.positions.numpy()[rows]
        _, _, I, A = oracle_rows(f64(qs), f64(ws), pos_rows, np.zeros(len(rows)), keys, np.array([0, S]))
        recall, _ = check_topk(ids.numpy(), scs.numpy(), c * C + rows, pos_rows, I, A)
        n_rows += len(rows)
        recalls.append(recall)
    print(f"chunked_128k: {n_rows} rows (every chunk, its first and last included) against the oracle, "
          f"recall min {min(recalls):.6f} mean {np.mean(recalls):.6f}")

"""CUDA path vs the CPU oracle on the same seeded inputs, through the C ABI.

Every test here needs a B200 and the built library (marked gpu)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import (assert_proj_close, check_sorted, check_topk, f64, oracle_project, oracle_topk_rows)

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


def _indexer(d, wts, max_tokens=16384, eps=1e-6):
    return d.Indexer(_cuda(wts.W_q), _cuda(wts.W_k), _cuda(wts.W_w), _cuda(wts.gamma), _cuda(wts.beta),
                     ln_eps=eps, max_tokens=max_tokens)


def _offsets(lens, dtype):
    o = torch.zeros(len(lens) + 1, dtype=dtype)
    o[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(dtype)
    return o


# ------------------------------------------------------------------------------------------ projections

def test_projections_match_oracle(dsa):
    wts = W.make_weights(11)
    batch = W.make_prefill(12, [170, 130], start_positions=[0, 40], cache_lens=[200, 180])
    ix = _indexer(dsa, wts)
    cache_rows = int(batch.cache_offsets[-1])
    sentinel = torch.full((cache_rows + 5, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), _cuda(batch.positions),
                      _cuda(batch.q_seq_offsets), sentinel, _cuda(batch.cache_offsets))
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    oq, ok_, ow = oracle_project(wts, batch.hidden, batch.q_latent)
    assert_proj_close(f64(q).reshape(len(oq), -1), oq.reshape(len(oq), -1), "q")
    assert_proj_close(f64(w), ow, "w")
    cache = f64(sentinel)
    written = np.zeros(cache.shape[0], bool)
    offs = batch.cache_offsets.tolist()
    seq = oracle.sequence_of(batch.q_seq_offsets.numpy(), len(oq))
    rows = [offs[seq[t]] + int(batch.positions[t]) for t in range(len(oq))]
    written[rows] = True
    assert_proj_close(cache[rows], ok_, "k")
    assert np.all(np.isnan(cache[~written])), "rows no token owns must stay untouched"


def test_key_norm_matches_oracle(dsa):
    wts = W.make_weights(13)
    raw = W.make_decode(14, lengths=[700, 300]).raw_keys
    ix = _indexer(dsa, wts)
    out = ix.key_norm(_cuda(raw))
    torch.cuda.synchronize()
    ref = oracle.key_norm(f64(raw), f64(wts.gamma), f64(wts.beta), 1e-6)
    assert_proj_close(f64(out), ref, "key_norm")


# ------------------------------------------------------------------------------------------ score + top-k (oracle-fed)

def _run_topk(d, ix, q, w, positions, qoff, keys, coff, flags=0):
    idx, sc = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff), flags=flags)
    torch.cuda.synchronize()
    assert ix.device_error() == d.DSA_OK
    return idx.cpu().numpy(), sc.cpu().numpy()


def _oracle_rows(q, w, positions, qoff, keys, coff, rows):
    return oracle_topk_rows(f64(q), f64(w), positions.numpy(), qoff.numpy(), f64(keys), coff.numpy(), rows)


@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 2047, 2048, 2049, 3000])
@pytest.mark.parametrize("flags", [0, 4])
def test_topk_single_sequence(dsa, T, flags):
    wts = W.make_weights(1, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    q, keys, w = W.make_scoring_inputs(100 + T, T, T)
    positions = torch.arange(T, dtype=torch.int32)
    qoff = _offsets([T], torch.int32)
    coff = _offsets([T], torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, flags)
    rows = np.arange(T) if T <= 600 else np.unique(np.concatenate([np.arange(0, T, 7), [T - 1, 2046, 2047, 2048]]))
    rows = rows[rows < T]
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)


@pytest.mark.parametrize("flags", [0, 2, 4])
def test_topk_ragged_batch(dsa, flags):
    lens = [1000, 2100, 37, 1, 2600]
    T = sum(lens)
    if flags == 2 and T > 256:
        lens = [100, 60, 1, 90]
        T = sum(lens)
    wts = W.make_weights(2, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    q, keys, w = W.make_scoring_inputs(7, T, T)
    positions = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
    qoff = _offsets(lens, torch.int32)
    coff = _offsets(lens, torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, flags)
    rows = np.arange(T) if T <= 400 else np.arange(0, T, 5)
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)


@pytest.mark.parametrize("flags", [0, 2])
def test_topk_decode_like_long_prefixes(dsa, flags):
    # one query per sequence at the end of its cache; lengths span 1..3 key chunks
    lens = [5000, 9000, 20000, 40000, 2048, 2049, 130]
    B = len(lens)
    wts = W.make_weights(3, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    q, keys, w = W.make_scoring_inputs(8, B, sum(lens))
    positions = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
    qoff = torch.arange(B + 1, dtype=torch.int32)
    coff = _offsets(lens, torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, flags)
    rows = np.arange(B)
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi, gs, rows, positions.numpy(), I, A)


def test_topk_chunk_with_offset_positions(dsa):
    # a chunk of 1000 queries at positions 4000..4999 of a 6000-row cache
    wts = W.make_weights(4, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    T, S = 1000, 6000
    q, keys, w = W.make_scoring_inputs(9, T, S)
    positions = torch.arange(4000, 5000, dtype=torch.int32)
    qoff = _offsets([T], torch.int32)
    coff = _offsets([S], torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, 4)
    rows = np.arange(0, T, 9)
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)


def test_topk_all_scores_tied(dsa):
    # w = 0: every score is 0, any 2048 of the prefix is a correct answer
    wts = W.make_weights(5, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    T = 2600
    q, keys, _ = W.make_scoring_inputs(10, T, T)
    w = torch.zeros(T, 32)
    positions = torch.arange(T, dtype=torch.int32)
    qoff = _offsets([T], torch.int32)
    coff = _offsets([T], torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, 4)
    rows = np.array([0, 5, 2047, 2048, 2500, T - 1])
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A, min_recall=None)


def test_topk_without_scores(dsa):
    wts = W.make_weights(6, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    T = 2300
    q, keys, w = W.make_scoring_inputs(11, T, T)
    positions = torch.arange(T, dtype=torch.int32)
    qoff = _offsets([T], torch.int32)
    coff = _offsets([T], torch.int64)
    idx, sc = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff),
                      return_scores=False)
    torch.cuda.synchronize()
    assert sc is None
    ref_idx, _ = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff))
    a = np.sort(idx.cpu().numpy(), axis=1)
    b = np.sort(ref_idx.cpu().numpy(), axis=1)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("flags", [1, 1 | 2, 1 | 4])
def test_topk_sorted_rows(dsa, flags):
    # DSA_TOPK_SORTED on the prefill path (default / NO_SPLIT) and on the split-key path, with
    # queries whose prefix is shorter and longer than 2,048; with and without score output
    if flags & 2:
        lens = [5000, 9000, 40000, 2048, 2049, 130]
        B = len(lens)
        q, keys, w = W.make_scoring_inputs(21, B, sum(lens))
        positions = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
        qoff = torch.arange(B + 1, dtype=torch.int32)
    else:
        lens = [3000, 37, 2600]
        B = len(lens)
        q, keys, w = W.make_scoring_inputs(22, sum(lens), sum(lens))
        positions = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
        qoff = _offsets(lens, torch.int32)
    wts = W.make_weights(9, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    coff = _offsets(lens, torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, flags)
    T = gi.shape[0]
    rows = np.arange(T) if T <= 64 else np.unique(np.concatenate([np.arange(0, T, 11), [2046, 2047, 2048, T - 1]]))
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, rows)
    check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)
    open_pairs = check_sorted(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)
    # without scores the order is the same (the sort key is the kernel's own score)
    idx2, _ = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff),
                      return_scores=False, flags=flags)
    torch.cuda.synchronize()
    assert np.array_equal(idx2.cpu().numpy(), gi)
    print(f"sorted rows flags={flags}: {len(rows)} rows, {open_pairs} neighbour pairs inside the band")


def test_malformed_offsets_pad_every_row(dsa):
    wts = W.make_weights(10, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    T = 200
    q, keys, w = W.make_scoring_inputs(23, T, T)
    positions = torch.arange(T, dtype=torch.int32)
    qoff = torch.tensor([0, 150, 100, T], dtype=torch.int32)    # not monotone
    coff = torch.tensor([0, 100, 150, T], dtype=torch.int64)
    for flags in (0, 2):
        idx, sc = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff), flags=flags)
        torch.cuda.synchronize()
        assert ix.device_error() == dsa.DSA_ERR_DEVICE_BOUNDS
        assert bool((idx == -1).all()) and bool(torch.isneginf(sc).all())


def test_topk_reuse_for_draft_steps(dsa):
    # first step: 6 anchor queries selected by dsa_indexer_topk (checked against the oracle);
    # draft steps: 14 tokens that reuse an anchor's row, one with an anchor out of range
    wts = W.make_weights(12, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    lens = [3000, 5000, 2100, 700, 9000, 4096]
    B = len(lens)
    q, keys, w = W.make_scoring_inputs(24, B, sum(lens))
    positions = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
    qoff = torch.arange(B + 1, dtype=torch.int32)
    coff = _offsets(lens, torch.int64)
    gi, gs = _run_topk(dsa, ix, q, w, positions, qoff, keys, coff, 0)
    _, _, I, A = _oracle_rows(q, w, positions, qoff, keys, coff, np.arange(B))
    check_topk(gi, gs, np.arange(B), positions.numpy(), I, A)
    anchors = torch.tensor([0, 0, 0, 1, 1, 2, 3, 3, 3, 3, 4, 5, 5, 5], dtype=torch.int32)
    anchors[7] = 17   # no such anchor: a padding row and a bounds report
    src_i, src_s = _cuda(torch.from_numpy(gi)), _cuda(torch.from_numpy(gs))
    ri, rs = ix.topk_reuse(_cuda(anchors), src_i, src_s)
    ri2, rs2 = ix.topk_reuse(_cuda(anchors), src_i)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_ERR_DEVICE_BOUNDS
    oi, os_ = oracle.reuse_topk(gi, gs, anchors.numpy())
    assert np.array_equal(ri.cpu().numpy(), oi) and np.array_equal(ri2.cpu().numpy(), oi)
    assert rs2 is None
    got_s = rs.cpu().numpy()
    assert np.array_equal(got_s[np.isfinite(os_)], os_[np.isfinite(os_)])
    assert np.all(np.isneginf(got_s[~np.isfinite(os_)]))


# ------------------------------------------------------------------------------------------ end to end

def test_end_to_end_prefill_3k(dsa):
    cfg = W.WORKLOADS["prefill_3k"]
    wts = W.make_weights(cfg["weight_seed"])
    batch = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
    T = batch.hidden.shape[0]
    ix = _indexer(dsa, wts)
    cache = torch.zeros((int(batch.cache_offsets[-1]), 128), dtype=torch.bfloat16, device="cuda")
    pos, qoff, coff = _cuda(batch.positions), _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, cache, coff)
    idx, sc = ix.topk(q, w, pos, qoff, cache, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    oq, ok_, ow = oracle_project(wts, batch.hidden, batch.q_latent)
    assert_proj_close(f64(q).reshape(T, -1), oq.reshape(T, -1), "q")
    assert_proj_close(f64(w), ow, "w")
    assert_proj_close(f64(cache), ok_, "k")
    rows = np.arange(T)
    _, _, I, A = oracle.topk(oq, ow, batch.positions.numpy(), batch.q_seq_offsets.numpy(), ok_,
                             batch.cache_offsets.numpy(), TOP_K, rows=rows, keep_scores=True)
    recall, _ = check_topk(idx.cpu().numpy(), sc.cpu().numpy(), rows, batch.positions.numpy(), I, A)
    print(f"prefill_3k end-to-end recall {recall:.6f}")


# ------------------------------------------------------------------------------------------ errors

def test_bad_position_is_reported_and_padded(dsa):
    wts = W.make_weights(7, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    T = 300
    q, keys, w = W.make_scoring_inputs(12, T, T)
    positions = torch.arange(T, dtype=torch.int32)
    positions[17] = T + 5       # outside its sequence's cache rows
    positions[18] = -3
    qoff = _offsets([T], torch.int32)
    coff = _offsets([T], torch.int64)
    idx, sc = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff))
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_ERR_DEVICE_BOUNDS
    assert ix.device_error() == dsa.DSA_OK   # cleared by the read
    gi = idx.cpu().numpy()
    assert np.all(gi[17] == -1) and np.all(gi[18] == -1)
    assert np.all(np.isneginf(sc.cpu().numpy()[17]))
    assert np.array_equal(gi[16, :17], np.arange(17))


def test_host_argument_errors(dsa):
    wts = W.make_weights(8, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts, max_tokens=64)
    q, keys, w = W.make_scoring_inputs(13, 100, 100)
    positions = torch.arange(100, dtype=torch.int32)
    qoff = _offsets([100], torch.int32)
    coff = _offsets([100], torch.int64)
    with pytest.raises(dsa.DSAError) as e:   # T > max_tokens
        ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff))
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
    qc = _cuda(q)[:10]
    buf = torch.empty(10 * 32 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    mis = buf[1:1 + 10 * 32 * 128].view(10, 32, 128)   # 2-byte offset: not 16-byte aligned
    mis.copy_(qc)
    with pytest.raises(dsa.DSAError) as e:
        ix.topk(mis, _cuda(w)[:10], _cuda(positions)[:10], _cuda(_offsets([10], torch.int32)), _cuda(keys),
                _cuda(coff))
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    with pytest.raises(dsa.DSAError) as e:
        ix.topk(qc, _cuda(w)[:10], _cuda(positions)[:10], _cuda(_offsets([10], torch.int32)), _cuda(keys),
                _cuda(coff), flags=1 | 2 | 4)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG


def test_bounded_wait_reports_timeout(dsa):
    # a kernel waits on a barrier nothing signals; its 20 ms limit must end the wait
    assert dsa.selftest_wait_timeout(20_000_000) == dsa.DSA_ERR_DEVICE_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0   # the context is still usable

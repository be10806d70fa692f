"""Sparse MLA attention over the indexer's selection ('Latent attention (MLA)' row of the pages
"Qwen3.5-397B-A17B vs Kimi K3.1 Pro" and "Kimi K3.1 Pro vs Gemma 4 31B": 96 heads, 576 cached
values per token, 2,048 selected tokens per query) against the oracle, through the C ABI.

Tolerance, from the kernel's arithmetic.  Scores are fp32 sums of 576 exact bf16 products:
their error is allowed e_s = 6 sqrt(576) 2^-24 scale |q_h| max_j |row_j| (a six-sigma
random-walk bound of the rounding).  The softmax weights enter P.V as bf16 (relative error
<= U = 2^-8 each) and the same rounded weights make up the normaliser, so o moves by at most
(U + e_s) max_j |v_j - o| per value; o is then rounded to bf16 (<= U |o|).  So, per value,
|o - o_ref| <= 1.01 U (spread + |o_ref|) + e_s spread + 1e-5, with spread = max_j |v_jd - o_d|
over the query's selected rows, and |lse - lse_ref| <= 1.01 U + e_s + 1e-5."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import f64, mla_tolerances

pytestmark = pytest.mark.gpu

U = 2.0 ** -8            # unit roundoff of bf16
SCALE = 1.0 / np.sqrt(192.0)


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dsa_lightning_indexer_03_b200 import build
    build.build()
    import dsa_lightning_indexer_03_b200 as d
    return d


@pytest.fixture(scope="module")
def ix(dsa):
    wts = W.make_weights(41, hidden_dim=256, q_latent_dim=128)
    return dsa.Indexer(*(t.to("cuda").contiguous() for t in (wts.W_q, wts.W_k, wts.W_w, wts.gamma, wts.beta)),
                       max_tokens=4096)


def _run(dsa, ix, batch, scale=SCALE, expect=None):
    dev = "cuda"
    o, lse = ix.sparse_mla(batch.q.to(dev), batch.kv.to(dev), batch.cache_offsets.to(dev),
                           batch.q_seq_offsets.to(dev), batch.idx.to(dev), scale)
    torch.cuda.synchronize()
    assert ix.device_error() == (dsa.DSA_OK if expect is None else expect)
    return f64(o.cpu()), lse.cpu().numpy().astype(np.float64)


def _selected_rows(batch, t):
    """The cache rows query t selects (valid entries only), float64."""
    qo, co = batch.q_seq_offsets.numpy(), batch.cache_offsets.numpy()
    b = int(np.searchsorted(qo, t, side="right") - 1)
    sel = batch.idx[t].to(torch.int64)
    sel = sel[(sel >= 0) & (sel < int(co[b + 1] - co[b]))]
    return f64(batch.kv[int(co[b]) + sel.to(batch.kv.device)])


def _tolerances(q_t, rows, o_ref_t, scale=SCALE):
    """Per-value bound on |o - o_ref| and per-head bound on |lse - lse_ref| of one query."""
    return mla_tolerances(q_t, rows, o_ref_t, scale)


def _ref(batch, scale=SCALE, rows=None):
    """The oracle's o and lse of every query (or of the sampled `rows`, each as a sequence of its
    own), with the tolerances of each."""
    qo = batch.q_seq_offsets.numpy()
    co = batch.cache_offsets.numpy()
    ts = range(batch.q.shape[0]) if rows is None else [int(r) for r in rows]
    o, lse, ot, lt = [], [], [], []
    kv_all = f64(batch.kv) if rows is None else None
    if rows is None:
        o_all, lse_all = oracle.sparse_mla(f64(batch.q), kv_all, co, qo, batch.idx.numpy(), scale)
    for i, t in enumerate(ts):
        q_t = f64(batch.q[t])
        if rows is None:
            oo, ll = o_all[t], lse_all[t]
        else:
            b = int(np.searchsorted(qo, t, side="right") - 1)
            kv_b = f64(batch.kv[int(co[b]):int(co[b + 1])])
            oo, ll = oracle.sparse_mla(q_t[None], kv_b, np.array([0, kv_b.shape[0]]), np.array([0, 1]),
                                       batch.idx.numpy()[t:t + 1], scale)
            oo, ll = oo[0], ll[0]
        a, c = _tolerances(q_t, _selected_rows(batch, t), oo, scale)
        o.append(oo)
        lse.append(ll)
        ot.append(a)
        lt.append(c)
    return np.stack(o), np.stack(lse), np.stack(ot), np.stack(lt)


def _check(o, lse, o_ref, lse_ref, o_tol, lse_tol):
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    d = np.abs(lse[fin] - lse_ref[fin])
    assert np.all(d <= lse_tol[fin]), d.max()
    err = np.abs(o - o_ref)
    assert np.all(err <= o_tol), (err.max(), (err / o_tol).max())


def test_sparse_mla_ragged_tiles_and_padding(dsa, ix):
    # 100 selected entries = three full 32-token tiles and a ragged tail of 4; some rows
    # padded with -1, two sequences, all 96 heads
    batch = W.make_mla(1, [700, 90], [3, 2], k_sel=100, pad=7)
    o, lse = _run(dsa, ix, batch)
    _check(o, lse, *_ref(batch))


def test_sparse_mla_full_selection_fewer_heads(dsa, ix):
    batch = W.make_mla(2, [5000, 2600, 1500], [2, 1, 2], n_heads=16, k_sel=2048)
    o, lse = _run(dsa, ix, batch)
    _check(o, lse, *_ref(batch))


def test_sparse_mla_peaked_scores_rescale(dsa, ix):
    # q of std 4: score spreads of tens of units, so the running maximum rises often by more
    # than the kernel's rescale threshold
    batch = W.make_mla(3, [4096], [4], n_heads=96, k_sel=2048, q_std=4.0)
    o, lse = _run(dsa, ix, batch)
    _check(o, lse, *_ref(batch))
    batch = W.make_mla(4, [3000], [2], n_heads=40, k_sel=2048, q_std=12.0)
    o, lse = _run(dsa, ix, batch)
    _check(o, lse, *_ref(batch))


def test_sparse_mla_uniform_weights_give_the_mean(dsa, ix):
    # q = 0: every score is 0, each weight is exactly 1 / n, o is the mean of the selected
    # latents (fp32 sum, then one bf16 rounding) and lse = ln n.  A token dropped, doubled or
    # read from a wrong row moves o by about |v - o| / n, far above this bound.
    batch = W.make_mla(9, [3000, 1200], [2, 2], n_heads=24, k_sel=2048, pad=37)
    batch.q.zero_()
    batch.idx[3, 5:9] = batch.idx[3, 100]
    o, lse = _run(dsa, ix, batch)
    o_ref, lse_ref, _, _ = _ref(batch)
    assert np.all(np.abs(o - o_ref) <= 1.01 * U * np.abs(o_ref) + 2e-5)
    n = (batch.idx.numpy() >= 0).sum(axis=1)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(n)[:, None], lse.shape), rtol=0, atol=1e-5)


def test_sparse_mla_duplicates_and_empty_rows(dsa, ix):
    batch = W.make_mla(5, [300], [4], n_heads=8, k_sel=64)
    batch.idx[0, :] = -1                         # no token: o = 0, lse = -inf
    batch.idx[1, 10:20] = batch.idx[1, 0]        # one token ten more times
    batch.idx[2, :] = -1
    batch.idx[2, 63] = 7                         # a single token, in the last tile's last slot
    o, lse = _run(dsa, ix, batch)
    o_ref, lse_ref, o_tol, lse_tol = _ref(batch)
    _check(o, lse, o_ref, lse_ref, o_tol, lse_tol)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    # one token: o is that token's latent, exactly (weight 1, bf16 value)
    np.testing.assert_array_equal(o[2], np.broadcast_to(f64(batch.kv[7, :512]), (8, 512)))


def test_sparse_mla_zero_selected_and_bounds(dsa, ix):
    batch = W.make_mla(6, [200, 150], [1, 1], n_heads=4, k_sel=0)
    o, lse = _run(dsa, ix, batch)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    # an entry past its sequence's rows is skipped and reported
    batch = W.make_mla(7, [200, 150], [1, 1], n_heads=4, k_sel=40)
    bad = batch.idx.clone()
    bad[1, 3] = 150                              # sequence 1 holds positions 0..149
    good = batch.idx.clone()
    good[1, 3] = -1
    o, lse = _run(dsa, ix, W.MlaBatch(batch.q, batch.kv, batch.cache_offsets, batch.q_seq_offsets, bad),
                  expect=dsa.DSA_ERR_DEVICE_BOUNDS)
    _check(o, lse, *_ref(W.MlaBatch(batch.q, batch.kv, batch.cache_offsets, batch.q_seq_offsets, good)))


def test_sparse_mla_consumes_the_indexer_selection(dsa):
    # the indexer's own top-k rows (prefill of 2,600 tokens: short rows padded with -1)
    # feed the attention unchanged
    wts = W.make_weights(43, hidden_dim=512, q_latent_dim=256)
    pre = W.make_prefill(44, [2600], hidden_dim=512, q_latent_dim=256)
    ix = dsa.Indexer(*(t.to("cuda").contiguous() for t in (wts.W_q, wts.W_k, wts.W_w, wts.gamma, wts.beta)),
                     max_tokens=4096)
    dev = "cuda"
    rows = int(pre.cache_offsets[-1])
    cache = torch.zeros((rows, 128), dtype=torch.bfloat16, device=dev)
    pos, qoff, coff = pre.positions.to(dev), pre.q_seq_offsets.to(dev), pre.cache_offsets.to(dev)
    q, w = ix.project(pre.hidden.to(dev), pre.q_latent.to(dev), pos, qoff, cache, coff)
    idx, _ = ix.topk(q, w, pos, qoff, cache, coff)
    mla = W.make_mla(45, [rows], [2600], n_heads=32, k_sel=2048)
    batch = W.MlaBatch(mla.q, mla.kv, mla.cache_offsets, mla.q_seq_offsets, idx.cpu())
    o, lse = _run(dsa, ix, batch)
    sample = W.stratified_rows(pre.q_seq_offsets, 24, seed=1, positions=pre.positions).numpy()
    _check(o[sample], lse[sample], *_ref(batch, rows=sample))


def test_sparse_mla_decode_full_size(dsa, ix):
    # the bench's decode step: 64 sequences of 16,384..131,072 cached rows, one query each,
    # 96 heads, 2,048 selected tokens
    lens = W.decode_lengths(5)
    batch = W.make_mla(5, lens.tolist(), [1] * 64, device="cuda")
    dev = "cuda"
    o, lse = ix.sparse_mla(batch.q.to(dev), batch.kv, batch.cache_offsets.to(dev), batch.q_seq_offsets.to(dev),
                           batch.idx.to(dev), SCALE)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    o, lse = f64(o.cpu()), lse.cpu().numpy().astype(np.float64)
    # the oracle on the selected rows only (each query's rows renumbered 0..2047)
    for t in range(0, 64, 3):
        kv_t = _selected_rows(batch, t)
        q_t = f64(batch.q[t])
        o_ref, lse_ref = oracle.sparse_mla(q_t[None], kv_t, np.array([0, 2048]), np.array([0, 1]),
                                           np.arange(2048)[None, :], SCALE)
        o_tol, lse_tol = _tolerances(q_t, kv_t, o_ref[0])
        _check(o[t:t + 1], lse[t:t + 1], o_ref, lse_ref, o_tol[None], lse_tol[None])


def test_sparse_mla_on_the_prefill_8k_selection_full_size(dsa):
    # the bench's prefill_8k workload (full-size weights and activations) through project and
    # top-k, its [8,192, 2,048] selection (rows of early queries padded with -1) feeding the
    # attention with all 96 heads: 16,384 CTAs; 24 stratified queries against the oracle
    cfg = W.WORKLOADS["prefill_8k"]
    wts = W.make_weights(cfg["weight_seed"])
    pre = W.make_prefill(cfg["act_seed"], cfg["seq_lens"])
    dev = "cuda"
    ix = dsa.Indexer(*(t.to(dev).contiguous() for t in (wts.W_q, wts.W_k, wts.W_w, wts.gamma, wts.beta)),
                     max_tokens=8192)
    T = pre.hidden.shape[0]
    cache = torch.zeros((T, 128), dtype=torch.bfloat16, device=dev)
    pos, qoff, coff = pre.positions.to(dev), pre.q_seq_offsets.to(dev), pre.cache_offsets.to(dev)
    q, w = ix.project(pre.hidden.to(dev), pre.q_latent.to(dev), pos, qoff, cache, coff)
    idx, _ = ix.topk(q, w, pos, qoff, cache, coff)
    mla = W.make_mla(47, [T], [T], n_heads=96, k_sel=1)          # q and cache only; idx replaced
    batch = W.MlaBatch(mla.q, mla.kv, mla.cache_offsets, mla.q_seq_offsets, idx.cpu())
    o, lse = _run(dsa, ix, batch)
    assert np.all(np.isfinite(lse)) and np.all(np.isfinite(o))
    sample = W.stratified_rows(pre.q_seq_offsets, 24, seed=2, positions=pre.positions).numpy()
    _check(o[sample], lse[sample], *_ref(batch, rows=sample))

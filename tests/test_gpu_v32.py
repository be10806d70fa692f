"""The DeepSeek-V3.2 form of the indexer -- 64 heads ('Sparse / compressed attn' row:
"DeepSeek-V3.2's indexer has 64 heads") and a rotary step on 64 of the 128 dims of q and k
('Partial RoPE / NoPE' row, page "Kimi K3.1 Pro vs Gemma 4 31B") -- against the oracle,
through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import assert_proj_close, check_sorted, check_topk, f64

pytestmark = pytest.mark.gpu

H = 64


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


def _indexer(d, wts, max_tokens=16384, rope_dim=64):
    return d.Indexer(_cuda(wts.W_q), _cuda(wts.W_k), _cuda(wts.W_w), _cuda(wts.gamma), _cuda(wts.beta),
                     max_tokens=max_tokens, rope_dim=rope_dim)


def _offsets(lens, dtype):
    o = torch.zeros(len(lens) + 1, dtype=dtype)
    o[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(dtype)
    return o


def _oracle_project(wts, batch, rope_dim=64):
    return oracle.project(f64(batch.hidden), f64(batch.q_latent), f64(wts.W_q), f64(wts.W_k), f64(wts.W_w),
                          f64(wts.gamma), f64(wts.beta), n_heads=H, head_dim=128, positions=batch.positions.numpy(),
                          rope_dim=rope_dim)


@pytest.mark.parametrize("rope_dim", [64, 0])
def test_v32_projections_match_oracle(dsa, rope_dim):
    wts = W.make_weights(61, hidden_dim=1024, q_latent_dim=256, n_heads=H)
    batch = W.make_prefill(62, [170, 130], start_positions=[0, 70_000], cache_lens=[200, 70_130],
                           hidden_dim=1024, q_latent_dim=256)
    ix = _indexer(dsa, wts, rope_dim=rope_dim)
    rows = int(batch.cache_offsets[-1])
    cache = torch.full((rows, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), _cuda(batch.positions),
                      _cuda(batch.q_seq_offsets), cache, _cuda(batch.cache_offsets))
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    assert q.shape == (300, H, 128) and w.shape == (300, H)
    oq, ok_, ow = _oracle_project(wts, batch, rope_dim)
    assert_proj_close(f64(q).reshape(300, -1), oq.reshape(300, -1), "q")
    assert_proj_close(f64(w), ow, "w")
    seq = oracle.sequence_of(batch.q_seq_offsets.numpy(), 300)
    written = [int(batch.cache_offsets[seq[t]]) + int(batch.positions[t]) for t in range(300)]
    assert_proj_close(f64(cache[written]), ok_, "k")


@pytest.mark.parametrize("flags", [0, 4, 2, 1])
def test_v32_topk_matches_oracle(dsa, flags):
    wts = W.make_weights(63, hidden_dim=128, q_latent_dim=64, n_heads=H)
    ix = _indexer(dsa, wts)
    if flags & 2:   # the split-key path: one query per sequence at the end of a long cache
        lens = [5000, 9000, 30000, 2048, 2049, 130]
        B = len(lens)
        q, keys, w = W.make_scoring_inputs(64, B, sum(lens), n_heads=H)
        positions = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
        qoff = torch.arange(B + 1, dtype=torch.int32)
    else:
        lens = [3000, 37, 2600]
        q, keys, w = W.make_scoring_inputs(65, sum(lens), sum(lens), n_heads=H)
        positions = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
        qoff = _offsets(lens, torch.int32)
    coff = _offsets(lens, torch.int64)
    idx, sc = ix.topk(_cuda(q), _cuda(w), _cuda(positions), _cuda(qoff), _cuda(keys), _cuda(coff), flags=flags)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    T = q.shape[0]
    rows = np.arange(T) if T <= 64 else np.unique(np.concatenate([np.arange(0, T, 11), [2046, 2047, 2048, T - 1]]))
    _, _, I, A = oracle.topk(f64(q), f64(w), positions.numpy(), qoff.numpy(), f64(keys), coff.numpy(),
                             rows=rows, keep_scores=True)
    gi, gs = idx.cpu().numpy()[rows], sc.cpu().numpy()[rows]
    recall, _ = check_topk(gi, gs, rows, positions.numpy()[rows], I, A)
    if flags & 1:
        check_sorted(gi, gs, rows, positions.numpy()[rows], I, A)
    print(f"64 heads flags={flags}: recall {recall:.6f}")


def test_v32_end_to_end(dsa):
    # projections with the rotary step, then the selection, at the model's widths
    wts = W.make_weights(66, n_heads=H)
    batch = W.make_prefill(67, [2500], start_positions=[100_000], cache_lens=[102_500])
    T = 2500
    ix = _indexer(dsa, wts, 4096)
    # the keys of positions 0..99,999 are not part of this batch: seeded N(0,1) rows stand in
    # for them (exactly tied zero rows would leave the selection free among ties)
    prefix = W.make_scoring_inputs(68, 1, 100_000, n_heads=H)[1]
    cache = torch.zeros((102_500, 128), dtype=torch.bfloat16, device="cuda")
    cache[:100_000] = _cuda(prefix)
    pos, qoff, coff = _cuda(batch.positions), _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    q, w = ix.project(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, cache, coff)
    idx, sc = ix.topk(q, w, pos, qoff, cache, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    oq, ok_, ow = _oracle_project(wts, batch)
    assert_proj_close(f64(q).reshape(T, -1), oq.reshape(T, -1), "q")
    assert_proj_close(f64(cache[100_000:]), ok_, "k")
    keys = np.zeros((102_500, 128))
    keys[:100_000] = f64(prefix)
    keys[100_000:] = ok_
    rows = np.arange(0, T, 50)
    _, _, I, A = oracle.topk(oq, ow, batch.positions.numpy(), batch.q_seq_offsets.numpy(), keys,
                             batch.cache_offsets.numpy(), rows=rows, keep_scores=True)
    recall, _ = check_topk(idx.cpu().numpy()[rows], sc.cpu().numpy()[rows], rows, batch.positions.numpy()[rows],
                           I, A)
    print(f"64 heads + RoPE end to end: recall {recall:.6f}")

"""FP8 indexer-key cache ('FP8 -> FP4 training' row, page "Kimi K3.1 Pro vs GLM-5": the
engines cache indexer keys in FP8) against the oracle, through the C ABI.

Quantisation decides integers (the e4m3 codes), so both sides take that decision from the
same bf16 value in float32: the codes of the FP8 projections must equal, bit for bit, the
oracle's quantisation of the bf16 projections of the same call (which are themselves checked
against the oracle's projections in the other tests).  Scores and selections are then
compared with the oracle's FP8 scores under the usual tolerance rule."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import check_sorted, check_topk, f64

pytestmark = pytest.mark.gpu


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


def _indexer(d, wts, max_tokens=16384):
    return d.Indexer(_cuda(wts.W_q), _cuda(wts.W_k), _cuda(wts.W_w), _cuda(wts.gamma), _cuda(wts.beta),
                     max_tokens=max_tokens)


def _offsets(lens, dtype):
    o = torch.zeros(len(lens) + 1, dtype=dtype)
    o[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(dtype)
    return o


def _codes_u8(codes: np.ndarray) -> torch.Tensor:
    """uint8 bit patterns of values on the e4m3 grid (exact conversion)."""
    return torch.tensor(codes, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)


def _codes_f64(u8: torch.Tensor) -> np.ndarray:
    return u8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _quantized_inputs(seed, T, S):
    q, keys, w = W.make_scoring_inputs(seed, T, S)
    q8, sq = oracle.quantize_fp8(f64(q).astype(np.float32))
    k8, sk = oracle.quantize_fp8(f64(keys).astype(np.float32))
    return q8, sq, k8, sk, w


def _run(dsa, ix, q8, sq, w, positions, qoff, k8, sk, coff, flags=0):
    idx, sc = ix.topk_fp8(_cuda(_codes_u8(q8)), _cuda(torch.tensor(sq, dtype=torch.float32)), _cuda(w),
                          _cuda(positions), _cuda(qoff), _cuda(_codes_u8(k8)),
                          _cuda(torch.tensor(sk, dtype=torch.float32)), _cuda(coff), flags=flags)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    return idx.cpu().numpy(), sc.cpu().numpy()


def test_fp8_projections_are_the_quantised_bf16_projections(dsa):
    wts = W.make_weights(31, hidden_dim=1024, q_latent_dim=256)
    batch = W.make_prefill(32, [170, 130], start_positions=[0, 40], cache_lens=[200, 180],
                           hidden_dim=1024, q_latent_dim=256)
    ix = _indexer(dsa, wts)
    rows = int(batch.cache_offsets[-1])
    hid, ql, pos = _cuda(batch.hidden), _cuda(batch.q_latent), _cuda(batch.positions)
    qoff, coff = _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    cache = torch.zeros((rows, 128), dtype=torch.bfloat16, device="cuda")
    q, w = ix.project(hid, ql, pos, qoff, cache, coff)
    k8 = torch.zeros((rows, 128), dtype=torch.uint8, device="cuda")
    ks = torch.full((rows,), -1.0, dtype=torch.float32, device="cuda")
    q8, qs, w8 = ix.project_fp8(hid, ql, pos, qoff, k8, ks, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    assert torch.equal(w, w8)
    oq8, osq = oracle.quantize_fp8(f64(q).astype(np.float32))
    assert np.array_equal(_codes_f64(q8), oq8), "query codes"
    assert np.array_equal(qs.cpu().numpy().astype(np.float64), osq), "query scales"
    seq = oracle.sequence_of(batch.q_seq_offsets.numpy(), batch.hidden.shape[0])
    written = [int(batch.cache_offsets[seq[t]]) + int(batch.positions[t]) for t in range(batch.hidden.shape[0])]
    ok8, osk = oracle.quantize_fp8(f64(cache[written]).astype(np.float32))
    assert np.array_equal(_codes_f64(k8[written]), ok8), "key codes"
    assert np.array_equal(ks[written].cpu().numpy().astype(np.float64), osk), "key scales"
    untouched = np.setdiff1d(np.arange(rows), written)
    assert bool((ks[untouched] == -1.0).all())


def test_fp8_key_quantiser_matches_the_oracle(dsa):
    wts = W.make_weights(33, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    g = torch.Generator().manual_seed(5)
    keys = (torch.randn((3000, 128), generator=g) * torch.rand((3000, 1), generator=g) * 3).to(torch.bfloat16)
    keys[7] = 0   # an all-zero row: scale 0, codes 0
    k8, ks = ix.quantize_keys_fp8(_cuda(keys))
    torch.cuda.synchronize()
    ok8, osk = oracle.quantize_fp8(f64(keys).astype(np.float32))
    assert np.array_equal(_codes_f64(k8), ok8)
    assert np.array_equal(ks.cpu().numpy().astype(np.float64), osk)


@pytest.mark.parametrize("flags", [0, 4, 1])
def test_fp8_topk_prefill_path(dsa, flags):
    wts = W.make_weights(34, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    lens = [3000, 37, 2600]
    T = sum(lens)
    q8, sq, k8, sk, w = _quantized_inputs(51, T, T)
    positions = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
    qoff, coff = _offsets(lens, torch.int32), _offsets(lens, torch.int64)
    gi, gs = _run(dsa, ix, q8, sq, w, positions, qoff, k8, sk, coff, flags)
    rows = np.unique(np.concatenate([np.arange(0, T, 13), [2046, 2047, 2048, 2999, T - 1]]))
    _, _, I, A = oracle.topk_fp8(q8, sq, f64(w), positions.numpy(), qoff.numpy(), k8, sk, coff.numpy(),
                                 rows=rows, keep_scores=True)
    recall, _ = check_topk(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)
    if flags & 1:
        check_sorted(gi[rows], gs[rows], rows, positions.numpy()[rows], I, A)
    print(f"fp8 prefill path flags={flags}: recall {recall:.6f}")


@pytest.mark.parametrize("flags", [0, 2])
def test_fp8_topk_long_prefixes(dsa, flags):
    # one query per sequence at the end of its cache (the decode shape; flags=2 forces the
    # split-key path with its merge)
    wts = W.make_weights(35, hidden_dim=128, q_latent_dim=64)
    ix = _indexer(dsa, wts)
    lens = [5000, 9000, 20000, 40000, 2048, 2049, 130]
    B = len(lens)
    q8, sq, k8, sk, w = _quantized_inputs(52, B, sum(lens))
    positions = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
    qoff = torch.arange(B + 1, dtype=torch.int32)
    coff = _offsets(lens, torch.int64)
    gi, gs = _run(dsa, ix, q8, sq, w, positions, qoff, k8, sk, coff, flags)
    _, _, I, A = oracle.topk_fp8(q8, sq, f64(w), positions.numpy(), qoff.numpy(), k8, sk, coff.numpy(),
                                 keep_scores=True)
    recall, _ = check_topk(gi, gs, np.arange(B), positions.numpy(), I, A)
    print(f"fp8 long prefixes flags={flags}: recall {recall:.6f}")


def test_fp8_end_to_end_prefill(dsa):
    # project_fp8 then topk_fp8 on a 3,000-token sequence of the model's shapes; the oracle
    # scores the GPU's codes (bit-exact to the oracle's quantisation of the bf16 projections,
    # checked above), and the bf16 oracle's selection is reported for reference
    wts = W.make_weights(36)
    batch = W.make_prefill(37, [3000])
    T = 3000
    ix = _indexer(dsa, wts, 4096)
    pos, qoff, coff = _cuda(batch.positions), _cuda(batch.q_seq_offsets), _cuda(batch.cache_offsets)
    k8 = torch.zeros((T, 128), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((T,), dtype=torch.float32, device="cuda")
    q8, qs, w = ix.project_fp8(_cuda(batch.hidden), _cuda(batch.q_latent), pos, qoff, k8, ks, coff)
    idx, sc = ix.topk_fp8(q8, qs, w, pos, qoff, k8, ks, coff)
    torch.cuda.synchronize()
    assert ix.device_error() == dsa.DSA_OK
    rows = np.unique(np.concatenate([np.arange(0, T, 29), [2047, 2048, T - 1]]))
    _, _, I, A = oracle.topk_fp8(_codes_f64(q8), qs.cpu().numpy().astype(np.float64), f64(w),
                                 batch.positions.numpy(), batch.q_seq_offsets.numpy(), _codes_f64(k8),
                                 ks.cpu().numpy().astype(np.float64), batch.cache_offsets.numpy(), rows=rows,
                                 keep_scores=True)
    recall, _ = check_topk(idx.cpu().numpy()[rows], sc.cpu().numpy()[rows], rows, batch.positions.numpy()[rows],
                           I, A)
    oq, ok_, ow = oracle.project(f64(batch.hidden), f64(batch.q_latent), f64(wts.W_q), f64(wts.W_k),
                                 f64(wts.W_w), f64(wts.gamma), f64(wts.beta))
    ref, _ = oracle.topk(oq, ow, batch.positions.numpy(), batch.q_seq_offsets.numpy(), ok_,
                         batch.cache_offsets.numpy(), rows=rows)
    gi = idx.cpu().numpy()[rows]
    long_ = batch.positions.numpy()[rows] >= 2048
    vs_bf16 = np.mean([len(np.intersect1d(gi[r], ref[r])) / 2048 for r in np.nonzero(long_)[0]])
    print(f"fp8 end to end: recall {recall:.6f} against the FP8 oracle, {vs_bf16:.4f} overlap with the bf16 "
          f"oracle's selection")

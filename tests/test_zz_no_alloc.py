"""dsa_indexer_topk_noalloc against dsa_indexer_topk, through the C ABI.

The allocation-free entry point serves callers that cannot let the library
allocate device memory (a memory pool that already owns the device's budget,
or a loop that must never pay for cudaMalloc / cudaFree).  It keeps its
scratch in the library's static device memory, so this test checks that two
calls in a row -- the second reusing the scratch the first left behind --
return what the handle-based entry point returns for the same inputs.

The rows are also checked against the CPU oracle (sampled rows, the parity
rule of the other tests), and the cases reach the limits that size the
static scratch: 4,096 queries in 4,096 sequences, and 4,096 queries of one
sequence whose prefixes all exceed 2,048 keys.

This file is collected last on purpose: a failure here leaves every other
test already run.  It passes both alone in a fresh process and after the
rest of the suite."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import check_topk, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dsa_lightning_indexer_03_b200 import build
    build.build()
    from dsa_lightning_indexer_03_b200 import _lib
    return _lib.load()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _case(seed, lens, starts=None):
    """Score + top-k inputs for sequences of `lens` query tokens (on the GPU); sequence b
    holds starts[b] + lens[b] key rows and its queries sit at positions starts[b] ..."""
    starts = starts or [0] * len(lens)
    T = sum(lens)
    rows = [s + n for s, n in zip(starts, lens)]
    q, keys, w = W.make_scoring_inputs(seed, T, sum(rows))
    positions = torch.cat([torch.arange(s, s + n, dtype=torch.int32) for s, n in zip(starts, lens)])
    qoff = torch.zeros(len(lens) + 1, dtype=torch.int32)
    qoff[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    coff = torch.zeros(len(lens) + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(torch.tensor(rows), 0)
    c = lambda t: t.to("cuda").contiguous()  # noqa: E731
    return dict(T=T, B=len(lens), q=c(q), w=c(w), pos=c(positions), qoff=c(qoff), keys=c(keys), coff=c(coff),
                host=dict(q=q, w=w, pos=positions, qoff=qoff, keys=keys, coff=coff))


def _with_handle(lib, x):
    from dsa_lightning_indexer_03_b200 import _lib
    cfg = _lib.Config()
    lib.dsa_indexer_default_config(ctypes.byref(cfg))
    cfg.hidden_dim, cfg.q_latent_dim, cfg.max_tokens = 128, 64, 8192
    wts = W.make_weights(0, hidden_dim=128, q_latent_dim=64)
    c = lambda t: t.to("cuda").contiguous()  # noqa: E731
    ws = [c(wts.W_q), c(wts.W_k), c(wts.W_w), c(wts.gamma), c(wts.beta)]
    h = ctypes.c_void_p()
    assert lib.dsa_indexer_create(ctypes.byref(cfg), *[_p(t) for t in ws], ctypes.byref(h)) == 0
    idx = torch.empty((x["T"], 2048), dtype=torch.int32, device="cuda")
    sc = torch.empty((x["T"], 2048), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.dsa_indexer_topk(h, x["T"], _p(x["q"]), _p(x["w"]), _p(x["pos"]), _p(x["qoff"]), x["B"], _p(x["keys"]),
                                x["keys"].shape[0], _p(x["coff"]), _p(idx), _p(sc), 4, stream) == 0
    torch.cuda.synchronize()
    assert lib.dsa_indexer_device_error(h) == 0
    lib.dsa_indexer_destroy(h)
    return idx.cpu().numpy(), sc.cpu().numpy()


def _no_alloc(lib, x):
    idx = torch.full((x["T"], 2048), -7, dtype=torch.int32, device="cuda")   # never a valid output
    sc = torch.zeros((x["T"], 2048), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.dsa_indexer_topk_noalloc(x["T"], _p(x["q"]), _p(x["w"]), _p(x["pos"]), _p(x["qoff"]), x["B"],
                                      _p(x["keys"]), x["keys"].shape[0], _p(x["coff"]), _p(idx), _p(sc), stream)
    assert st == 0
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


def _same_selection(a_idx, a_sc, b_idx, b_sc):
    """Equal rows, except that among keys tied at the cut either may be kept; the
    kept scores must then agree as multisets (the tolerance the tests use for
    index sets: identical outside the tie band, here of width zero)."""
    for r in range(a_idx.shape[0]):
        if np.array_equal(a_idx[r], b_idx[r]):
            continue
        sa, sb = np.sort(a_idx[r]), np.sort(b_idx[r])
        if np.array_equal(sa, sb):
            continue
        assert np.array_equal(np.sort(a_sc[r]), np.sort(b_sc[r])), f"row {r}: kept scores differ"
        diff = np.setxor1d(sa, sb)
        cut = max(a_sc[r][a_idx[r] >= 0].min(), b_sc[r][b_idx[r] >= 0].min())
        sel = np.concatenate([a_sc[r][np.isin(a_idx[r], diff)], b_sc[r][np.isin(b_idx[r], diff)]])
        assert np.all(sel == cut), f"row {r}: index sets differ away from a tie"
    # scores of identical positions are identical (same kernels, same inputs)
    for r in range(a_idx.shape[0]):
        m = dict(zip(a_idx[r].tolist(), a_sc[r].tolist()))
        for i, s in zip(b_idx[r].tolist(), b_sc[r].tolist()):
            if i >= 0 and i in m:
                assert m[i] == s


def _against_oracle(x, idx, sc, rows):
    """Sampled rows of a no-alloc result against the CPU oracle (same rule as the other tests)."""
    h = x["host"]
    _, _, I, A = oracle.topk(f64(h["q"]), f64(h["w"]), h["pos"].numpy(), h["qoff"].numpy(), f64(h["keys"]),
                             h["coff"].numpy(), 2048, rows=rows, keep_scores=True)
    recall, _ = check_topk(idx[rows], sc[rows], rows, h["pos"].numpy()[rows], I, A)
    return recall


def _rows(x, n, seed):
    rng = np.random.default_rng(seed)
    T = x["T"]
    return np.unique(np.concatenate([rng.choice(T, size=min(n, T), replace=False), [0, T - 1]]))


def test_no_alloc_matches_handle_entry_on_two_calls_in_a_row(lib):
    first = _case(41, [3000])                              # one sequence, long and short prefixes
    second = _case(42, [700, 2600, 1, 45], [0, 100, 0, 5])  # ragged batch, offset positions
    for k, x in enumerate((first, second)):
        ref_idx, ref_sc = _with_handle(lib, x)
        got_idx, got_sc = _no_alloc(lib, x)
        assert not np.any(got_idx == -7)   # every output slot was written
        _same_selection(ref_idx, ref_sc, got_idx, got_sc)
        recall = _against_oracle(x, got_idx, got_sc, _rows(x, 300, k))
        print(f"no-alloc call {k}: recall against the oracle {recall:.6f}")
    assert lib.dsa_indexer_noalloc_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


def test_no_alloc_at_the_limits_of_its_scratch(lib):
    # 4,096 sequences of one query each (the work list's owner bases then live in the scratch,
    # not in shared memory): 64 of them with prefixes of 2,049..2,600 keys, the rest short
    rng = np.random.default_rng(7)
    starts = rng.integers(0, 12, 4096)
    long_ = rng.choice(4096, 64, replace=False)
    starts[long_] = rng.integers(2048, 2600, 64)
    many = _case(44, [1] * 4096, [int(v) for v in starts])
    # 4,096 queries of one sequence, at positions 3,000..7,095: every prefix is long, so the
    # streaming selection runs for every item of the longest work list the scratch holds
    deep = _case(45, [4096], [3000])
    for k, (x, rows) in enumerate(((many, np.unique(np.concatenate([long_, np.arange(0, 4096, 97)]))),
                                   (deep, _rows(deep, 120, 9)))):
        ref_idx, ref_sc = _with_handle(lib, x)
        got_idx, got_sc = _no_alloc(lib, x)
        assert not np.any(got_idx == -7)
        _same_selection(ref_idx, ref_sc, got_idx, got_sc)
        recall = _against_oracle(x, got_idx, got_sc, rows)
        print(f"no-alloc limit case {k}: recall against the oracle {recall:.6f}")
    assert lib.dsa_indexer_noalloc_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


def test_no_alloc_pads_rows_and_reports_malformed_offsets(lib):
    x = _case(46, [100, 50, 50])
    x["qoff"] = torch.tensor([0, 150, 100, 200], dtype=torch.int32, device="cuda")   # not monotone
    idx, sc = _no_alloc(lib, x)
    assert np.all(idx == -1) and np.all(np.isneginf(sc))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.dsa_indexer_noalloc_device_error(stream) == 7   # DSA_ERR_DEVICE_BOUNDS
    # the next call starts from a clear error word
    y = _case(47, [300])
    _no_alloc(lib, y)
    assert lib.dsa_indexer_noalloc_device_error(stream) == 0


def test_no_alloc_rejects_sizes_beyond_its_scratch(lib):
    x = _case(43, [5])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.dsa_indexer_topk_noalloc(4097, _p(x["q"]), _p(x["w"]), _p(x["pos"]), _p(x["qoff"]), 1, _p(x["keys"]),
                                      x["keys"].shape[0], _p(x["coff"]), _p(x["q"]), None, stream)
    assert st == 5   # DSA_ERR_WORKSPACE, nothing launched

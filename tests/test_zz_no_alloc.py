"""dsa_indexer_topk_noalloc against dsa_indexer_topk, through the C ABI.

The allocation-free entry point serves callers that cannot let the library
allocate device memory (a memory pool that already owns the device's budget,
or a loop that must never pay for cudaMalloc / cudaFree).  It keeps its
scratch in the library's static device memory, so this test checks that two
calls in a row -- the second reusing the scratch the first left behind --
return what the handle-based entry point returns for the same inputs.

This file is collected last on purpose: a failure here leaves every other
test already run.  It passes both alone in a fresh process and after the
rest of the suite."""

import ctypes

import numpy as np
import pytest
import torch

import workloads as W

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
    """Score + top-k inputs for sequences of `lens` query tokens (on the GPU)."""
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
    return dict(T=T, B=len(lens), q=c(q), w=c(w), pos=c(positions), qoff=c(qoff), keys=c(keys), coff=c(coff))


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


def test_no_alloc_matches_handle_entry_on_two_calls_in_a_row(lib):
    first = _case(41, [3000])                              # one sequence, long and short prefixes
    second = _case(42, [700, 2600, 1, 45], [0, 100, 0, 5])  # ragged batch, offset positions
    for x in (first, second):
        ref_idx, ref_sc = _with_handle(lib, x)
        got_idx, got_sc = _no_alloc(lib, x)
        assert not np.any(got_idx == -7)   # every output slot was written
        _same_selection(ref_idx, ref_sc, got_idx, got_sc)


def test_no_alloc_rejects_sizes_beyond_its_scratch(lib):
    x = _case(43, [5])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.dsa_indexer_topk_noalloc(4097, _p(x["q"]), _p(x["w"]), _p(x["pos"]), _p(x["qoff"]), 1, _p(x["keys"]),
                                      x["keys"].shape[0], _p(x["coff"]), _p(x["q"]), None, stream)
    assert st == 5   # DSA_ERR_WORKSPACE, nothing launched

"""Parity helpers shared by the GPU tests: oracle runs on the workloads' CPU
tensors and the comparison rules.

Comparison rules (the tolerances follow from bf16 inputs with fp32 accumulation):
  * projections: |gpu - oracle| <= 1e-2 * max(|oracle|, 2^-8 * rms(oracle row))
    (1e-2 relative, with a floor of one bf16 step of the row's typical size so
    that values that cancel to ~0 are judged on the row's scale);
  * masking and padding: bit-exact;
  * scores: |I_gpu - I_oracle| <= 2e-3 * A with A = sum_h |w_h q_h.k|;
  * index sets: identical except for keys whose oracle score lies within
    2e-3 * (A[s] + A[s*]) of the k-th oracle score I*; recall reported.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

PROJ_RTOL = 1e-2
SCORE_TOL = 2e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def oracle_project(weights, hidden, q_latent, eps=1e-6):
    return oracle.project(f64(hidden), f64(q_latent), f64(weights.W_q), f64(weights.W_k), f64(weights.W_w),
                          f64(weights.gamma), f64(weights.beta), eps,
                          n_heads=weights.W_w.shape[1], head_dim=weights.W_k.shape[1])


def assert_proj_close(gpu: np.ndarray, ora: np.ndarray, what: str, rtol: float = PROJ_RTOL):
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    assert gpu.shape == ora.shape, (what, gpu.shape, ora.shape)
    assert np.all(np.isfinite(gpu)), what
    rms = np.sqrt(np.mean(ora ** 2, axis=-1, keepdims=True))
    scale = np.maximum(np.abs(ora), 2.0 ** -8 * rms)
    err = np.abs(gpu - ora) / scale
    worst = float(err.max()) if err.size else 0.0
    assert worst <= rtol, f"{what}: worst scaled error {worst:.3e} > {rtol}"
    return worst


def check_topk(gpu_idx: np.ndarray, gpu_score, rows, positions, I_list, A_list, top_k: int = 2048,
               tol: float = SCORE_TOL, min_recall: float | None = 0.999):
    """gpu_idx/gpu_score: [R, top_k] for the R query rows `rows` (global token ids);
    positions: positions of those rows; I_list/A_list: oracle prefix scores per row."""
    recalls = []
    n_band = 0
    for r in range(len(rows)):
        p = int(positions[r])
        n = p + 1
        I = I_list[r]
        A = A_list[r]
        g = np.asarray(gpu_idx[r], np.int64)
        if n <= top_k:
            exp = np.concatenate([np.arange(n), -np.ones(top_k - n, np.int64)])
            assert np.array_equal(g, exp), f"row {rows[r]} (pos {p}): padding row differs"
            if gpu_score is not None:
                gs = np.asarray(gpu_score[r], np.float64)
                assert np.all(np.abs(gs[:n] - I) <= tol * A + 1e-30), f"row {rows[r]}: scores"
                assert np.all(np.isneginf(gs[n:])), f"row {rows[r]}: padding scores"
            recalls.append(1.0)
            continue
        assert g.min() >= 0 and g.max() <= p, f"row {rows[r]}: index outside the causal prefix"
        assert len(np.unique(g)) == top_k, f"row {rows[r]}: duplicate indices"
        order = np.lexsort((np.arange(n), -I))
        o = order[:top_k]
        s_star = o[-1]
        I_star = I[s_star]
        diff = np.setxor1d(g, o)
        if diff.size:
            band = tol * (A[diff] + A[s_star])
            bad = np.abs(I[diff] - I_star) > band
            assert not bad.any(), (f"row {rows[r]}: {int(bad.sum())} keys differ outside the tolerance band; "
                                   f"e.g. s={int(diff[bad][0])} I={I[diff[bad][0]]:.6g} I*={I_star:.6g}")
            n_band += diff.size
        recalls.append(len(np.intersect1d(g, o)) / top_k)
        if gpu_score is not None:
            gs = np.asarray(gpu_score[r], np.float64)
            assert np.all(np.abs(gs - I[g]) <= tol * A[g] + 1e-30), f"row {rows[r]}: scores"
    recall = float(np.mean(recalls)) if recalls else 1.0
    if min_recall is not None:
        assert recall >= min_recall, f"recall {recall:.5f} < {min_recall}"
    return recall, n_band


def oracle_topk_rows(q, w, positions, q_seq_offsets, key_cache, cache_offsets, rows, top_k=2048):
    idx, sc, I_list, A_list = oracle.topk(q, w, positions, q_seq_offsets, key_cache, cache_offsets, top_k,
                                          rows=rows, keep_scores=True)
    return idx, sc, I_list, A_list


def check_sorted(gpu_idx: np.ndarray, gpu_score: np.ndarray, rows, positions, I_list, A_list, top_k: int = 2048,
                 tol: float = SCORE_TOL):
    """DSA_TOPK_SORTED rows: a short prefix keeps [0..p, -1...]; a long one is ordered by the
    GPU's own scores descending, positions ascending among exactly equal scores (bit-exact,
    it is the sort's own key), and by the oracle's scores descending wherever two neighbours'
    oracle scores differ by more than the tolerance band (the set itself is checked by
    check_topk).  Returns the number of neighbour pairs whose order the band leaves open."""
    open_pairs = 0
    for r in range(len(rows)):
        n = int(positions[r]) + 1
        g = np.asarray(gpu_idx[r], np.int64)
        if n <= top_k:
            exp = np.concatenate([np.arange(n), -np.ones(top_k - n, np.int64)])
            assert np.array_equal(g, exp), f"row {rows[r]}: short rows keep position order"
            continue
        s = np.asarray(gpu_score[r], np.float64)
        assert np.all(s[:-1] >= s[1:]), f"row {rows[r]}: GPU scores not descending"
        eq = s[:-1] == s[1:]
        assert np.all(g[:-1][eq] < g[1:][eq]), f"row {rows[r]}: equal scores not in position order"
        I, A = I_list[r], A_list[r]
        a, b = g[:-1], g[1:]
        band = tol * (A[a] + A[b])
        assert np.all(I[a] >= I[b] - band), f"row {rows[r]}: order contradicts the oracle outside the band"
        open_pairs += int(np.sum(np.abs(I[a] - I[b]) <= band))
    return open_pairs


def mla_tolerances(q_t, rows, o_ref_t, scale):
    """Bounds of the sparse MLA check for one query (q_t [H, 576], the selected rows [n, 576]
    in float64, the oracle's o [H, 512]): per value, |o - o_ref| <= 1.01 U (spread + |o_ref|)
    + e_s spread + 1e-5 with U = 2^-8 (bf16 unit roundoff: the weights enter P.V as bf16 and
    o is written as bf16), spread = max_j |v_jd - o_d| over the selected latents and
    e_s = 6 sqrt(576) 2^-24 scale |q_h| max_j |row_j| (a six-sigma random-walk allowance for
    the fp32 score sums); per head, |lse - lse_ref| <= 1.01 U + e_s + 1e-5."""
    U = 2.0 ** -8
    if rows.shape[0] == 0:
        return np.full(o_ref_t.shape, 1e-5), np.full(o_ref_t.shape[0], 1e-5)
    v = rows[:, :512]
    spread = np.maximum(v.max(0)[None, :] - o_ref_t, o_ref_t - v.min(0)[None, :])
    e_s = 6 * np.sqrt(576) * 2.0 ** -24 * scale * np.linalg.norm(q_t, axis=1) * np.linalg.norm(rows, axis=1).max()
    o_tol = 1.01 * U * (spread + np.abs(o_ref_t)) + e_s[:, None] * spread + 1e-5
    return o_tol, 1.01 * U + e_s + 1e-5

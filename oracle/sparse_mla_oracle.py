"""CPU oracle of the sparse MLA attention over the indexer's selection -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import or run this
module; it shares no code with the CUDA library.

What it computes ('Latent attention (MLA)' row of the archdiff.com compare pages "Qwen3.5-
397B-A17B vs Kimi K3.1 Pro" and "Kimi K3.1 Pro vs Gemma 4 31B"): 96 heads; keys and values
come from a 512-dim latent plus a 64-dim shared key slot, 576 cached values per token; each
query attends only to the 2,048 tokens its layer's indexer selects.

Readings where the pages are silent (each is listed in the design notes):
  * the attention runs in the latent ("absorbed") form: a head's 128-dim no-rope query is
    taken into the 512-dim latent space beforehand (its product with the head's key up-
    projection), so the query is 576 values per head (512 latent + 64 rope) and scores the
    cached 576-value row directly; the value is the row's 512-dim latent, and the per-head
    value up-projection (512 -> 128) and the output projection are dense products after it;
  * score = scale * (q . row) with scale a parameter (1/sqrt(192) for a 192-dim q/k head);
    softmax over the selected tokens of the query's own sequence; a -1 index is no token;
  * outputs: o = sum_j p_j * latent_j (512 per head) and lse = log(sum_j exp(score_j)),
    natural log; a query with no selected token gets o = 0 and lse = -inf.
"""

from __future__ import annotations

import numpy as np

MLA_HEADS = 96
MLA_DIM = 576        # cached values per token: 512 latent + 64 rope key
MLA_LATENT = 512     # the value part


def sparse_mla(q, kv_cache, cache_offsets, q_seq_offsets, idx, scale: float):
    """q [T, H, 576], kv_cache [rows, 576], cache_offsets [B+1] (first row of each sequence),
    q_seq_offsets [B+1] (the queries of each sequence), idx [T, K] positions within the
    query's sequence (-1 = none).  Returns o [T, H, 512] and lse [T, H] in float64."""
    q = np.asarray(q, np.float64)
    kv = np.asarray(kv_cache, np.float64)
    co = np.asarray(cache_offsets, np.int64)
    qo = np.asarray(q_seq_offsets, np.int64)
    idx = np.asarray(idx, np.int64)
    T, H, D = q.shape
    o = np.zeros((T, H, MLA_LATENT))
    lse = np.full((T, H), -np.inf)
    for t in range(T):
        b = int(np.searchsorted(qo, t, side="right") - 1)
        sel = idx[t][idx[t] >= 0]
        if sel.size == 0:
            continue
        rows = kv[co[b] + sel]                      # [n, 576]
        s = scale * (q[t] @ rows.T)                 # [H, n]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        o[t] = (e / z) @ rows[:, :MLA_LATENT]
        lse[t] = (m + np.log(z))[:, 0]
    return o, lse

"""Seeded generators for the indexer's five workloads (random draws only).

Shapes and value distributions:
  * weights: W_q [1536, 4096], W_k [7168, 128], W_w [7168, 32], bf16, each
    N(0, 1/fan_in); LayerNorm gain 1 + N(0, 0.02^2) and bias N(0, 0.02^2), bf16.
  * prefill activations: hidden [T, 7168] and query latent [T, 1536], bf16
    N(0, 1); token positions 0..n_b-1 per sequence (or a chunk's offset).
  * decode: 64 sequences with cache lengths uniform in [16384, 131072]; the
    pre-norm key rows of every cached token are fp32 N(0, 1) (the key cache is
    the LayerNorm of these rows, computed by whichever side consumes them).

Each tensor is drawn from its own torch CPU generator whose seed is derived
from (workload seed, stream id), so that no two tensors share a random stream.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

# Kimi K3.1 Pro indexer dimensions ('Sparse / compressed attn' row of the
# archdiff.com compare pages): hidden width 7,168, query latent 1,536,
# 32 heads x 128 dims, top 2,048 tokens per query.
MODEL_DIMS = dict(hidden_dim=7168, q_latent_dim=1536, n_heads=32, head_dim=128, top_k=2048)

# The five workloads: three single-shot prefills, one decode step, one chunked
# long-context prefill.
WORKLOADS = {
    "prefill_3k": dict(kind="prefill", seq_lens=[3072], weight_seed=0, act_seed=0),
    "prefill_8k": dict(kind="prefill", seq_lens=[8192], weight_seed=1, act_seed=2),
    "prefill_2x32k_heavy": dict(kind="prefill", seq_lens=[32768, 32768], weight_seed=3,
                                act_seed=4, heavy_frac=0.01, heavy_scale=4.0),
    "decode_64": dict(kind="decode", batch=64, L_min=16384, L_max=131072, weight_seed=5,
                      act_seed=5),
    "chunked_128k": dict(kind="chunked", seq_len=131072, chunk=8192, weight_seed=6, act_seed=7),
}

# stream ids: one per tensor kind
_S_WQ, _S_WK, _S_WW, _S_GAMMA, _S_BETA = 1, 2, 3, 4, 5
_S_HIDDEN, _S_QLAT, _S_LENS, _S_RAWK, _S_HEAVY = 11, 12, 13, 14, 15
_S_MLA_Q, _S_MLA_KV, _S_MLA_IDX = 21, 22, 23

# Sparse MLA consumer ('Latent attention (MLA)' row): 96 heads, 576 cached values per token
# (512 latent + 64 rope key), 2,048 selected tokens per query.
MLA_DIMS = dict(n_heads=96, dim=576, latent=512, k_sel=2048)


def _gen(seed: int, stream: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed((int(seed) * 1_000_003 + stream * 7919 + int(sub) * 104_729) & 0x7FFF_FFFF_FFFF)
    return g


def _normal(g: torch.Generator, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


@dataclass
class Weights:
    W_q: torch.Tensor      # bf16 [q_latent_dim, n_heads*head_dim]   (in x out)
    W_k: torch.Tensor      # bf16 [hidden_dim, head_dim]
    W_w: torch.Tensor      # bf16 [hidden_dim, n_heads]
    gamma: torch.Tensor    # bf16 [head_dim]
    beta: torch.Tensor     # bf16 [head_dim]


@dataclass
class PrefillBatch:
    hidden: torch.Tensor         # bf16 [T, hidden_dim]
    q_latent: torch.Tensor       # bf16 [T, q_latent_dim]
    positions: torch.Tensor      # int32 [T], position of each query token in its sequence
    q_seq_offsets: torch.Tensor  # int32 [B+1], token ranges of the B sequences
    cache_offsets: torch.Tensor  # int64 [B+1], key-cache row ranges of the B sequences
    extra: dict = field(default_factory=dict)


@dataclass
class DecodeBatch:
    lengths: torch.Tensor        # int64 [B], cached tokens per sequence (incl. the new one)
    raw_keys: torch.Tensor       # fp32 [sum L, head_dim], pre-norm key rows of every cached token
    hidden: torch.Tensor         # bf16 [B, hidden_dim], the new token of each sequence
    q_latent: torch.Tensor       # bf16 [B, q_latent_dim]
    positions: torch.Tensor      # int32 [B] = L_b - 1
    q_seq_offsets: torch.Tensor  # int32 [B+1] = 0..B
    cache_offsets: torch.Tensor  # int64 [B+1]


def make_weights(seed: int, hidden_dim: int = 7168, q_latent_dim: int = 1536,
                 n_heads: int = 32, head_dim: int = 128) -> Weights:
    """Random-init weights of one indexer layer, N(0, 1/fan_in), bf16."""
    W_q = _normal(_gen(seed, _S_WQ), (q_latent_dim, n_heads * head_dim), q_latent_dim ** -0.5)
    W_k = _normal(_gen(seed, _S_WK), (hidden_dim, head_dim), hidden_dim ** -0.5)
    W_w = _normal(_gen(seed, _S_WW), (hidden_dim, n_heads), hidden_dim ** -0.5)
    gamma = _normal(_gen(seed, _S_GAMMA), (head_dim,), 0.02, 1.0)
    beta = _normal(_gen(seed, _S_BETA), (head_dim,), 0.02)
    bf = torch.bfloat16
    return Weights(W_q.to(bf), W_k.to(bf), W_w.to(bf), gamma.to(bf), beta.to(bf))


def make_prefill(seed: int, seq_lens, start_positions=None, cache_lens=None,
                 hidden_dim: int = 7168, q_latent_dim: int = 1536, sub: int = 0) -> PrefillBatch:
    """B sequences of query tokens.  Sequence b has seq_lens[b] tokens at
    positions start_b .. start_b+n_b-1 and owns cache_lens[b] key-cache rows
    (default start_b + n_b, i.e. exactly the causal prefix of its last token)."""
    seq_lens = [int(n) for n in seq_lens]
    B = len(seq_lens)
    starts = [0] * B if start_positions is None else [int(s) for s in start_positions]
    clens = [s + n for s, n in zip(starts, seq_lens)] if cache_lens is None else [int(c) for c in cache_lens]
    for s, n, c in zip(starts, seq_lens, clens):
        if s + n > c:
            raise ValueError("a sequence's positions must fit inside its cache rows")
    T = sum(seq_lens)
    hidden = _normal(_gen(seed, _S_HIDDEN, sub), (T, hidden_dim)).to(torch.bfloat16)
    q_latent = _normal(_gen(seed, _S_QLAT, sub), (T, q_latent_dim)).to(torch.bfloat16)
    positions = torch.cat([torch.arange(s, s + n, dtype=torch.int32) for s, n in zip(starts, seq_lens)]) \
        if T > 0 else torch.zeros(0, dtype=torch.int32)
    q_seq_offsets = torch.zeros(B + 1, dtype=torch.int32)
    q_seq_offsets[1:] = torch.cumsum(torch.tensor(seq_lens, dtype=torch.int64), 0).to(torch.int32)
    cache_offsets = torch.zeros(B + 1, dtype=torch.int64)
    cache_offsets[1:] = torch.cumsum(torch.tensor(clens, dtype=torch.int64), 0)
    return PrefillBatch(hidden, q_latent, positions, q_seq_offsets, cache_offsets)


def decode_lengths(seed: int, batch: int = 64, L_min: int = 16384, L_max: int = 131072) -> torch.Tensor:
    """Cache length of each decode sequence, uniform in [L_min, L_max]."""
    return torch.randint(L_min, L_max + 1, (batch,), generator=_gen(seed, _S_LENS), dtype=torch.int64)


def make_decode(seed: int, batch: int = 64, L_min: int = 16384, L_max: int = 131072,
                hidden_dim: int = 7168, q_latent_dim: int = 1536, head_dim: int = 128,
                lengths=None) -> DecodeBatch:
    """One new query token per sequence; sequence b holds L_b cached tokens
    (the new token is the last, at position L_b - 1)."""
    if lengths is None:
        lengths = decode_lengths(seed, batch, L_min, L_max)
    else:
        lengths = torch.as_tensor(lengths, dtype=torch.int64)
        batch = int(lengths.numel())
    total = int(lengths.sum())
    raw_keys = _normal(_gen(seed, _S_RAWK), (total, head_dim))
    hidden = _normal(_gen(seed, _S_HIDDEN), (batch, hidden_dim)).to(torch.bfloat16)
    q_latent = _normal(_gen(seed, _S_QLAT), (batch, q_latent_dim)).to(torch.bfloat16)
    positions = (lengths - 1).to(torch.int32)
    q_seq_offsets = torch.arange(batch + 1, dtype=torch.int32)
    cache_offsets = torch.zeros(batch + 1, dtype=torch.int64)
    cache_offsets[1:] = torch.cumsum(lengths, 0)
    return DecodeBatch(lengths, raw_keys, hidden, q_latent, positions, q_seq_offsets, cache_offsets)


def heavy_hitter_rows(seed: int, cache_offsets: torch.Tensor, frac: float = 0.01) -> torch.Tensor:
    """Global key-cache rows to scale (round(frac * L_b) per sequence, drawn
    without replacement).  Scaling a bf16 row by 4 is exact."""
    rows = []
    g = _gen(seed, _S_HEAVY)
    offs = [int(v) for v in cache_offsets.tolist()]
    for b in range(len(offs) - 1):
        L = offs[b + 1] - offs[b]
        m = int(round(frac * L))
        if m > 0:
            rows.append(torch.randperm(L, generator=g)[:m] + offs[b])
    return torch.cat(rows).to(torch.int64) if rows else torch.zeros(0, dtype=torch.int64)


def make_scoring_inputs(seed: int, n_queries: int, n_keys: int, n_heads: int = 32, head_dim: int = 128,
                        key_scale: float = 1.0):
    """Direct inputs of the score + top-k step, for testing it on its own:
    q bf16 N(0,1) [T, n_heads, head_dim], keys bf16 N(0, key_scale^2) [S, head_dim]
    (the scale of LayerNorm outputs), w fp32 N(0,1) [T, n_heads]."""
    q = _normal(_gen(seed, _S_QLAT, 1), (n_queries, n_heads, head_dim)).to(torch.bfloat16)
    keys = _normal(_gen(seed, _S_RAWK, 1), (n_keys, head_dim), key_scale).to(torch.bfloat16)
    w = _normal(_gen(seed, _S_WW, 1), (n_queries, n_heads))
    return q, keys, w


def causal_pairs(positions: torch.Tensor) -> int:
    """Number of (query, key) pairs a causal pass scores: sum over queries of pos + 1."""
    return int(positions.to(torch.int64).sum()) + int(positions.numel())


def stratified_rows(q_seq_offsets, n: int, seed: int = 0, chunk: int | None = None,
                    positions=None) -> "torch.Tensor":
    """Query rows (global token indices) that sample a workload for checking or timing.

    Always included: the first and last token of every sequence, the first and last
    token of every `chunk`-token chunk (when given), and the tokens at positions
    2,046..2,049 (where a prefix reaches the 2,048 kept tokens), when present.  The
    rest, up to n rows, is one seeded draw per equal stratum of the token range, so
    that every part of the prefix-length range is represented.  Sorted, unique."""
    offs = [int(v) for v in torch.as_tensor(q_seq_offsets).tolist()]
    T = offs[-1]
    must = set()
    for b in range(len(offs) - 1):
        if offs[b + 1] > offs[b]:
            must.update((offs[b], offs[b + 1] - 1))
    if chunk:
        for c0 in range(0, T, chunk):
            must.update((c0, min(c0 + chunk, T) - 1))
    if positions is not None:
        pos = torch.as_tensor(positions).to(torch.int64)
        hit = torch.nonzero((pos >= 2046) & (pos <= 2049)).flatten().tolist()
        must.update(hit)
    must = sorted(t for t in must if 0 <= t < T)
    rest = max(0, min(n, T) - len(must))
    g = _gen(seed, 21)
    picked = set(must)
    if rest:
        edges = torch.linspace(0, T, rest + 1).round().to(torch.int64).tolist()
        for i in range(rest):
            lo, hi = edges[i], max(edges[i + 1], edges[i] + 1)
            picked.add(int(torch.randint(lo, min(hi, T), (1,), generator=g)))
    while len(picked) < min(n, T):   # a draw that hit an included row: draw again
        picked.add(int(torch.randint(0, T, (1,), generator=g)))
    return torch.tensor(sorted(picked), dtype=torch.int64)


@dataclass
class MlaBatch:
    q: torch.Tensor              # bf16 [T, H, 576]
    kv: torch.Tensor             # bf16 [rows, 576]
    cache_offsets: torch.Tensor  # int64 [B+1]
    q_seq_offsets: torch.Tensor  # int32 [B+1]
    idx: torch.Tensor            # int32 [T, k_sel], positions in the query's sequence, -1 = none


def make_mla(seed: int, lengths, queries_per_seq, n_heads: int = 96, k_sel: int = 2048, q_std: float = 1.0,
             pad: int = 0, device: str = "cpu") -> MlaBatch:
    """Inputs of the sparse MLA step: sequence b holds lengths[b] cached 576-value rows (bf16
    N(0, 1): the normalised latent and rope key) and queries_per_seq[b] queries (bf16
    N(0, q_std^2) per value).  Each query selects min(k_sel - pad, L_b) distinct positions of
    its sequence in random order (as an unsorted top-k row would hold them); the rest of the
    row is -1.  The cache is drawn on `device` (a large decode cache is drawn on the GPU with
    a seeded CUDA generator); everything else on the CPU."""
    lengths = [int(v) for v in lengths]
    qps = [int(v) for v in queries_per_seq]
    B = len(lengths)
    T = sum(qps)
    cache_offsets = torch.zeros(B + 1, dtype=torch.int64)
    cache_offsets[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0)
    q_seq_offsets = torch.zeros(B + 1, dtype=torch.int32)
    q_seq_offsets[1:] = torch.cumsum(torch.tensor(qps, dtype=torch.int64), 0).to(torch.int32)
    rows = int(cache_offsets[-1])
    q = _normal(_gen(seed, _S_MLA_Q), (T, n_heads, MLA_DIMS["dim"]), q_std).to(torch.bfloat16)
    if device == "cpu":
        kv = _normal(_gen(seed, _S_MLA_KV), (rows, MLA_DIMS["dim"])).to(torch.bfloat16)
    else:
        g = torch.Generator(device=device)
        g.manual_seed((int(seed) * 1_000_003 + _S_MLA_KV * 7919) & 0x7FFF_FFFF_FFFF)
        kv = torch.randn((rows, MLA_DIMS["dim"]), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    idx = torch.full((T, k_sel), -1, dtype=torch.int32)
    g = _gen(seed, _S_MLA_IDX)
    t = 0
    for b in range(B):
        n = min(k_sel - pad, lengths[b])
        for _ in range(qps[b]):
            if n > 0:
                idx[t, :n] = torch.randperm(lengths[b], generator=g)[:n].to(torch.int32)
            t += 1
    return MlaBatch(q, kv, cache_offsets, q_seq_offsets, idx)

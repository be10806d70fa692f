"""CPU oracle of the DSA lightning indexer (Kimi K3.1 Pro) -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
or run this module.  The CUDA library never calls it, and it shares no code with
the CUDA path: it is a plain, slow, obviously-correct restatement of what the
pages define, in float64, with numpy's matmul/sort as library steps.

What it computes (every citation is a row of the component table on the
archdiff.com "compare" pages):

  * 'Sparse / compressed attn' row, Kimi K3.1 Pro column (pages "Qwen3.5-397B-A17B
    vs Kimi K3.1 Pro", "Kimi K3 vs Kimi K3.1 Pro", "Kimi K3.1 Pro vs Gemma 4 31B"):
    32 heads x 128 dims; queries from the 1,536-dim query latent (1,536 -> 4,096);
    one shared 128-dim key from the hidden state with a LayerNorm; per-head
    weights from a 7,168 -> 32 projection; score I = sum_h w_h * ReLU(q_h . k);
    keep the top 2,048 tokens per query; 7.44M parameters per layer.
  * 'QK-Clip and normalized latents; LayerNorm on the indexer key' row: the key
    norm is a LayerNorm (and no per-head norm on q or k).
  * 'Partial RoPE / NoPE' row (page "Kimi K3.1 Pro vs Gemma 4 31B"): the indexer
    sets index_rope_dim = 0, so no rotary encoding touches q or k; positions
    enter only through the causal mask.
  * 'FP8 -> FP4 training' row (page "Kimi K3.1 Pro vs GLM-5"): the indexer is
    BF16; 178.5M indexer parameters over the model (24 layers).
  * 'Long-context extension' row (page "Kimi K3.1 Pro vs Gemma 4 31B"): the
    indexer scores the whole prefix of each query.

Readings where the pages are silent (each is listed in the design notes):
  * causal prefix is inclusive: query at position p scores keys 0..p;
  * no scale factor in I (none is printed);
  * LayerNorm is affine (gamma, beta -- forced by the 7,438,592 count), biased
    variance, eps = 1e-6 unless the caller passes another;
  * q and k are rounded once to bf16 (q after the projection, k after the
    LayerNorm which runs on the unrounded projection); w stays fp32;
  * selection order: score descending, then position ascending; a query whose
    prefix holds at most top_k tokens gets [0, 1, ..., p, -1, -1, ...];
  * sequences are independent (no key from another sequence).

Parity pins for every function live in tests/test_oracle_pins.py.
"""

from __future__ import annotations

import numpy as np

TOP_K = 2048
LN_EPS = 1e-6

# largest finite bf16: (2 - 2^-7) * 2^127
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# --------------------------------------------------------------------------
# bf16 rounding (the pages fix BF16 storage: 'FP8 -> FP4 training' row)
# --------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bf16 keeps 8 significant bits and the float32 exponent range, so a value
    in [2^(e-1), 2^e) is rounded to a multiple of 2^(e-8); below the smallest
    normal (2^-126) the spacing stays 2^-133.  Values that round past the
    largest finite bf16 become +-inf.  Returned as float64 (exact)."""
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0.0)
    v = x[fin]
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    y = np.where(np.abs(y) > BF16_MAX, np.copysign(np.inf, y), y)
    out[fin] = y
    return out


def bf16_bits_to_float64(bits) -> np.ndarray:
    """Interpret uint16 bf16 bit patterns as float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def float64_to_bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns of float64 values that already lie on the bf16 grid."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# parameters ('Sparse / compressed attn' row: 7.44M per layer)
# --------------------------------------------------------------------------

def parameter_shapes(hidden_dim: int = 7168, q_latent_dim: int = 1536,
                     n_heads: int = 32, head_dim: int = 128) -> dict:
    """Every parameter tensor the indexer of one layer owns, as `project` consumes
    them: three bias-free projections stored in x out, and the key LayerNorm's
    gain and bias."""
    return {
        "W_q": (q_latent_dim, n_heads * head_dim),   # 1,536 -> 4,096
        "W_k": (hidden_dim, head_dim),               # hidden -> one shared 128-dim key
        "W_w": (hidden_dim, n_heads),                # 7,168 -> 32 head weights
        "ln_gamma": (head_dim,),
        "ln_beta": (head_dim,),
    }


def parameter_count(**dims) -> int:
    return int(sum(int(np.prod(s)) for s in parameter_shapes(**dims).values()))


# --------------------------------------------------------------------------
# projections (a1, a2 of the hot path)
# --------------------------------------------------------------------------

def layer_norm(x, gamma, beta, eps: float = LN_EPS) -> np.ndarray:
    """Affine LayerNorm over the last axis in float64, biased variance:
    gamma * (x - mean) / sqrt(var + eps) + beta."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def key_norm(raw_keys, gamma, beta, eps: float = LN_EPS) -> np.ndarray:
    """Indexer key from its pre-norm projection: bf16(LayerNorm(raw))."""
    return bf16_round(layer_norm(raw_keys, gamma, beta, eps))


def project_keys(hidden, W_k, gamma, beta, eps: float = LN_EPS) -> np.ndarray:
    """The key path of `project` alone: k = bf16(LayerNorm(hidden @ W_k)) in float64."""
    return key_norm(np.asarray(hidden, np.float64) @ np.asarray(W_k, np.float64), gamma, beta, eps)


def rope(x, positions, rope_dim: int, theta: float = 10000.0) -> np.ndarray:
    """Rotary encoding of the first rope_dim dims of the last axis: for i < rope_dim / 2 the
    pair (x[2i], x[2i+1]) is rotated by the angle p * theta^(-2i / rope_dim), p the row's
    position; the other dims pass unchanged.  positions broadcast against x's leading axes
    (one per row).  DeepSeek-V3.2's indexer rotates 64 of its 128 dims ('Partial RoPE /
    NoPE' row, page "Kimi K3.1 Pro vs Gemma 4 31B"); Kimi K3.1's rotates none."""
    x = np.array(x, dtype=np.float64, copy=True)
    if rope_dim == 0:
        return x
    i = np.arange(rope_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / rope_dim)
    ang = np.asarray(positions, np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., 0:rope_dim:2].copy()
    b = x[..., 1:rope_dim:2].copy()
    x[..., 0:rope_dim:2] = a * c - b * s
    x[..., 1:rope_dim:2] = a * s + b * c
    return x


def project(hidden, q_latent, W_q, W_k, W_w, gamma, beta, eps: float = LN_EPS,
            n_heads: int = 32, head_dim: int = 128, positions=None, rope_dim: int = 0,
            rope_theta: float = 10000.0):
    """Indexer projections of T tokens.

    q = bf16(RoPE(q_latent @ W_q)) viewed [T, n_heads, head_dim] (head h = columns
        h*head_dim .. h*head_dim + head_dim - 1);
    k = bf16(RoPE(LayerNorm(hidden @ W_k)));
    w = fp32(hidden @ W_w).
    RoPE (rope_dim > 0, the DeepSeek-V3.2 form; needs `positions`) rotates the first
    rope_dim dims of every head of q and of k by the token's position; with rope_dim = 0
    (Kimi K3.1) there is no rotary step.  All products and sums in float64; one rounding
    per output."""
    hidden = np.asarray(hidden, np.float64)
    q_latent = np.asarray(q_latent, np.float64)
    shapes = parameter_shapes(hidden.shape[1], q_latent.shape[1], n_heads, head_dim)
    for name, arr in (("W_q", W_q), ("W_k", W_k), ("W_w", W_w), ("ln_gamma", gamma), ("ln_beta", beta)):
        if tuple(np.shape(arr)) != shapes[name]:
            raise ValueError(f"{name} has shape {np.shape(arr)}, expected {shapes[name]}")
    T = hidden.shape[0]
    if rope_dim:
        if positions is None:
            raise ValueError("rope_dim > 0 needs the token positions")
        pos = np.asarray(positions, np.float64)
        q = bf16_round(rope((q_latent @ np.asarray(W_q, np.float64)).reshape(T, n_heads, head_dim),
                            pos[:, None], rope_dim, rope_theta))
        k = bf16_round(rope(layer_norm(hidden @ np.asarray(W_k, np.float64), gamma, beta, eps), pos, rope_dim,
                            rope_theta))
    else:
        q = bf16_round(q_latent @ np.asarray(W_q, np.float64)).reshape(T, n_heads, head_dim)
        k = project_keys(hidden, W_k, gamma, beta, eps)
    w = (hidden @ np.asarray(W_w, np.float64)).astype(np.float32).astype(np.float64)
    return q, k, w


# --------------------------------------------------------------------------
# score and selection (a3, a4, a5 of the hot path)
# --------------------------------------------------------------------------

def index_scores(q_t, w_t, keys):
    """Scores of one query against keys [n, D]:
        I[s] = sum_h w_h * max(0, q_h . k_s)
    and the tolerance scale A[s] = sum_h |w_h * (q_h . k_s)|."""
    logits = np.asarray(keys, np.float64) @ np.asarray(q_t, np.float64).T   # [n, H]
    w_t = np.asarray(w_t, np.float64)
    I = np.maximum(logits, 0.0) @ w_t
    A = np.abs(logits) @ np.abs(w_t)
    return I, A


def select_topk(I, top_k: int = TOP_K):
    """Indices kept for one query whose prefix scores are I[0..n-1].

    n <= top_k: every position, in position order, then -1 padding.
    n  > top_k: the top_k positions by (score descending, position ascending),
                in that order."""
    I = np.asarray(I, np.float64)
    n = I.shape[0]
    if n <= top_k:
        return np.concatenate([np.arange(n, dtype=np.int64), -np.ones(top_k - n, dtype=np.int64)])
    order = np.lexsort((np.arange(n), -I))
    return order[:top_k].astype(np.int64)


def sequence_of(q_seq_offsets, T):
    """Sequence id of each of the T query tokens from the cu_seqlens offsets."""
    offs = np.asarray(q_seq_offsets, np.int64)
    seq = np.empty(T, dtype=np.int64)
    for b in range(len(offs) - 1):
        seq[offs[b]:offs[b + 1]] = b
    return seq


def topk(q, w, positions, q_seq_offsets, key_cache, cache_offsets, top_k: int = TOP_K,
         rows=None, keep_scores: bool = False):
    """Top-k of every (or every listed) query token.

    q [T, H, D], w [T, H], key_cache [rows, D] (float64 holding bf16 values).
    Query t of sequence b at position p scores the keys
    key_cache[cache_offsets[b] + s] for s = 0..p.

    Returns (idx [R, top_k] int64, score [R, top_k] float64 with -inf in the
    padding) for the R selected rows; with keep_scores, also the per-row lists
    of I and A over the whole prefix."""
    q = np.asarray(q, np.float64)
    w = np.asarray(w, np.float64)
    positions = np.asarray(positions, np.int64)
    cache_offsets = np.asarray(cache_offsets, np.int64)
    T = q.shape[0]
    seq = sequence_of(q_seq_offsets, T)
    rows = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    idx = np.empty((len(rows), top_k), dtype=np.int64)
    score = np.empty((len(rows), top_k), dtype=np.float64)
    all_I, all_A = [], []
    for r, t in enumerate(rows):
        b = seq[t]
        p = positions[t]
        base = cache_offsets[b]
        if p < 0 or base + p >= cache_offsets[b + 1]:
            raise ValueError(f"query {t}: position {p} outside its sequence's cache rows")
        keys = key_cache[base: base + p + 1]
        I, A = index_scores(q[t], w[t], keys)
        sel = select_topk(I, top_k)
        idx[r] = sel
        score[r] = np.where(sel >= 0, I[np.maximum(sel, 0)], -np.inf)
        if keep_scores:
            all_I.append(I)
            all_A.append(A)
    if keep_scores:
        return idx, score, all_I, all_A
    return idx, score


def sort_selected(idx_row, I):
    """The DSA_SORTED order of one row: score descending, position ascending,
    padding (-1) last."""
    idx_row = np.asarray(idx_row, np.int64)
    valid = idx_row[idx_row >= 0]
    order = np.lexsort((valid, -np.asarray(I, np.float64)[valid]))
    out = -np.ones_like(idx_row)
    out[: len(valid)] = valid[order]
    return out


# --------------------------------------------------------------------------
# index reuse across speculative draft steps
# --------------------------------------------------------------------------

def reuse_topk(idx, score, anchor_rows):
    """Selections of speculative draft tokens ('MTP' row, page "Kimi K3.1 Pro vs GLM-5":
    GLM-5.2 reuses the first step's top-k indices in its later draft steps).

    idx [n_src, top_k] and score [n_src, top_k] are the first step's selections; draft
    token d takes row anchor_rows[d] unchanged.  An anchor outside [0, n_src) has no
    selection to reuse: its row is all padding (-1, -inf)."""
    idx = np.asarray(idx)
    score = np.asarray(score, np.float64)
    a = np.asarray(anchor_rows, np.int64)
    n_src, k = idx.shape
    ok = (a >= 0) & (a < n_src)
    out_i = np.full((len(a), k), -1, dtype=np.int64)
    out_s = np.full((len(a), k), -np.inf)
    out_i[ok] = idx[a[ok]]
    out_s[ok] = score[a[ok]]
    return out_i, out_s


# --------------------------------------------------------------------------
# FP8 indexer-key cache ('FP8 -> FP4 training' row, page "Kimi K3.1 Pro vs GLM-5":
# vLLM and SGLang cache the indexer keys in FP8 by default)
# --------------------------------------------------------------------------

E4M3_MAX = 448.0   # largest finite e4m3 value: 2^8 * 1.75


def e4m3_round(x) -> np.ndarray:
    """Round values to the nearest FP8 e4m3 value (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits; no infinities), ties to even, saturating at +-448.  A value in
    [2^(e-1), 2^e) with e - 1 >= -6 is rounded to a multiple of 2^(e-4); below 2^-6 the
    spacing stays 2^-9 (subnormals).  Returned as float64 (exact)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0.0) & np.isfinite(x)
    v = x[nz]
    _, e = np.frexp(v)                   # |v| in [2^(e-1), 2^e)
    q = np.maximum(e - 4, -9)
    y = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    out[nz] = np.clip(y, -E4M3_MAX, E4M3_MAX)
    return out


def quantize_fp8(v, axis: int = -1):
    """FP8 e4m3 codes and fp32 scale of rows of float32-representable values, one scale per
    row (the pages fix no granularity; one scale per 128-value key row, and per head of a
    query, is the reading taken):
        amax  = max |v| over the row
        scale = fp32(amax / 448),  inv = fp32(448 / amax)      (both 0 when amax = 0)
        code  = e4m3(fp32(v * inv))
    so that code * scale approximates v.  Every operation is a single float32 rounding, as
    on the device.  Returns (codes as float64 on the e4m3 grid, scale as float64)."""
    v = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v), axis=axis, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(0))
        inv = np.where(amax > 0, (np.float32(E4M3_MAX) / amax).astype(np.float32), np.float32(0))
    prod = (v * inv).astype(np.float32)
    codes = e4m3_round(prod.astype(np.float64))
    return codes, np.squeeze(scale, axis=axis).astype(np.float64)


def fp8_index_scores(q8_t, sq_t, w_t, k8, sk):
    """Scores of one query against FP8 keys: with q_h ~ q8_h * sq_h and k_s ~ k8_s * sk_s
    (positive scales),
        I[s] = sum_h w_h * max(0, (q8_h sq_h) . (k8_s sk_s))
             = sk_s * sum_h (w_h sq_h) * max(0, q8_h . k8_s),
    and the tolerance scale A[s] = sk_s * sum_h |w_h sq_h| |q8_h . k8_s|."""
    logits = np.asarray(k8, np.float64) @ np.asarray(q8_t, np.float64).T          # [n, H]
    wq = np.asarray(w_t, np.float64) * np.asarray(sq_t, np.float64)
    sk = np.asarray(sk, np.float64)
    I = sk * (np.maximum(logits, 0.0) @ wq)
    A = sk * (np.abs(logits) @ np.abs(wq))
    return I, A


def topk_fp8(q8, sq, w, positions, q_seq_offsets, k8, sk, cache_offsets, top_k: int = TOP_K, rows=None,
             keep_scores: bool = False):
    """As topk, over FP8 queries q8 [T, H, D] with per-head scales sq [T, H] and FP8 keys
    k8 [rows, D] with per-row scales sk [rows]."""
    q8 = np.asarray(q8, np.float64)
    positions = np.asarray(positions, np.int64)
    cache_offsets = np.asarray(cache_offsets, np.int64)
    T = q8.shape[0]
    seq = sequence_of(q_seq_offsets, T)
    rows = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    idx = np.empty((len(rows), top_k), dtype=np.int64)
    score = np.empty((len(rows), top_k), dtype=np.float64)
    all_I, all_A = [], []
    for r, t in enumerate(rows):
        b = seq[t]
        p = positions[t]
        base = cache_offsets[b]
        if p < 0 or base + p >= cache_offsets[b + 1]:
            raise ValueError(f"query {t}: position {p} outside its sequence's cache rows")
        I, A = fp8_index_scores(q8[t], sq[t], w[t], k8[base: base + p + 1], sk[base: base + p + 1])
        sel = select_topk(I, top_k)
        idx[r] = sel
        score[r] = np.where(sel >= 0, I[np.maximum(sel, 0)], -np.inf)
        if keep_scores:
            all_I.append(I)
            all_A.append(A)
    if keep_scores:
        return idx, score, all_I, all_A
    return idx, score

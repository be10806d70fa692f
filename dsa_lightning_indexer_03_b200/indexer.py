"""Python binding of the C ABI: argument marshalling only.

torch supplies device memory and the CUDA stream; every step of the indexer
(projections, key LayerNorm, score, masking, top-k) runs in libdsa_indexer.so.
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import check


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Indexer:
    """One layer's DSA lightning indexer (owns a C handle)."""

    def __init__(self, W_q: torch.Tensor, W_k: torch.Tensor, W_w: torch.Tensor, ln_gamma: torch.Tensor,
                 ln_beta: torch.Tensor, *, ln_eps: float = 1e-6, max_tokens: int = 131072, rope_dim: int = 0,
                 rope_theta: float = 10000.0):
        """The head count comes from W_w ([hidden, n_heads]: 32, or 64 for the DeepSeek-V3.2
        form); rope_dim = 64 adds that form's rotary step on the first 64 dims of q and k."""
        self._lib = _lib.load()
        dev = W_q.device
        if dev.type != "cuda":
            raise ValueError("weights must live on a CUDA device")
        for name, t in (("W_q", W_q), ("W_k", W_k), ("W_w", W_w), ("ln_gamma", ln_gamma), ("ln_beta", ln_beta)):
            _need(t, name, torch.bfloat16, dev)
        cfg = _lib.Config()
        self._lib.dsa_indexer_default_config(ctypes.byref(cfg))
        cfg.hidden_dim = W_k.shape[0]
        cfg.q_latent_dim = W_q.shape[0]
        cfg.n_heads = W_w.shape[1]
        cfg.head_dim = W_k.shape[1]
        cfg.ln_eps = float(ln_eps)
        cfg.max_tokens = int(max_tokens)
        cfg.rope_dim = int(rope_dim)
        cfg.rope_theta = float(rope_theta)
        self.cfg = cfg
        self.device = dev
        self.n_heads = cfg.n_heads
        self.head_dim = cfg.head_dim
        self.top_k = cfg.top_k
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            check(self._lib.dsa_indexer_create(ctypes.byref(cfg), _ptr(W_q), _ptr(W_k), _ptr(W_w), _ptr(ln_gamma),
                                               _ptr(ln_beta), ctypes.byref(h)), "dsa_indexer_create")
        self._h = h

    # ------------------------------------------------------------------ life cycle
    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            with torch.cuda.device(self.device):
                self._lib.dsa_indexer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ------------------------------------------------------------------ entry points
    def project(self, hidden, q_latent, positions, q_seq_offsets, key_cache, cache_offsets, q_out=None, w_out=None,
                stream=None):
        """q [T, n_heads, head_dim] bf16 and w [T, n_heads] fp32; writes each token's key
        into key_cache[cache_offsets[b] + positions[t]]."""
        dev = self.device
        T = hidden.shape[0]
        _need(hidden, "hidden", torch.bfloat16, dev)
        _need(q_latent, "q_latent", torch.bfloat16, dev)
        _need(positions, "positions", torch.int32, dev)
        _need(q_seq_offsets, "q_seq_offsets", torch.int32, dev)
        _need(key_cache, "key_cache", torch.bfloat16, dev)
        _need(cache_offsets, "cache_offsets", torch.int64, dev)
        if q_out is None:
            q_out = torch.empty((T, self.n_heads, self.head_dim), dtype=torch.bfloat16, device=dev)
        if w_out is None:
            w_out = torch.empty((T, self.n_heads), dtype=torch.float32, device=dev)
        _need(q_out, "q_out", torch.bfloat16, dev)
        _need(w_out, "w_out", torch.float32, dev)
        B = q_seq_offsets.numel() - 1
        check(self._lib.dsa_indexer_project(self._h, T, _ptr(hidden), _ptr(q_latent), _ptr(positions),
                                            _ptr(q_seq_offsets), B, _ptr(key_cache), key_cache.shape[0],
                                            _ptr(cache_offsets), _ptr(q_out), _ptr(w_out), _stream(stream)),
              "dsa_indexer_project")
        return q_out, w_out

    def key_norm(self, raw_keys, out=None, stream=None):
        """bf16 LayerNorm of pre-norm key rows raw_keys [n, head_dim] fp32."""
        dev = self.device
        _need(raw_keys, "raw_keys", torch.float32, dev)
        n = raw_keys.shape[0]
        if out is None:
            out = torch.empty((n, self.head_dim), dtype=torch.bfloat16, device=dev)
        _need(out, "out", torch.bfloat16, dev)
        check(self._lib.dsa_indexer_key_norm(self._h, n, _ptr(raw_keys), _ptr(out), _stream(stream)),
              "dsa_indexer_key_norm")
        return out

    def topk(self, q, w, positions, q_seq_offsets, key_cache, cache_offsets, idx_out=None, score_out=None,
             return_scores: bool = True, flags: int = 0, stream=None):
        """idx [T, top_k] int32 (and scores [T, top_k] fp32 when requested)."""
        dev = self.device
        T = q.shape[0]
        _need(q, "q", torch.bfloat16, dev)
        _need(w, "w", torch.float32, dev)
        _need(positions, "positions", torch.int32, dev)
        _need(q_seq_offsets, "q_seq_offsets", torch.int32, dev)
        _need(key_cache, "key_cache", torch.bfloat16, dev)
        _need(cache_offsets, "cache_offsets", torch.int64, dev)
        if idx_out is None:
            idx_out = torch.empty((T, self.top_k), dtype=torch.int32, device=dev)
        _need(idx_out, "idx_out", torch.int32, dev)
        if score_out is None and return_scores:
            score_out = torch.empty((T, self.top_k), dtype=torch.float32, device=dev)
        if score_out is not None:
            _need(score_out, "score_out", torch.float32, dev)
        B = q_seq_offsets.numel() - 1
        check(self._lib.dsa_indexer_topk(self._h, T, _ptr(q), _ptr(w), _ptr(positions), _ptr(q_seq_offsets), B,
                                         _ptr(key_cache), key_cache.shape[0], _ptr(cache_offsets), _ptr(idx_out),
                                         _ptr(score_out), int(flags), _stream(stream)),
              "dsa_indexer_topk")
        return idx_out, score_out

    # ------------------------------------------------------------------ FP8 key cache
    def project_fp8(self, hidden, q_latent, positions, q_seq_offsets, key_cache_fp8, key_scale, cache_offsets,
                    q_out=None, q_scale=None, w_out=None, stream=None):
        """FP8 projections: e4m3 codes q [T, n_heads, head_dim] (uint8) with per-head scales
        [T, n_heads] and w [T, n_heads] fp32; each token's key goes to key_cache_fp8 (uint8
        [rows, head_dim]) with its scale in key_scale (fp32 [rows])."""
        dev = self.device
        T = hidden.shape[0]
        _need(hidden, "hidden", torch.bfloat16, dev)
        _need(q_latent, "q_latent", torch.bfloat16, dev)
        _need(positions, "positions", torch.int32, dev)
        _need(q_seq_offsets, "q_seq_offsets", torch.int32, dev)
        _need(key_cache_fp8, "key_cache_fp8", torch.uint8, dev)
        _need(key_scale, "key_scale", torch.float32, dev)
        _need(cache_offsets, "cache_offsets", torch.int64, dev)
        if q_out is None:
            q_out = torch.empty((T, self.n_heads, self.head_dim), dtype=torch.uint8, device=dev)
        if q_scale is None:
            q_scale = torch.empty((T, self.n_heads), dtype=torch.float32, device=dev)
        if w_out is None:
            w_out = torch.empty((T, self.n_heads), dtype=torch.float32, device=dev)
        _need(q_out, "q_out", torch.uint8, dev)
        _need(q_scale, "q_scale", torch.float32, dev)
        _need(w_out, "w_out", torch.float32, dev)
        B = q_seq_offsets.numel() - 1
        check(self._lib.dsa_indexer_project_fp8(self._h, T, _ptr(hidden), _ptr(q_latent), _ptr(positions),
                                                _ptr(q_seq_offsets), B, _ptr(key_cache_fp8), _ptr(key_scale),
                                                key_cache_fp8.shape[0], _ptr(cache_offsets), _ptr(q_out),
                                                _ptr(q_scale), _ptr(w_out), _stream(stream)),
              "dsa_indexer_project_fp8")
        return q_out, q_scale, w_out

    def quantize_keys_fp8(self, keys, out=None, scale=None, stream=None):
        """FP8 codes (uint8 [n, head_dim]) and per-row scales (fp32 [n]) of bf16 key rows."""
        dev = self.device
        _need(keys, "keys", torch.bfloat16, dev)
        n = keys.shape[0]
        if out is None:
            out = torch.empty((n, self.head_dim), dtype=torch.uint8, device=dev)
        if scale is None:
            scale = torch.empty((n,), dtype=torch.float32, device=dev)
        _need(out, "out", torch.uint8, dev)
        _need(scale, "scale", torch.float32, dev)
        check(self._lib.dsa_indexer_quantize_keys_fp8(self._h, n, _ptr(keys), _ptr(out), _ptr(scale),
                                                      _stream(stream)), "dsa_indexer_quantize_keys_fp8")
        return out, scale

    def topk_fp8(self, q, q_scale, w, positions, q_seq_offsets, key_cache_fp8, key_scale, cache_offsets,
                 idx_out=None, score_out=None, return_scores: bool = True, flags: int = 0, stream=None):
        """topk over FP8 queries and an FP8 key cache."""
        dev = self.device
        T = q.shape[0]
        _need(q, "q", torch.uint8, dev)
        _need(q_scale, "q_scale", torch.float32, dev)
        _need(w, "w", torch.float32, dev)
        _need(positions, "positions", torch.int32, dev)
        _need(q_seq_offsets, "q_seq_offsets", torch.int32, dev)
        _need(key_cache_fp8, "key_cache_fp8", torch.uint8, dev)
        _need(key_scale, "key_scale", torch.float32, dev)
        _need(cache_offsets, "cache_offsets", torch.int64, dev)
        if idx_out is None:
            idx_out = torch.empty((T, self.top_k), dtype=torch.int32, device=dev)
        _need(idx_out, "idx_out", torch.int32, dev)
        if score_out is None and return_scores:
            score_out = torch.empty((T, self.top_k), dtype=torch.float32, device=dev)
        if score_out is not None:
            _need(score_out, "score_out", torch.float32, dev)
        B = q_seq_offsets.numel() - 1
        check(self._lib.dsa_indexer_topk_fp8(self._h, T, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(positions),
                                             _ptr(q_seq_offsets), B, _ptr(key_cache_fp8), _ptr(key_scale),
                                             key_cache_fp8.shape[0], _ptr(cache_offsets), _ptr(idx_out),
                                             _ptr(score_out), int(flags), _stream(stream)),
              "dsa_indexer_topk_fp8")
        return idx_out, score_out

    def topk_reuse(self, anchor_rows, src_idx, src_score=None, idx_out=None, score_out=None, stream=None):
        """Rows of earlier dsa_indexer_topk results reused by speculative draft tokens: row d of
        the output is row anchor_rows[d] of src_idx (and src_score, when given)."""
        dev = self.device
        _need(anchor_rows, "anchor_rows", torch.int32, dev)
        _need(src_idx, "src_idx", torch.int32, dev)
        n = anchor_rows.numel()
        if idx_out is None:
            idx_out = torch.empty((n, self.top_k), dtype=torch.int32, device=dev)
        _need(idx_out, "idx_out", torch.int32, dev)
        if src_score is not None:
            _need(src_score, "src_score", torch.float32, dev)
            if score_out is None:
                score_out = torch.empty((n, self.top_k), dtype=torch.float32, device=dev)
        if score_out is not None:
            _need(score_out, "score_out", torch.float32, dev)
        check(self._lib.dsa_indexer_topk_reuse(self._h, n, _ptr(anchor_rows), src_idx.shape[0], _ptr(src_idx),
                                               _ptr(src_score), _ptr(idx_out), _ptr(score_out), _stream(stream)),
              "dsa_indexer_topk_reuse")
        return idx_out, score_out

    def sparse_mla(self, q, kv_cache, cache_offsets, q_seq_offsets, idx, scale, out=None, lse=None, stream=None):
        """Attention of each query (q bf16 [T, H, 576]) over the kv_cache rows (bf16 [rows, 576])
        its idx row selects (int32 [T, k_sel], positions in its sequence, -1 = none), latent
        form: returns out bf16 [T, H, 512] and lse fp32 [T, H]."""
        dev = self.device
        _need(q, "q", torch.bfloat16, dev)
        _need(kv_cache, "kv_cache", torch.bfloat16, dev)
        _need(cache_offsets, "cache_offsets", torch.int64, dev)
        _need(q_seq_offsets, "q_seq_offsets", torch.int32, dev)
        _need(idx, "idx", torch.int32, dev)
        if q.dim() != 3 or q.shape[2] != 576 or kv_cache.dim() != 2 or kv_cache.shape[1] != 576:
            raise ValueError("q must be [T, H, 576] and kv_cache [rows, 576]")
        T, H = q.shape[0], q.shape[1]
        if idx.dim() != 2 or idx.shape[0] != T:
            raise ValueError("idx must be [T, k_sel]")
        if out is None:
            out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((T, H), dtype=torch.float32, device=dev)
        _need(out, "out", torch.bfloat16, dev)
        _need(lse, "lse", torch.float32, dev)
        check(self._lib.dsa_indexer_sparse_mla(self._h, T, _ptr(q), H, _ptr(kv_cache), kv_cache.shape[0],
                                               _ptr(cache_offsets), _ptr(q_seq_offsets), cache_offsets.numel() - 1,
                                               _ptr(idx), idx.shape[1], float(scale), _ptr(out), _ptr(lse),
                                               _stream(stream)),
              "dsa_indexer_sparse_mla")
        return out, lse

    def device_error(self) -> int:
        """Synchronises and returns (then clears) the handle's device error status."""
        with torch.cuda.device(self.device):
            return int(self._lib.dsa_indexer_device_error(self._h))


def selftest_wait_timeout(timeout_ns: int, stream=None) -> int:
    """Runs the bounded-wait self test; returns the status code (6 = timeout seen)."""
    lib = _lib.load()
    return int(lib.dsa_indexer_selftest_wait_timeout(int(timeout_ns), _stream(stream)))

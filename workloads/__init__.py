"""Seeded synthetic inputs for the DSA lightning indexer.

This module is shared by the CPU oracle tests, the CUDA parity tests and the
benchmark.  It holds random draws and bookkeeping (shapes, offsets, positions)
only: none of the indexer's arithmetic (no projection, no LayerNorm, no score,
no selection) lives here.  Every tensor is a CPU torch tensor; bf16 inputs are
drawn in fp32 and rounded to bf16 by torch's own conversion.

Workloads follow the indexer described on the archdiff.com "compare" pages for
Kimi K3.1 Pro ('Sparse / compressed attn' row): a 7,168-wide hidden state, a
1,536-dim query latent, 32 heads x 128 dims, top 2,048.
"""

from .generate import (  # noqa: F401
    MODEL_DIMS,
    WORKLOADS,
    Weights,
    PrefillBatch,
    DecodeBatch,
    make_weights,
    make_prefill,
    make_decode,
    decode_lengths,
    heavy_hitter_rows,
    causal_pairs,
    make_scoring_inputs,
    stratified_rows,
    MLA_DIMS,
    MlaBatch,
    make_mla,
)

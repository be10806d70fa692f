"""CPU oracle of the DSA lightning indexer -- test infrastructure.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  It shares no code with the CUDA library.
"""

from .indexer_oracle import (  # noqa: F401
    TOP_K,
    LN_EPS,
    bf16_round,
    bf16_bits_to_float64,
    float64_to_bf16_bits,
    parameter_shapes,
    parameter_count,
    layer_norm,
    key_norm,
    rope,
    project,
    project_keys,
    index_scores,
    select_topk,
    sequence_of,
    topk,
    sort_selected,
    reuse_topk,
    E4M3_MAX,
    e4m3_round,
    quantize_fp8,
    fp8_index_scores,
    topk_fp8,
)
from .sparse_mla_oracle import (  # noqa: F401
    MLA_HEADS,
    MLA_DIM,
    MLA_LATENT,
    sparse_mla,
)

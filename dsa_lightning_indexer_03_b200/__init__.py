"""B200 (sm_100a) DSA lightning indexer: C-ABI library + thin Python binding.

The compute path lives in libdsa_indexer.so (built by `build.py`); this package
only marshals torch tensors into its entry points.
"""

from ._lib import (  # noqa: F401
    DSA_OK,
    DSA_ERR_INVALID_ARG,
    DSA_ERR_UNSUPPORTED,
    DSA_ERR_CUDA,
    DSA_ERR_OOM,
    DSA_ERR_WORKSPACE,
    DSA_ERR_DEVICE_TIMEOUT,
    DSA_ERR_DEVICE_BOUNDS,
    DSA_TOPK_SORTED,
    DSA_TOPK_SPLIT,
    DSA_TOPK_NO_SPLIT,
    DSAError,
    LIB_PATH,
    load,
)
from .indexer import Indexer, selftest_wait_timeout  # noqa: F401

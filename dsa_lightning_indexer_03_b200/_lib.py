"""ctypes view of libdsa_indexer.so (the C ABI in include/dsa_indexer.h).

Loading fails loudly if the library has not been built: there is no fallback
implementation of any step.
"""

from __future__ import annotations

import ctypes
import os

LIB_NAME = "libdsa_indexer.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), LIB_NAME)

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_CUDA = 3
DSA_ERR_OOM = 4
DSA_ERR_WORKSPACE = 5
DSA_ERR_DEVICE_TIMEOUT = 6
DSA_ERR_DEVICE_BOUNDS = 7

DSA_TOPK_SORTED = 1
DSA_TOPK_SPLIT = 2
DSA_TOPK_NO_SPLIT = 4


class Config(ctypes.Structure):
    _fields_ = [
        ("hidden_dim", ctypes.c_int32),
        ("q_latent_dim", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("ln_eps", ctypes.c_float),
        ("max_tokens", ctypes.c_int64),
        ("rope_dim", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
    ]


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_u32 = ctypes.c_uint32

# name -> (restype, argtypes)
SIGNATURES = {
    "dsa_indexer_default_config": (None, [ctypes.POINTER(Config)]),
    "dsa_indexer_create": (ctypes.c_int, [ctypes.POINTER(Config), _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "dsa_indexer_destroy": (ctypes.c_int, [_vp]),
    "dsa_indexer_project": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _vp, _i64, _vp, _vp, _vp, _vp]),
    "dsa_indexer_key_norm": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp]),
    "dsa_indexer_topk": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _vp, _i64, _vp, _vp, _vp, _u32, _vp]),
    "dsa_indexer_topk_noalloc": (ctypes.c_int, [_i64, _vp, _vp, _vp, _vp, _i32, _vp, _i64, _vp, _vp, _vp, _vp]),
    "dsa_indexer_project_fp8": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i64, _vp, _vp, _vp,
                                                _vp, _vp]),
    "dsa_indexer_quantize_keys_fp8": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp, _vp]),
    "dsa_indexer_topk_fp8": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i64, _vp, _vp, _vp,
                                             _u32, _vp]),
    "dsa_indexer_topk_reuse": (ctypes.c_int, [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp]),
    "dsa_indexer_sparse_mla": (ctypes.c_int, [_vp, _i64, _vp, _i32, _vp, _i64, _vp, _vp, _i32, _vp, _i32,
                                              ctypes.c_float, _vp, _vp, _vp]),
    "dsa_indexer_device_error": (ctypes.c_int, [_vp]),
    "dsa_indexer_noalloc_device_error": (ctypes.c_int, [_vp]),
    "dsa_indexer_selftest_wait_timeout": (ctypes.c_int, [_i64, _vp]),
    "dsa_indexer_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dsa_indexer_abi_version": (ctypes.c_int32, []),
}

_LIB = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Loads (once) and returns the library with every signature declared."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{LIB_NAME} is not built (expected at {p}); run "
            "`python -m dsa_lightning_indexer_03_b200.build` -- there is no fallback path")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _LIB = lib
    return lib


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = load().dsa_indexer_status_string(status).decode()
        super().__init__(f"{where}: {name} ({status})")


def check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DSAError(status, where)

"""The C-ABI library loads without a GPU, exports every entry point the header
declares, and rejects bad arguments before touching CUDA.  CPU only."""

import ctypes
import os
import re

import pytest

from dsa_lightning_indexer_03_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa_indexer.h")


@pytest.fixture(scope="module")
def lib():
    path = B.build()
    from dsa_lightning_indexer_03_b200 import _lib
    return _lib.load(path)


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"#define[^\n]*", "", text)
    return sorted(set(re.findall(r"\b(dsa_indexer_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("dsa_indexer_create", "dsa_indexer_project", "dsa_indexer_topk", "dsa_indexer_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from dsa_lightning_indexer_03_b200 import _lib
    for name in _declared():
        assert hasattr(lib, name), f"{name} is declared in the header but not exported"
        assert name in _lib.SIGNATURES, f"{name} has no binding signature"


def test_library_has_no_cuda_driver_link_dependency():
    # the library reaches the driver through the runtime's entry-point query, so it
    # loads on machines without a GPU driver
    import subprocess
    out = subprocess.run(["ldd", B.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings_and_version(lib):
    assert lib.dsa_indexer_abi_version() == 2
    assert lib.dsa_indexer_status_string(0) == b"DSA_OK"
    assert lib.dsa_indexer_status_string(5) == b"DSA_ERR_WORKSPACE"
    assert lib.dsa_indexer_status_string(99) == b"DSA_ERR_UNKNOWN"


def test_default_config_is_the_k31_indexer(lib):
    from dsa_lightning_indexer_03_b200 import _lib
    cfg = _lib.Config()
    lib.dsa_indexer_default_config(ctypes.byref(cfg))
    assert (cfg.hidden_dim, cfg.q_latent_dim, cfg.n_heads, cfg.head_dim, cfg.top_k) == (7168, 1536, 32, 128, 2048)
    assert abs(cfg.ln_eps - 1e-6) < 1e-12
    assert cfg.rope_dim == 0 and cfg.rope_theta == 10000.0 and cfg.max_tokens == 131072


def test_argument_validation_without_a_gpu(lib):
    from dsa_lightning_indexer_03_b200 import _lib
    cfg = _lib.Config()
    lib.dsa_indexer_default_config(ctypes.byref(cfg))
    h = ctypes.c_void_p(123)
    # NULL weights
    assert lib.dsa_indexer_create(ctypes.byref(cfg), None, None, None, None, None, ctypes.byref(h)) == 1
    assert h.value is None
    # unsupported head count or rotary width (checked before any weight is read)
    fake = ctypes.c_void_p(0x1000)
    cfg.n_heads = 48
    assert lib.dsa_indexer_create(ctypes.byref(cfg), fake, fake, fake, fake, fake, ctypes.byref(h)) == 2
    cfg.n_heads = 64
    cfg.rope_dim = 32
    assert lib.dsa_indexer_create(ctypes.byref(cfg), fake, fake, fake, fake, fake, ctypes.byref(h)) == 2
    cfg.rope_dim = 64
    cfg.rope_theta = 0.5     # a rotary base must exceed 1
    assert lib.dsa_indexer_create(ctypes.byref(cfg), fake, fake, fake, fake, fake, ctypes.byref(h)) == 1
    cfg.n_heads, cfg.rope_dim, cfg.rope_theta = 32, 0, 10000.0
    cfg.hidden_dim = 7100   # not a multiple of 64
    assert lib.dsa_indexer_create(ctypes.byref(cfg), fake, fake, fake, fake, fake, ctypes.byref(h)) == 1
    # NULL handle on every call
    assert lib.dsa_indexer_project(None, 1, *([None] * 4), 1, None, 1, None, None, None, None) == 1
    assert lib.dsa_indexer_topk(None, 1, *([None] * 4), 1, None, 1, None, None, None, 0, None) == 1
    assert lib.dsa_indexer_key_norm(None, 1, None, None, None) == 1
    assert lib.dsa_indexer_project_fp8(None, 1, *([None] * 4), 1, None, None, 1, None, None, None, None, None) == 1
    assert lib.dsa_indexer_topk_fp8(None, 1, *([None] * 5), 1, None, None, 1, None, None, None, 0, None) == 1
    assert lib.dsa_indexer_quantize_keys_fp8(None, 1, None, None, None, None) == 1
    assert lib.dsa_indexer_topk_reuse(None, 1, None, 1, None, None, None, None, None) == 1
    assert lib.dsa_indexer_sparse_mla(None, 1, None, 96, None, 1, None, None, 1, None, 2048, 0.07, None, None,
                                      None) == 1
    assert lib.dsa_indexer_destroy(None) == 1
    assert lib.dsa_indexer_device_error(None) == 1
    assert lib.dsa_indexer_selftest_wait_timeout(0, None) == 1


def test_binding_fails_loudly_without_the_library(tmp_path):
    from dsa_lightning_indexer_03_b200 import _lib
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load(str(tmp_path / "missing.so"))

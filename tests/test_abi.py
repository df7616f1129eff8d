"""The C-ABI library loads and exports what include/mlra.h declares (no GPU needed).

Only host-side argument checks are exercised here: they return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import rank_latent_kv_mlra_b200 as M
from rank_latent_kv_mlra_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mlra.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return M.load_library()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mlra_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ["mlra_create", "mlra_decode", "mlra_append_cache", "mlra_destroy"]:
        assert required in names
    assert all(n.isascii() for n in names)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_exported_dynamic_symbols_are_ascii():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True).stdout
    syms = [l.split()[-1] for l in out.splitlines() if " T " in l and "mlra_" in l]
    assert syms and all(s.isascii() for s in syms)
    assert set(_declared()) <= set(syms)


def test_status_strings(lib):
    for code in M.STATUS:
        assert M.mlra_status_string(code) != "unknown status"
    assert M.mlra_status_string(12345) == "unknown status"


def test_host_argument_checks_return_codes(lib):
    P = ctypes.c_void_p
    out = P()
    cfg = M.mlra_config(128, 128, 512, 64, 4, 64, 0.0)
    assert lib.mlra_create(None, P(16), P(16), ctypes.byref(out)) == -1
    assert lib.mlra_create(ctypes.byref(cfg), None, P(16), ctypes.byref(out)) == -1
    bad = M.mlra_config(128, 128, 510, 64, 4, 64, 0.0)  # k does not divide d_c
    assert lib.mlra_create(ctypes.byref(bad), P(16), P(16), ctypes.byref(out)) == -1
    bad = M.mlra_config(128, 128, 512, 64, 4, 32, 0.0)  # page size other than 64
    assert lib.mlra_create(ctypes.byref(bad), P(16), P(16), ctypes.byref(out)) == -2
    bad = M.mlra_config(128, 96, 512, 64, 4, 64, 0.0)   # d_h outside the compiled set
    assert lib.mlra_create(ctypes.byref(bad), P(16), P(16), ctypes.byref(out)) == -2
    n = ctypes.c_size_t()
    assert lib.mlra_workspace_size(None, 4, ctypes.byref(n)) == -1
    assert lib.mlra_decode(None, None, 0, None, 0, None, 0, None, 0, None, 0, None, None, 0, None) == -1
    assert lib.mlra_project_workspace_size(None, 4, 5120, ctypes.byref(n)) == -1
    assert lib.mlra_project_append(None, None, 5120, None, 0.0, None, None, 0, None, 0, 4, None, 0, None) == -1
    assert lib.mlra_get_info(None, None) == -1
    assert lib.mlra_get_status(None, None) == -1
    lib.mlra_destroy(None)  # NULL-safe


def test_host_checks_of_the_reading_and_cache_options(lib):
    """The summed-blocks reading and the E4M3 cache are refused, before any CUDA call, for
    shapes and settings that were not built or make no sense."""
    P = ctypes.c_void_p
    out = P()

    def create(**kw):
        f = dict(h=128, d_h=128, d_c=512, d_rope=64, k=4, page_size=64, softmax_scale=0.0,
                 blocks_summed=0, attn_scale=0.0, cache_fp8=0, latent_scale=1.0, rope_scale=1.0)
        f.update(kw)
        cfg = M.mlra_config(*[f[n] for n, _ in M.mlra_config._fields_])
        return lib.mlra_create(ctypes.byref(cfg), P(16), P(16), ctypes.byref(out))

    assert create(blocks_summed=2) == -1                      # a flag: 0 or 1
    assert create(cache_fp8=2) == -1
    assert create(blocks_summed=1, k=1) == -2                 # summed reading: k = 2 or 4 only
    assert create(cache_fp8=1, blocks_summed=1) == -2         # E4M3 with the partitioned MLRA-4 only
    assert create(cache_fp8=1, k=2) == -2
    assert create(cache_fp8=1, latent_scale=-1.0) == -1       # scales: finite and not negative
    assert create(cache_fp8=1, rope_scale=float("inf")) == -1
    assert create(cache_fp8=1, latent_scale=float("nan")) == -1
    assert lib.mlra_create(None, P(16), P(16), ctypes.byref(out)) == -1
    cfg = M.mlra_config(128, 128, 512, 64, 4, 64, 0.0)
    assert lib.mlra_create(ctypes.byref(cfg), P(8), P(16), ctypes.byref(out)) == -1  # 16-byte aligned weights

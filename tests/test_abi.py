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

"""The C-ABI library loads on a CPU-only host and exports every declared symbol."""
import ctypes
import os
import re

import pytest

import sparse_moe_transformer_b200 as smt
from sparse_moe_transformer_b200 import build as smt_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    smt_build.build()
    return smt.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"moe_create", "moe_route", "moe_forward", "moe_destroy"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert set(smt.EXPORTS) == names


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.moe_version()
    for s in range(7):
        assert lib.moe_status_string(s)
    assert lib.moe_status_string(99) == b"unknown status"


def test_argument_errors_without_gpu(lib):
    h = ctypes.c_void_p()
    # NULL config / out pointer: rejected before any CUDA call
    assert lib.moe_create(None, 0, *([None] * 8), ctypes.byref(h)) == smt.MOE_ERR_INVALID_ARG
    assert b"NULL" in lib.moe_last_error(None)
    cfg = smt._Config(1024, 128, 6, 384, 768, smt.DTYPE_BF16, 1, 1e-6)
    assert lib.moe_create(ctypes.byref(cfg), 0, *([None] * 8), ctypes.byref(h)) == \
        smt.MOE_ERR_INVALID_ARG
    bad = smt._Config(1024, 128, 200, 384, 768, smt.DTYPE_BF16, 1, 1e-6)   # k > E
    assert lib.moe_create(ctypes.byref(bad), 0, *([None] * 8), ctypes.byref(h)) == \
        smt.MOE_ERR_INVALID_ARG
    nr = smt._Config(1024, 128, 6, 384, 768, smt.DTYPE_BF16, 0, 1e-6)      # norm_topk_prob = 0
    assert lib.moe_create(ctypes.byref(nr), 0, *([ctypes.c_void_p(16)] * 8),
                          ctypes.byref(h)) == smt.MOE_ERR_UNSUPPORTED
    # NULL handle on every entry point
    assert lib.moe_forward(None, None, None, None, 4, None, None, None) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_route(None, None, 4, None, None, None) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_reserve(None, 4) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_check(None, None) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_set_option(None, 0, 1) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(None, None, None, None, 4, None) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_last_routing(None, None, None, None, None) == smt.MOE_ERR_INVALID_ARG
    assert lib.moe_destroy(None) == smt.MOE_OK


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(OSError):
        smt._lib_backup = smt._lib
        try:
            smt._lib = None
            smt.load(str(tmp_path / "missing.so"))
        finally:
            smt._lib = smt._lib_backup


def test_noalloc_argument_errors_without_gpu(lib):
    """moe_route_noalloc rejects bad arguments before it touches the CUDA runtime
    (the pointer values below are never dereferenced)."""
    P = ctypes.c_void_p
    ok = smt._Config(1024, 128, 6, 384, 768, smt.DTYPE_BF16, 1, 1e-6)
    x, w, idx, wt = P(256), P(512), P(1024), P(2048)

    def call(cfg, T, x=x, w=w, idx=idx, wt=wt):
        return lib.moe_route_noalloc(None if cfg is None else ctypes.byref(cfg), x, w, None, T,
                                     idx, wt, None)

    assert call(None, 8) == smt.MOE_ERR_INVALID_ARG
    for bad in (smt._Config(0, 128, 6, 384, 768, smt.DTYPE_BF16, 1, 1e-6),      # H = 0
                smt._Config(1024, 2048, 6, 384, 768, smt.DTYPE_BF16, 1, 1e-6),  # E > 1024
                smt._Config(1024, 4, 6, 384, 768, smt.DTYPE_BF16, 1, 1e-6),     # k > E
                smt._Config(1024, 128, 17, 384, 768, smt.DTYPE_BF16, 1, 1e-6),  # k > 16
                smt._Config(1024, 128, 6, 384, 768, 7, 1, 1e-6)):               # dtype
        assert call(bad, 8) == smt.MOE_ERR_INVALID_ARG
    nr = smt._Config(1024, 128, 6, 384, 768, smt.DTYPE_BF16, 0, 1e-6)
    assert call(nr, 8) == smt.MOE_ERR_UNSUPPORTED
    assert call(ok, -1) == smt.MOE_ERR_INVALID_ARG
    assert call(ok, 0, x=None, w=None, idx=None, wt=None) == smt.MOE_OK       # T = 0: no-op
    assert call(ok, 8, x=None) == smt.MOE_ERR_INVALID_ARG
    assert call(ok, 8, idx=None) == smt.MOE_ERR_INVALID_ARG
    assert call(ok, 8, x=P(264)) == smt.MOE_ERR_INVALID_ARG                    # misaligned
    assert b"aligned" in lib.moe_last_error(None)
    # the fixed scratch holds T = 8183 tokens at E = 128; one more is refused
    assert call(ok, 8184) == smt.MOE_ERR_INVALID_ARG
    assert b"fixed" in lib.moe_last_error(None)

"""The C-ABI library loads on a CPU-only host and exports every declared symbol."""
import ctypes
import os
import re
import shutil
import subprocess

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


class _FakeCudaTensor:
    """Just enough of a CUDA tensor for the binding's argument checks (no GPU here)."""

    def __init__(self, shape, dtype, contiguous=True, device="cuda:0"):
        import torch
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.is_cuda = True
        self.device = torch.device(device)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)


def test_binding_argument_checks_without_gpu():
    """The binding refuses tensors the library would read or write out of bounds, before
    it calls the library (a bare layer object: no handle is needed to get that far)."""
    import torch
    layer = object.__new__(smt.MoELayer)
    layer.cfg = smt.LayerConfig(64, 8, 2, 128, 128, "bf16")
    layer.torch_dtype = torch.bfloat16
    bf = torch.bfloat16
    x = _FakeCudaTensor((5, 64), bf)
    layer._check_tokens(x, residual=_FakeCudaTensor((5, 64), bf), out=None)
    bad_x = [torch.zeros(5, 64, dtype=bf),                        # host tensor
             _FakeCudaTensor((5, 32), bf),                         # wrong hidden size
             _FakeCudaTensor((5, 64), torch.float32),              # wrong dtype
             _FakeCudaTensor((5, 64), bf, contiguous=False),
             _FakeCudaTensor((5, 2, 32), bf)]
    for t in bad_x:
        with pytest.raises(ValueError):
            layer._check_tokens(t)
        with pytest.raises(ValueError):
            layer.forward(t)
    bad_other = [_FakeCudaTensor((4, 64), bf), _FakeCudaTensor((5, 64), torch.float32),
                 _FakeCudaTensor((5, 64), bf, contiguous=False),
                 _FakeCudaTensor((5, 64), bf, device="cuda:1")]
    for t in bad_other:
        for name in ("residual", "out"):
            with pytest.raises(ValueError, match=name):
                layer._check_tokens(x, **{name: t})
    xh = torch.zeros(5, 64, dtype=bf)
    for bad in (torch.zeros(4, 64, dtype=bf), torch.zeros(5, 64, dtype=torch.float32),
                torch.zeros(64, 5, dtype=bf).t()):
        with pytest.raises(ValueError):
            layer.forward_host(xh, bad)
        with pytest.raises(ValueError):
            layer.forward_host(xh, torch.zeros(5, 64, dtype=bf), residual_host=bad)


def test_binding_weight_checks_without_gpu():
    """moe_create copies E x I x H elements and so on from the weight pointers: the
    binding refuses weights of another shape, dtype or layout before calling it."""
    import torch
    bf = torch.bfloat16
    H, E, k, I, Is = 64, 8, 2, 128, 32
    cfg = smt.LayerConfig(H, E, k, I, Is, "bf16")
    good = dict(w_router=(E, H), w_gate=(E, I, H), w_up=(E, I, H), w_down=(E, H, I),
                ws_gate=(Is, H), ws_up=(Is, H), ws_down=(H, Is))

    def make(**over):
        ws = {n: _FakeCudaTensor(shape, bf) for n, shape in good.items()}
        ws.update(over)
        return smt.MoELayer(cfg, **ws, device=0)

    for name, shape in good.items():
        wrong = tuple(reversed(shape)) if len(set(shape)) > 1 else shape + (1,)
        with pytest.raises(ValueError, match=name):
            make(**{name: _FakeCudaTensor(wrong, bf)})
        with pytest.raises(ValueError, match=name):
            make(**{name: _FakeCudaTensor(shape, torch.float32)})
        with pytest.raises(ValueError, match=name):
            make(**{name: _FakeCudaTensor(shape, bf, contiguous=False)})
        with pytest.raises(ValueError, match=name):
            make(**{name: None})
    with pytest.raises(ValueError, match="rms_weight"):
        make(rms_weight=_FakeCudaTensor((H + 1,), bf))


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { ++fails; printf("failed: %s (line %d)\n", #c, __LINE__); } } while (0)

int main(void) {
    CHECK(strstr(moe_version(), "sm_100a") != NULL);
    CHECK(strcmp(moe_status_string(MOE_OK), "ok") == 0);
    CHECK(strcmp(moe_status_string((moe_status)42), "unknown status") == 0);
    moe_handle h = (moe_handle)0;
    moe_config cfg = {1024, 128, 6, 384, 768, MOE_DTYPE_BF16, 1, 1e-6f};
    /* argument errors are returned before any CUDA call */
    CHECK(moe_create(NULL, 0, 0, 0, 0, 0, 0, 0, 0, 0, &h) == MOE_ERR_INVALID_ARG);
    CHECK(moe_create(&cfg, 0, 0, 0, 0, 0, 0, 0, 0, 0, &h) == MOE_ERR_INVALID_ARG);
    CHECK(h == NULL);
    CHECK(strlen(moe_last_error(NULL)) > 0);
    CHECK(moe_forward(NULL, 0, 0, 0, 8, 0, 0, 0) == MOE_ERR_INVALID_ARG);
    CHECK(moe_route(NULL, 0, 8, 0, 0, 0) == MOE_ERR_INVALID_ARG);
    CHECK(moe_reserve(NULL, 8) == MOE_ERR_INVALID_ARG);
    CHECK(moe_set_option(NULL, MOE_OPT_WAIT_LIMIT_NS, 1) == MOE_ERR_INVALID_ARG);
    CHECK(moe_kernel_stats(NULL, NULL, NULL, 0) == MOE_ERR_INVALID_ARG);
    CHECK(moe_destroy(NULL) == MOE_OK);
    CHECK(moe_route_noalloc(&cfg, 0, 0, 0, 0, 0, 0, 0) == MOE_OK);           /* T = 0 */
    CHECK(moe_route_noalloc(&cfg, (const void*)8, (const void*)16, 0, 4,
                            (int32_t*)16, (float*)16, 0) == MOE_ERR_INVALID_ARG);  /* misaligned x */
    printf(fails ? "FAIL %d\n" : "OK\n", fails);
    return fails ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c_and_links_from_c(lib, tmp_path):
    """include/moe.h compiles as C11 and a C program links against the library and gets
    the documented argument errors (no GPU: nothing here reaches the CUDA runtime)."""
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(smt.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmoe_b200",
                    f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr

"""Compiler resource report of every kernel (nvcc cross-compiles sm_100a here).

Each source under csrc/ is compiled with the library's flags plus `-Xptxas -v`; the
assembler's per-kernel report must show no register spills (a spill in these kernels
would put local-memory traffic next to the weight stream), and the tensor-core
kernels, launched one CTA per SM with 320 threads, must fit the SM's 64 K registers.
"""
import os
import re
import shutil
import subprocess
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

from sparse_moe_transformer_b200 import build as smt_build

REPORT = re.compile(r"Compiling entry function '(\w+)'.*?"
                    r"(\d+) bytes spill stores, (\d+) bytes spill loads.*?"
                    r"Used (\d+) registers", re.S)


def _reports():
    out = {}
    with tempfile.TemporaryDirectory() as d:
        def compile_one(src):
            obj = os.path.join(d, os.path.basename(src) + ".o")
            return subprocess.run([smt_build.nvcc(), *smt_build.ARCH, *smt_build.FLAGS,
                                   "-Xptxas", "-v", "-c", src, "-o", obj],
                                  capture_output=True, text=True)
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            runs = list(ex.map(compile_one, smt_build.sources()))
        for r in runs:
            assert r.returncode == 0, r.stderr[-2000:]
            for name, st, ld, regs in REPORT.findall(r.stderr):
                out[name] = (int(st), int(ld), int(regs))
    return out


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_no_spills_and_register_budget():
    rep = _reports()
    for kernel in ("tc_fused_experts_kernel", "tc_routed_experts_kernel", "router_tc_kernel",
                   "router_kernel", "permute_kernel", "combine_partials_kernel"):
        assert any(kernel in name for name in rep), f"no report for {kernel}"
    for name, (st, ld, regs) in rep.items():
        assert st == 0 and ld == 0, f"{name}: {st} bytes spill stores, {ld} spill loads"
    for kernel in ("tc_fused_experts_kernel", "tc_routed_experts_kernel", "router_tc_kernel",
                   "tc_router_logits_kernel"):
        for name, (_, _, regs) in rep.items():
            if kernel in name:
                assert regs * 320 <= 65536, f"{name}: {regs} registers x 320 threads"

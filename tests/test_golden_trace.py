"""The stored step-by-step oracle trace of the tiny fp32 workload.

tests/golden/trace_tiny_fp32.txt is written by tests/golden/trace_tiny_fp32.py from
the oracle alone.  This test (1) regenerates it and compares every number (within
1e-12 relative: libm's exp may round differently on another host) and every index,
and (2) redoes by hand the checks a reader of the trace would make: the weights are
the softmax of the selected logits, the k-gap is the gap between the k-th and the
(k+1)-th largest logit, and y is the shared output plus the weighted expert outputs
(routing and combine equation of page "3C . Talker MoE (20 lop, 128 Experts Top-6)
& Dau ra ma ngu nghia c_0", section 3).
"""
import importlib.util
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _parse(lines):
    tokens = []
    for ln in lines:
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        key, *vals = ln.split()
        if key == "token":
            tokens.append({})
            continue
        tokens[-1][key] = [int(v) for v in vals] if key == "S" else np.array(vals, dtype=float)
    return tokens


def _generator():
    spec = importlib.util.spec_from_file_location("trace_tiny_fp32",
                                                  os.path.join(GOLDEN, "trace_tiny_fp32.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_trace_reproduces():
    with open(os.path.join(GOLDEN, "trace_tiny_fp32.txt")) as f:
        stored = _parse(f.read().splitlines())
    fresh = _parse(_generator().trace_lines())
    assert len(stored) == len(fresh) == 4
    for a, b in zip(stored, fresh):
        assert a.keys() == b.keys()
        for key in a:
            if key == "S":
                assert a[key] == b[key]
            else:
                scale = max(1.0, float(np.max(np.abs(b[key]))))
                assert np.max(np.abs(a[key] - b[key])) <= 1e-12 * scale, key


def test_trace_checks_by_hand():
    with open(os.path.join(GOLDEN, "trace_tiny_fp32.txt")) as f:
        tokens = _parse(f.read().splitlines())
    for tok in tokens:
        l, S, w = tok["logits"], tok["S"], tok["w"]
        k = len(S)
        ranked = sorted(range(len(l)), key=lambda e: (-l[e], e))
        assert S == ranked[:k]
        z = sum(math.exp(l[e]) for e in S)
        assert np.allclose(w, [math.exp(l[e]) / z for e in S], rtol=0, atol=1e-15)
        assert abs(tok["k_gap"][0] - (l[ranked[k - 1]] - l[ranked[k]])) <= 1e-15
        y = tok["shared"] + sum(w[i] * tok[f"E_{e}"] for i, e in enumerate(S))
        assert np.max(np.abs(y - tok["y"])) <= 1e-14

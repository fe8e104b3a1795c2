"""Host-side logic of bench.py, checked on the CPU.

* The algorithmic bytes and FLOPs the roofline divides by: bytes are counted
  from the sizes of the arrays a step must move (the weights of the experts
  the routing touched, the router and shared-expert weights, the tokens in and
  out, the Top-k indices and weights), FLOPs from the list of matrix products
  the layer is defined by (router logits W_r x; per selected expert gate, up
  and down projections; the shared expert's three projections).
* The clock summary that decides whether a run is kept (median SM clock under
  load, the throttle reasons seen).
* The ncu traffic table: each entry names a kernel whose source file is still
  the one that was captured, so a bench line never reports stale counters.
* The reference arm's JSON line (the oracle timed on the host cores), and that
  ranks other than 0 print nothing under torchrun.
"""
import json
import os
import shutil
import subprocess
import sys

import numpy as np

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def test_algorithmic_work_counts_moved_arrays_and_products():
    inp = synth.make_custom(H=64, E=8, k=2, I=32, Is=48, T=5, dtype="bf16", seed=3)
    wl, L = inp.workload, inp.layers[0]
    T, H, E, k, I, Is = wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is
    for seed in range(4):
        idx = _routing(T, E, k, seed)
        touched = sorted(set(idx.ravel().tolist()))
        (w,) = bench.algorithmic_work(wl, [idx])
        assert w["touched"] == len(touched)
        expert_w = sum(L.w_gate[e].nbytes + L.w_up[e].nbytes + L.w_down[e].nbytes
                       for e in touched)
        slot_rows = 2 * (T * k) * inp.x[0].nbytes          # permuted rows in, expert rows out
        assert w["experts_bytes"] == expert_w + slot_rows
        topk = np.zeros((T, k), np.int32).nbytes + np.zeros((T, k), np.float32).nbytes
        assert w["layer_bytes"] == (L.w_router.nbytes + expert_w + L.ws_gate.nbytes
                                    + L.ws_up.nbytes + L.ws_down.nbytes
                                    + 2 * inp.x.nbytes + topk)
        (wr,) = bench.algorithmic_work(wl, [idx], residual=True)
        assert wr["layer_bytes"] == w["layer_bytes"] + inp.x.nbytes   # the residual's read
        assert all(wr[key] == w[key] for key in w if key != "layer_bytes")
        mm = lambda m, n, p: 2 * m * n * p                 # FLOPs of an (m,n)x(n,p) product
        per_slot = mm(1, H, I) + mm(1, H, I) + mm(1, I, H)
        assert w["experts_flops"] == T * k * per_slot
        assert w["layer_flops"] == (mm(T, H, E) + T * k * per_slot
                                    + T * (mm(1, H, Is) + mm(1, H, Is) + mm(1, Is, H)))


def test_algorithmic_work_fp32_and_full_coverage():
    inp = synth.make("tiny_fp32")
    wl, L = inp.workload, inp.layers[0]
    idx = np.tile(np.arange(wl.E, dtype=np.int32)[: wl.k], (wl.T, 1))
    idx[-1] = np.arange(wl.E - wl.k, wl.E)                 # touches 2k distinct experts
    (w,) = bench.algorithmic_work(wl, [idx])
    assert w["touched"] == min(wl.E, 2 * wl.k)
    per_expert = L.w_gate[0].nbytes + L.w_up[0].nbytes + L.w_down[0].nbytes
    assert w["experts_bytes"] == w["touched"] * per_expert + 2 * wl.T * wl.k * inp.x[0].nbytes


def test_clock_summary():
    s = bench.ClockSampler("GPU-0")
    s.lines = ["1965, 1965, Not Active, Not Active, Not Active, Not Active",
               "1800, 1965, Not Active, Not Active, Not Active, Active",
               "garbage line",
               "[N/A], 1965, Not Active, Not Active, Not Active, Not Active",
               "1900, 1965, Not Active, Not Active, Not Active, Not Active",
               "1700, 1965, Active, Not Active, Not Active, Not Active"]
    out = s.summary()
    assert out["samples"] == 4
    assert out["sm_mhz"] == 1850.0                         # median of 1965, 1800, 1900, 1700
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]
    empty = bench.ClockSampler("GPU-0")
    assert empty.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_table_matches_sources(tmp_path, monkeypatch):
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        table = json.load(f)
    assert table, "no ncu traffic entries"
    for workload, e in table.items():
        assert workload in synth.WORKLOADS
        src = os.path.join(ROOT, "sparse_moe_transformer_b200", "csrc", e["source"])
        assert bench.source_sha(src) == e["source_sha"], f"{workload}: stale counters"
        assert os.path.exists(os.path.join(ROOT, e["capture"]))
        with open(os.path.join(ROOT, e["capture"])) as f:
            assert e["kernel"] in f.read()
        assert bench.recorded_traffic(workload, e["kernel"]) == e["dram_bytes_per_launch"]
        assert bench.recorded_traffic(workload, e["kernel"] + "_other") is None
    # an edited source invalidates its entry
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    (fake / "sparse_moe_transformer_b200" / "csrc").mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "profiles", "ncu_traffic.json"), fake / "profiles")
    workload, e = next(iter(table.items()))
    src = os.path.join(ROOT, "sparse_moe_transformer_b200", "csrc", e["source"])
    with open(src) as f:
        text = f.read()
    (fake / "sparse_moe_transformer_b200" / "csrc" / e["source"]).write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.recorded_traffic(workload, e["kernel"]) == e["dram_bytes_per_launch"]
    (fake / "sparse_moe_transformer_b200" / "csrc" / e["source"]).write_text(text + "\n// edit\n")
    assert bench.recorded_traffic(workload, e["kernel"]) is None


def _run_reference(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny_fp32", "--steps", "3", "--warmup", "1"],
                          capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)


def test_reference_arm_line():
    r = _run_reference()
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 3 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["vs_baseline"] is None
    assert d["config"]["workload"] == "tiny_fp32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_are_silent():
    r = _run_reference({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_graph_plan_times_exactly_k_steps():
    """The captured graphs hold exactly K timed steps, and with several weight copies
    no two consecutive steps read the same copy (each step misses in L2)."""
    import pytest
    for rotate in (1, 3, 8):
        for K in list(range(1, 80)) + [400, 20000, 20001]:
            cycle, n_rep, rem = bench.graph_plan(K, rotate)
            assert cycle * n_rep + rem == K and 1 <= cycle <= 32 and 0 <= rem < cycle
            if K >= 32:
                assert cycle % rotate == 0          # replays start again at copy 0
            copies = [i % rotate for i in range(cycle)] * n_rep + [i % rotate
                                                                   for i in range(rem)]
            assert len(copies) == K
            if rotate > 1:
                assert all(a != b for a, b in zip(copies, copies[1:]))
    with pytest.raises(ValueError):
        bench.graph_plan(0, 8)


def test_reference_arm_under_torchrun():
    """Launched like the multi-GPU bench (torchrun, two ranks): one line, from rank 0."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--workload", "tiny_fp32", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 3


def test_load_peaks(tmp_path):
    good = tmp_path / "good.json"
    good.write_text(json.dumps({"hbm_gbs": 6458.1, "bf16_tflops": 1672.0,
                                "bf16_tflops_sustained": 1408.4}))
    p = bench.load_peaks(str(good))
    assert p["source"] == "measured" and p["hbm_gbs"] == 6458.1 and p["bf16_tflops"] == 1672.0
    for bad in ("{}", "not json", json.dumps({"hbm_gbs": 0, "bf16_tflops": 1.0}),
                json.dumps({"hbm_gbs": None, "bf16_tflops": 1.0})):
        f = tmp_path / "bad.json"
        f.write_text(bad)
        assert bench.load_peaks(str(f)) == bench.FALLBACK_PEAKS
    assert bench.load_peaks(str(tmp_path / "missing.json")) == bench.FALLBACK_PEAKS

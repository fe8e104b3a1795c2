"""The skewed prefill workload's stored calibration still produces the statistics it
records, and the ones the workload is meant to have (about 70 % of the Top-6 slots
on 8 hot experts, 40 or more experts without a token).

tests/golden/skew_talker_prefill_skewed.json was written by
tests/golden/calibrate_skew.py from the oracle's routing; this test routes the same
16384 seeded tokens with the oracle again (router only, fp64) and compares.
"""
import numpy as np

import oracle
import synth


def test_skew_calibration_reproduces():
    wl = synth.WORKLOADS["talker_prefill_skewed"]
    p = synth.load_skew()
    inp = synth.make_skewed(wl, wl.T, p["s"], p["dead_steps"], p["hot_bias"], router_only=True)
    assert inp.skew["hot"] == p["hot"] and inp.skew["dead"] == p["dead"]
    dummy = np.zeros((wl.E, 1, wl.H), np.uint16)
    lw = oracle.LayerWeights(inp.layers[0].w_router, dummy, dummy,
                             np.zeros((wl.E, wl.H, 1), np.uint16), None, None, None, top_k=wl.k)
    _, idx, _, gap = oracle.Oracle(lw).route(inp.x)
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    share = float(np.isin(idx, p["hot"]).mean())
    assert abs(share - p["hot_share"]) < 1e-12
    assert abs(share - 0.70) <= 0.005
    assert counts[p["dead"]].sum() == 0
    assert int((counts == 0).sum()) == p["empty_experts"] >= 40
    assert int(counts.max()) == p["max_expert_tokens"]
    assert int((gap <= 1e-3).sum()) == p["near_ties_1e3"]

"""Routing statistics of the synthetic workloads, from the oracle's router (fp64).

* Skewed prefill: the stored calibration (tests/golden/skew_talker_prefill_skewed.json,
  written by tests/golden/calibrate_skew.py from the oracle's routing) still produces
  the statistics it records and the ones the workload is meant to have: about 70 % of
  the Top-6 slots on 8 hot experts, 40 or more experts without a token.
* Decode and prefill: near-uniform routing, as random router rows give.  8 tokens x
  Top-6 touch close to the 128 (1 - (122/128)^8) = 40.8 experts a uniform choice
  expects (the roofline's weight bytes scale with that count); 4096 tokens reach
  every expert, each within a factor of two of the mean of 192 slots.
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


def _routing(name):
    inp = synth.make(name)
    wl = inp.workload
    lw = oracle.LayerWeights(**inp.layers[0].arrays(), top_k=wl.k)
    _, idx, _, _ = oracle.Oracle(lw).route(inp.x)
    return wl, np.bincount(idx.ravel(), minlength=wl.E)


def test_decode_and_prefill_routing_is_near_uniform():
    wl, c = _routing("talker_decode")
    expected = wl.E * (1 - ((wl.E - wl.k) / wl.E) ** wl.T)
    assert abs(int((c > 0).sum()) - expected) <= 4
    wl, c = _routing("talker_prefill")
    mean = wl.T * wl.k / wl.E
    assert c.min() > mean / 2 and c.max() < mean * 2

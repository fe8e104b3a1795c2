"""Write tests/golden/skew_talker_prefill_skewed.json (calls only the oracle).

The skewed prefill workload (T=16384) adds a shared unit direction d to every
token (times s) and +0.05*d to 8 "hot" router rows, so that about 70% of the
Top-6 slots land on the hot experts; 48 "dead" rows get -dead_steps*0.05*d so
that 40+ experts receive no token.  This script picks s by bisection on the
oracle's routing of the exact bf16 inputs (hot slot share 0.70 +- 0.005), and
raises dead_steps until no dead expert is selected.

Run:  python tests/golden/calibrate_skew.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

TARGET, TOL = 0.70, 0.005


def routing(wl, s, dead_steps):
    inp = synth.make_skewed(wl, wl.T, s, dead_steps, router_only=True)
    wr = inp.layers[0].w_router
    dummy = np.zeros((wl.E, 1, wl.H), np.uint16)
    lw = oracle.LayerWeights(wr, dummy, dummy, np.zeros((wl.E, wl.H, 1), np.uint16),
                             None, None, None, top_k=wl.k)
    _, idx, _, gap = oracle.Oracle(lw).route(inp.x)
    return inp.skew, idx, gap


def main():
    wl = synth.WORKLOADS["talker_prefill_skewed"]
    for dead_steps in range(1, 20):
        lo, hi = 0.0, 80.0
        for _ in range(24):
            s = 0.5 * (lo + hi)
            skew, idx, gap = routing(wl, s, dead_steps)
            share = float(np.isin(idx, skew["hot"]).mean())
            print(f"dead_steps={dead_steps} s={s:.4f} hot share={share:.4f}", flush=True)
            if abs(share - TARGET) <= TOL:
                break
            lo, hi = (s, hi) if share < TARGET else (lo, s)
        counts = np.bincount(idx.ravel(), minlength=wl.E)
        if counts[skew["dead"]].sum() == 0 and abs(share - TARGET) <= TOL:
            out = dict(s=s, dead_steps=dead_steps, hot_bias=0.05, hot=skew["hot"],
                       dead=skew["dead"], hot_share=share,
                       empty_experts=int((counts == 0).sum()),
                       max_expert_tokens=int(counts.max()),
                       near_ties_1e3=int((gap <= 1e-3).sum()),
                       written_by="python tests/golden/calibrate_skew.py (oracle routing only)")
            with open(synth.SKEW_FILE, "w") as f:
                json.dump(out, f, indent=1)
            print(json.dumps(out))
            return
    raise SystemExit("no calibration found")


if __name__ == "__main__":
    main()

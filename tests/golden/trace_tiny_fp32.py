"""Write tests/golden/trace_tiny_fp32.txt: a step-by-step trace of the oracle on the
tiny fp32 workload (calls only the oracle).

For each token the trace lists the layer input x, the router logits l = W_r x, the
selected experts S (descending logit, ties to the lower index), their renormalised
weights w, the k-gap, each selected expert's SwiGLU output, the shared expert's
output and the layer output y, so that a reader can check every step by hand:
w_i = exp(l_i) / sum_{j in S} exp(l_j) and y = shared + sum_i w_i E_i (routing and
combine equation of page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra ma
ngu nghia c_0", section 3).  Each expert's output comes from the oracle run as a
one-expert layer (k = 1, so its weight is 1) on that expert's weights.

Run:  python tests/golden/trace_tiny_fp32.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "trace_tiny_fp32.txt")


def single_mlp(gate, up, down):
    """The oracle as a one-expert layer with no shared expert: y = down(SiLU(gate x) * up x)."""
    H = gate.shape[1]
    return oracle.Oracle(oracle.LayerWeights(np.zeros((1, H), np.float32), gate[None], up[None],
                                             down[None], None, None, None, top_k=1))


def trace_lines():
    inp = synth.make("tiny_fp32")
    wl, L = inp.workload, inp.layers[0]
    o = oracle.Oracle(oracle.LayerWeights(**L.arrays(), top_k=wl.k))
    logits, idx_r, _, _ = o.route(inp.x)
    y, idx, w, gap = o.forward(inp.x)
    assert np.array_equal(idx, idx_r)
    experts = [single_mlp(L.w_gate[e], L.w_up[e], L.w_down[e]) for e in range(wl.E)]
    shared = single_mlp(L.ws_gate, L.ws_up, L.ws_down)
    fmt = lambda a: " ".join(repr(float(v)) for v in np.ravel(a))
    lines = [f"# oracle trace: workload tiny_fp32 (T={wl.T}, H={wl.H}, E={wl.E}, k={wl.k}, "
             f"I={wl.I}, I_s={wl.Is}, fp32 inputs, seed {wl.seed}); written by "
             "tests/golden/trace_tiny_fp32.py",
             "# per token: x, logits l = W_r x, S (descending l, ties to the lower index),",
             "# w_i = exp(l_i) / sum_{j in S} exp(l_j), k_gap = l_(k) - l_(k+1), the selected",
             "# experts' outputs E_<e>, the shared expert's output, y = shared + sum_i w_i E_i"]
    for t in range(wl.T):
        xt = inp.x[t:t + 1]
        lines.append(f"token {t}")
        lines.append(f"x {fmt(xt)}")
        lines.append(f"logits {fmt(logits[t])}")
        lines.append("S " + " ".join(str(int(e)) for e in idx[t]))
        lines.append(f"w {fmt(w[t])}")
        lines.append(f"k_gap {fmt(gap[t])}")
        for e in idx[t]:
            lines.append(f"E_{int(e)} {fmt(experts[int(e)].forward(xt)[0])}")
        lines.append(f"shared {fmt(shared.forward(xt)[0])}")
        lines.append(f"y {fmt(y[t])}")
    return lines


def main():
    with open(OUT, "w") as f:
        f.write("\n".join(trace_lines()) + "\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()

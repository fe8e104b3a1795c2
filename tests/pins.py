"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin takes an ``Oracle`` factory (so the mutation tests can point it at a
deliberately broken copy of the C oracle) and raises AssertionError on failure.

  O1  renormalised Top-k weights sum to 1 within 1e-12 (the lab's check (2))
  O2  sparse result == brute-force dense evaluation of every expert, masked
  O3  permuting experts (router rows + expert weights together) permutes S only
  O4  tokens are independent (single-token calls, shuffled batches)
  O5  hand-derived golden case (tests/golden/hand_case_h2_e3_k2.txt)
  O6  special cases: E=1,k=1 dense MLPs; k=E softmax mixture; identical experts;
      zero router (all ties -> lower indices, w = 1/k)
  O7  independent NumPy statement agrees with the C oracle
  O8  bf16 storage at the Talker size: bf16 bits == their exact fp64 values, bit for
      bit, and == a brute-force dense evaluation of all 128 experts on a token sample
  O9  forced routing (the near-tie re-evaluation): forcing the oracle's own sets changes
      nothing; forcing other sets gives the masked dense evaluation over those sets
  R   pre-RMSNorm and residual special cases; k-gap equals the sorted-logit gap
"""
from __future__ import annotations

import ast
import functools
import math
import operator
import os

import numpy as np

import synth
from oracle import LayerWeights, numpy_ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers
def _f64_layer(rng, H, E, k, I, Is, scale=0.5):
    n = lambda *s: rng.standard_normal(s) * scale
    return LayerWeights(n(E, H), n(E, I, H), n(E, I, H), n(E, H, I),
                        n(Is, H) if Is else None, n(Is, H) if Is else None,
                        n(H, Is) if Is else None, top_k=k)


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _dense_swiglu(x, g, u, d):
    """Textbook dense SwiGLU MLP on rows of x with numpy matmuls."""
    return (_silu(x @ g.T) * (x @ u.T)) @ d.T


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


_OPS = {ast.Add: operator.add, ast.Sub: operator.sub, ast.Mult: operator.mul,
        ast.Div: operator.truediv, ast.USub: operator.neg, ast.UAdd: operator.pos}
_NAMES = {"ln2": math.log(2.0), "ln3": math.log(3.0)}


def _eval(expr: str) -> float:
    def ev(n):
        if isinstance(n, ast.Expression):
            return ev(n.body)
        if isinstance(n, ast.Constant):
            return float(n.value)
        if isinstance(n, ast.Name):
            return _NAMES[n.id]
        if isinstance(n, ast.BinOp):
            return _OPS[type(n.op)](ev(n.left), ev(n.right))
        if isinstance(n, ast.UnaryOp):
            return _OPS[type(n.op)](ev(n.operand))
        raise ValueError(expr)
    return ev(ast.parse(expr, mode="eval"))


def load_hand_case(path=os.path.join(GOLDEN, "hand_case_h2_e3_k2.txt")):
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(None, 1)
            rows[key] = [[_eval(v) for v in r.split()] for r in rest.split(";")]
    dims = {k: int(rows[k][0][0]) for k in ("H", "E", "k", "I", "Is")}
    H, E, k, I, Is = (dims[n] for n in ("H", "E", "k", "I", "Is"))
    a = lambda key, shape: np.array(rows[key], dtype=np.float64).reshape(shape)
    w = LayerWeights(a("w_router", (E, H)), a("w_gate", (E, I, H)), a("w_up", (E, I, H)),
                     a("w_down", (E, H, I)), a("ws_gate", (Is, H)), a("ws_up", (Is, H)),
                     a("ws_down", (H, Is)), top_k=k)
    T = len(rows["x"])
    return (w, a("x", (T, H)), np.array(rows["expect_idx"], dtype=np.int32),
            a("expect_w", (T, k)), a("expect_y", (T, H)))


# ---------------------------------------------------------------- pins
def pin_weights_sum_to_one(make):
    """O1: |sum_{i in S} w_i - 1| < 1e-12 for every token (lab check (2))."""
    for name in ("tiny_fp32",):
        inp = synth.make(name)
        o = make(LayerWeights(**inp.layers[0].arrays(), top_k=inp.workload.k))
        _, _, w, _ = o.forward(inp.x)
        assert np.all(np.abs(w.sum(1) - 1.0) < 1e-12), w.sum(1)
    rng = np.random.default_rng(1)
    lw = _f64_layer(rng, 16, 12, 5, 8, 8)
    _, _, w, _ = make(lw).forward(rng.standard_normal((20, 16)))
    assert np.all(np.abs(w.sum(1) - 1.0) < 1e-12)


def brute_force_dense(lw: LayerWeights, x):
    """O2 reference: evaluate ALL experts densely, then mask to the Top-k set.

    Selection: rank experts by (logit descending, index ascending) with Python's
    sort; mask m_e = 1 for the first k; weights m_e p_e / sum(m p)."""
    H, E, k, I, Is = lw.dims
    x = numpy_ref.widen(x)
    Wr = numpy_ref.widen(lw.w_router)
    logits = x @ Wr.T
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    every = np.stack([_dense_swiglu(x, numpy_ref.widen(lw.w_gate)[e], numpy_ref.widen(lw.w_up)[e],
                                    numpy_ref.widen(lw.w_down)[e]) for e in range(E)], axis=1)
    mask = np.zeros_like(p)
    for t in range(x.shape[0]):
        ranked = sorted(range(E), key=lambda e: (-logits[t, e], e))
        mask[t, ranked[:k]] = 1.0
    wts = mask * p / (mask * p).sum(1, keepdims=True)
    y = np.einsum("te,teh->th", wts, every)
    if Is:
        y += _dense_swiglu(x, numpy_ref.widen(lw.ws_gate), numpy_ref.widen(lw.ws_up),
                           numpy_ref.widen(lw.ws_down))
    return y


def pin_brute_force_dense(make):
    """O2: sparse y equals the masked dense evaluation within 1e-12 (relative)."""
    inp = synth.make("tiny_fp32")
    lw = LayerWeights(**inp.layers[0].arrays(), top_k=inp.workload.k)
    y, *_ = make(lw).forward(inp.x)
    assert _rel(y, brute_force_dense(lw, inp.x)) < 1e-12
    rng = np.random.default_rng(2)
    lw = _f64_layer(rng, 12, 10, 3, 6, 5)
    x = rng.standard_normal((17, 12))
    y, *_ = make(lw).forward(x)
    assert _rel(y, brute_force_dense(lw, x)) < 1e-12


def pin_expert_permutation(make):
    """O3: permuting experts with their router rows leaves y unchanged; S maps by pi."""
    rng = np.random.default_rng(3)
    lw = _f64_layer(rng, 10, 9, 3, 7, 6)
    x = rng.standard_normal((11, 10))
    y, idx, w, _ = make(lw).forward(x)
    pi = rng.permutation(9)          # new expert e' is old expert pi[e']
    lp = LayerWeights(lw.w_router[pi], lw.w_gate[pi], lw.w_up[pi], lw.w_down[pi],
                      lw.ws_gate, lw.ws_up, lw.ws_down, top_k=3)
    yp, idxp, wp, _ = make(lp).forward(x)
    assert _rel(yp, y) < 1e-12
    assert np.array_equal(pi[idxp], idx)
    assert np.max(np.abs(wp - w)) < 1e-12


def pin_token_independence(make):
    """O4: y(x)[t] == y(x[t:t+1]) bit for bit; a shuffled batch gives shuffled rows."""
    rng = np.random.default_rng(4)
    lw = _f64_layer(rng, 8, 6, 2, 5, 4)
    x = rng.standard_normal((9, 8))
    o = make(lw)
    y, idx, _, _ = o.forward(x)
    for t in range(9):
        yt, it, _, _ = o.forward(x[t:t + 1])
        assert np.array_equal(yt[0], y[t]) and np.array_equal(it[0], idx[t])
    perm = rng.permutation(9)
    ys, _, _, _ = o.forward(x[perm])
    assert np.array_equal(ys, y[perm])


def pin_hand_case(make):
    """O5: the hand-derived case in tests/golden/hand_case_h2_e3_k2.txt."""
    lw, x, e_idx, e_w, e_y = load_hand_case()
    y, idx, w, _ = make(lw).forward(x)
    assert np.array_equal(idx, e_idx), idx
    assert np.max(np.abs(w - e_w)) < 1e-15
    assert np.max(np.abs(y - e_y)) < 1e-14, (y, e_y)


def pin_special_cases(make):
    """O6: cases that reduce to textbook computations."""
    rng = np.random.default_rng(6)
    H, I, Is = 12, 7, 5
    # (i) one expert, k=1: w = 1 and y = SwiGLU_0(x) + SwiGLU_s(x)
    lw = _f64_layer(rng, H, 1, 1, I, Is)
    x = rng.standard_normal((6, H))
    y, idx, w, _ = make(lw).forward(x)
    ref = (_dense_swiglu(x, lw.w_gate[0], lw.w_up[0], lw.w_down[0])
           + _dense_swiglu(x, lw.ws_gate, lw.ws_up, lw.ws_down))
    assert np.all(w == 1.0) and np.all(idx == 0)
    assert _rel(y, ref) < 1e-12
    # (ii) k = E: y = Shared + sum_e softmax(l)_e E_e(x), a dense softmax mixture
    E = 5
    lw = _f64_layer(rng, H, E, E, I, Is)
    y, _, _, _ = make(lw).forward(x)
    logits = x @ lw.w_router.T
    p = np.exp(logits) / np.exp(logits).sum(1, keepdims=True)
    ref = sum(p[:, [e]] * _dense_swiglu(x, lw.w_gate[e], lw.w_up[e], lw.w_down[e])
              for e in range(E))
    ref = ref + _dense_swiglu(x, lw.ws_gate, lw.ws_up, lw.ws_down)
    assert _rel(y, ref) < 1e-12
    # (iii) identical experts: routed part is E(x) whatever the routing (sum w = 1)
    lw = _f64_layer(rng, H, 6, 3, I, 0)
    for a in (lw.w_gate, lw.w_up, lw.w_down):
        a[:] = a[0]
    y, _, _, _ = make(lw).forward(x)
    assert _rel(y, _dense_swiglu(x, lw.w_gate[0], lw.w_up[0], lw.w_down[0])) < 1e-12
    # (iv) zero router: every logit ties -> S = (0..k-1), w = 1/k
    lw = _f64_layer(rng, H, 6, 4, I, Is)
    lw.w_router[:] = 0.0
    _, idx, w, gap = make(lw).forward(x)
    assert np.array_equal(idx, np.tile(np.arange(4, dtype=np.int32), (6, 1)))
    assert np.max(np.abs(w - 0.25)) < 1e-15 and np.all(gap == 0.0)


def pin_numpy_statement(make):
    """O7: the independent NumPy statement agrees (C0 within 1e-13, random within 1e-12)."""
    inp = synth.make("tiny_fp32")
    L = inp.layers[0]
    lw = LayerWeights(**L.arrays(), top_k=2)
    y, idx, w, _ = make(lw).forward(inp.x)
    y2, idx2, w2 = numpy_ref.layer(inp.x, L.w_router, L.w_gate, L.w_up, L.w_down,
                                   L.ws_gate, L.ws_up, L.ws_down, 2)
    assert np.array_equal(idx, idx2) and _rel(y, y2) < 1e-13 and np.max(np.abs(w - w2)) < 1e-13
    rng = np.random.default_rng(7)
    lw = _f64_layer(rng, 9, 7, 3, 4, 3)
    lw.rms_w = 1.0 + 0.1 * rng.standard_normal(9)
    x = rng.standard_normal((5, 9)) * 3.0
    r = rng.standard_normal((5, 9))
    y, idx, w, _ = make(lw).forward(x, residual=r)
    y2, idx2, w2 = numpy_ref.layer(x, lw.w_router, lw.w_gate, lw.w_up, lw.w_down, lw.ws_gate,
                                   lw.ws_up, lw.ws_down, 3, rms_w=lw.rms_w, residual=r)
    assert np.array_equal(idx, idx2) and _rel(y, y2) < 1e-12


def pin_rms_residual_gap(make):
    """R: pre-RMSNorm closed form (x = (3, 4, 0, ...), eps = 0: mean x^2 = 25/H, so the
    normalised input is (3, 4, 0, ...) * sqrt(H) / 5 times the scale g; and with eps = 1/2
    at H = 16); the residual is added exactly; the k-gap equals the k-th minus the
    (k+1)-th sorted logit."""
    rng = np.random.default_rng(8)
    H = 16
    lw = _f64_layer(rng, H, 8, 3, 6, 4)
    g = 1.0 + 0.1 * rng.standard_normal(H)
    x = np.zeros((1, H)); x[0, 0], x[0, 1] = 3.0, 4.0
    x_normed = x * math.sqrt(H) / 5.0 * g
    y_plain, idx_plain, *_ = make(lw).forward(x_normed)
    normed = LayerWeights(lw.w_router, lw.w_gate, lw.w_up, lw.w_down, lw.ws_gate, lw.ws_up,
                          lw.ws_down, rms_w=g, rms_eps=0.0, top_k=3)
    y_rms, idx_rms, *_ = make(normed).forward(x * 7.0)   # RMSNorm is scale-invariant
    assert np.array_equal(idx_rms, idx_plain) and _rel(y_rms, y_plain) < 1e-13
    y_raw, *_ = make(lw).forward(x * 7.0)
    assert _rel(y_raw, y_plain) > 1e-3          # the norm matters: the pin is not vacuous
    # eps sits inside the square root: eps = 1/2 gives mean x^2 + eps = 25/16 + 8/16, so the
    # normalised input is (3, 4, 0, ...) * 4 / sqrt(33) times g
    with_eps = LayerWeights(lw.w_router, lw.w_gate, lw.w_up, lw.w_down, lw.ws_gate, lw.ws_up,
                            lw.ws_down, rms_w=g, rms_eps=0.5, top_k=3)
    y_eps, idx_eps, *_ = make(with_eps).forward(x)
    y_ref, idx_ref, *_ = make(lw).forward(x * 4.0 / math.sqrt(33.0) * g)
    assert np.array_equal(idx_eps, idx_ref) and _rel(y_eps, y_ref) < 1e-13
    x = rng.standard_normal((7, H))
    r = rng.standard_normal((7, H))
    o = make(lw)
    y0, *_ = o.forward(x)
    y1, *_ = o.forward(x, residual=r)
    assert np.max(np.abs((y1 - y0) - r)) < 1e-13
    logits, idx, _, gap = o.route(x)
    srt = -np.sort(-logits, axis=1)
    assert np.max(np.abs(gap - (srt[:, 2] - srt[:, 3]))) < 1e-15
    assert np.max(np.abs(logits - x @ lw.w_router.T)) < 1e-12


@functools.lru_cache(maxsize=1)
def _talker_sample():
    """Talker decode weights (bf16 bits and their exact fp64 values), three of its tokens,
    and the brute-force dense evaluation of all E experts on them (numpy fp64, once)."""
    inp = synth.make("talker_decode")
    L = inp.layers[0]
    W = {n: numpy_ref.widen(a) for n, a in L.arrays().items()}
    rows = [0, 3, 7]
    x = numpy_ref.widen(inp.x[rows])
    k = inp.workload.k
    logits = x @ W["w_router"].T
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    g = np.einsum("eih,th->tei", W["w_gate"], x)
    u = np.einsum("eih,th->tei", W["w_up"], x)
    every = np.einsum("ehi,tei->teh", W["w_down"], _silu(g) * u)     # [T, E, H]: all experts
    S = np.array([sorted(range(p.shape[1]), key=lambda e: (-logits[t, e], e))[:k]
                  for t in range(len(rows))], dtype=np.int32)
    mask = np.zeros_like(p)
    np.put_along_axis(mask, S, 1.0, axis=1)
    wts = mask * p / (mask * p).sum(1, keepdims=True)
    y = np.einsum("te,teh->th", wts, every) + _dense_swiglu(x, W["ws_gate"], W["ws_up"],
                                                            W["ws_down"])
    return inp, L, W, rows, x, S, y


def pin_bf16_talker_size(make):
    """O8: at H=1024, E=128, k=6, I=384, I_s=768 with bf16 storage, the oracle on the bit
    patterns equals the oracle on their exact fp64 values bit for bit (bf16 is the upper
    half of a binary32), and both match the brute-force dense evaluation within 1e-12."""
    inp, L, W, rows, x, S, y_ref = _talker_sample()
    k = inp.workload.k
    y_bf, idx_bf, w_bf, _ = make(LayerWeights(**L.arrays(), top_k=k)).forward(inp.x[rows])
    y_64, idx_64, w_64, _ = make(LayerWeights(**W, top_k=k)).forward(x)
    assert np.array_equal(idx_bf, idx_64) and np.array_equal(y_bf, y_64)
    assert np.array_equal(w_bf, w_64)
    assert np.array_equal(idx_bf, S)
    assert _rel(y_bf, y_ref) < 1e-12


def pin_forced_routing(make):
    """O9: forward(x, forced_idx=S') uses the sets S' as given: forcing the oracle's own
    selection is the identity (bit for bit), and any other set gives the dense evaluation
    of every expert masked to S', weights p_i / sum_{j in S'} p_j, indices in S' order."""
    rng = np.random.default_rng(9)
    H, E, k = 10, 7, 3
    lw = _f64_layer(rng, H, E, k, 6, 5)
    x = rng.standard_normal((6, H))
    o = make(lw)
    y, idx, w, _ = o.forward(x)
    y2, idx2, w2, _ = o.forward(x, forced_idx=idx)
    assert np.array_equal(y2, y) and np.array_equal(idx2, idx) and np.array_equal(w2, w)
    forced = np.array([rng.permutation(E)[:k] for _ in range(x.shape[0])], dtype=np.int32)
    y3, idx3, w3, _ = o.forward(x, forced_idx=forced)
    assert np.array_equal(idx3, forced)
    logits = x @ lw.w_router.T
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    every = np.stack([_dense_swiglu(x, lw.w_gate[e], lw.w_up[e], lw.w_down[e])
                      for e in range(E)], axis=1)
    mask = np.zeros_like(p)
    np.put_along_axis(mask, forced, 1.0, axis=1)
    wts = mask * p / (mask * p).sum(1, keepdims=True)
    ref = np.einsum("te,teh->th", wts, every) + _dense_swiglu(x, lw.ws_gate, lw.ws_up, lw.ws_down)
    assert _rel(y3, ref) < 1e-12
    assert np.max(np.abs(w3 - np.take_along_axis(wts, forced, axis=1))) < 1e-15


ALL_PINS = [pin_weights_sum_to_one, pin_brute_force_dense, pin_expert_permutation,
            pin_token_independence, pin_hand_case, pin_special_cases, pin_numpy_statement,
            pin_rms_residual_gap, pin_bf16_talker_size, pin_forced_routing]

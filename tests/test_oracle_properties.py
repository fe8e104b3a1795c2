"""Properties of the fp64 oracle over many small random layer shapes (hypothesis,
derandomised so every run draws the same cases).

Each case draws H, E, k <= E, I, I_s (0 = no shared expert), T and fp64 weights, then
checks what must hold whatever the shape (routing and combine equation of page
"3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra ma ngu nghia c_0", section 3):

* y equals the brute-force dense evaluation of every expert masked to the Top-k set;
* the selected weights are positive and sum to 1, in selection order of descending
  logit, and the set is a Top-k of the logits;
* each token's output depends on that token alone (batch of one == row of the batch);
* scaling the router rows by c > 0 keeps the selection (softmax is increasing) and
  raises each weight ratio w_i / w_j to the power c.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from oracle import LayerWeights
from tests.pins import _rel, brute_force_dense

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@st.composite
def layers(draw):
    H = draw(st.integers(1, 12))
    E = draw(st.integers(1, 9))
    k = draw(st.integers(1, E))
    I = draw(st.integers(1, 7))
    Is = draw(st.sampled_from([0, 1, 5]))
    T = draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    n = lambda *s: rng.standard_normal(s) * 0.7
    lw = LayerWeights(n(E, H), n(E, I, H), n(E, I, H), n(E, H, I),
                      n(Is, H) if Is else None, n(Is, H) if Is else None,
                      n(H, Is) if Is else None, top_k=k)
    return lw, rng.standard_normal((T, H))


@SETTINGS
@given(layers())
def test_sparse_equals_masked_dense(case):
    lw, x = case
    y, idx, w, gap = oracle.Oracle(lw).forward(x)
    assert _rel(y, brute_force_dense(lw, x)) < 1e-11


@SETTINGS
@given(layers())
def test_selection_and_weights(case):
    lw, x = case
    H, E, k, _, _ = lw.dims
    o = oracle.Oracle(lw)
    logits, idx, w, gap = o.route(x)
    assert np.all(w > 0) and np.all(np.abs(w.sum(1) - 1) < 1e-12)
    for t in range(x.shape[0]):
        sel = logits[t, idx[t]]
        assert np.all(np.diff(sel) <= 0)                       # descending logit
        assert len(set(idx[t].tolist())) == k
        if k < E:
            rest = np.delete(logits[t], idx[t])
            assert sel.min() >= rest.max()                      # a Top-k of the logits
            assert abs(gap[t] - (sel.min() - rest.max())) < 1e-12
        else:
            assert gap[t] == np.inf                             # no (k+1)-th expert


@SETTINGS
@given(layers())
def test_tokens_are_independent(case):
    lw, x = case
    o = oracle.Oracle(lw)
    y, idx, _, _ = o.forward(x)
    for t in range(x.shape[0]):
        yt, it, _, _ = o.forward(x[t:t + 1])
        assert np.array_equal(yt[0], y[t]) and np.array_equal(it[0], idx[t])


@SETTINGS
@given(layers(), st.floats(0.25, 4.0))
def test_router_scale_sharpens_weights(case, c):
    lw, x = case
    H, E, k, _, _ = lw.dims
    o = oracle.Oracle(lw)
    _, idx, w, gap = o.forward(x)
    scaled = LayerWeights(lw.w_router * c, lw.w_gate, lw.w_up, lw.w_down, lw.ws_gate,
                          lw.ws_up, lw.ws_down, top_k=k)
    _, idx_c, w_c, _ = oracle.Oracle(scaled).forward(x)
    clear = gap > 1e-9                                          # no exact ties to reorder
    assert np.array_equal(idx_c[clear], idx[clear])
    for t in np.nonzero(clear)[0]:
        # w_i / w_0 = exp(l_i - l_0); scaling the logits by c raises the ratio to the c
        assert np.allclose(w_c[t] / w_c[t, 0], (w[t] / w[t, 0]) ** c, rtol=1e-9, atol=0)


def test_thread_count_does_not_change_results():
    """The oracle parallelises over tokens only, so any thread count gives the same bits
    (the parity tests and the timed baselines use different counts)."""
    import synth
    inp = synth.make("talker_decode")
    L, wl = inp.layers[0], inp.workload
    o = oracle.Oracle(LayerWeights(**L.arrays(), top_k=wl.k))
    ref = o.forward(inp.x, nthreads=1)
    for n in (2, 3, 0):
        out = o.forward(inp.x, nthreads=n)
        assert all(np.array_equal(a, b) for a, b in zip(out, ref))
    r1 = o.route(inp.x, nthreads=1)
    r0 = o.route(inp.x, nthreads=0)
    assert all(np.array_equal(a, b) for a, b in zip(r0, r1))

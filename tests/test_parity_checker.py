"""The parity checker (tests/parity.py) on the CPU, with planted "GPU" results.

The GPU tests trust compare() / assert_parity() to reject wrong outputs, wrong
weights and wrong expert sets, and to accept the one legitimate difference: a
near-tie token (k-th / (k+1)-th logit gap <= 1e-3) whose set differs, provided its
output matches the oracle re-evaluated with that set.  Here the results handed to
the checker are made from the oracle itself (exact, or deliberately altered), so
each verdict is known in advance.
"""
import numpy as np
import pytest

import oracle
from tests.parity import NEAR_TIE, TOL_W, TOL_Y, assert_parity, compare

H, E, K = 8, 6, 2


def _layer_with_near_tie(gap=1e-4, seed=11):
    """An fp64 layer and two tokens: token 0 has k-gap `gap`, token 1 a clear gap."""
    rng = np.random.default_rng(seed)
    n = lambda *s: rng.standard_normal(s) * 0.5
    wr = n(E, H)
    x = n(2, H)
    l0 = wr @ x[0]
    order = sorted(range(E), key=lambda e: (-l0[e], e))
    a, b = order[K - 1], order[K]
    wr[b] += ((l0[a] - gap) - l0[b]) * x[0] / (x[0] @ x[0])   # move l_b to l_a - gap
    lw = oracle.LayerWeights(wr, n(E, 16, H), n(E, 16, H), n(E, H, 16), n(12, H), n(12, H),
                             n(H, 12), top_k=K)
    o = oracle.Oracle(lw)
    _, idx, w, kgap = o.forward(x)
    assert kgap[0] <= NEAR_TIE and kgap[1] > NEAR_TIE
    return o, x, a, b


def test_exact_results_pass_and_near_ties_are_counted():
    o, x, _, _ = _layer_with_near_tie()
    y, idx, w, _ = o.forward(x)
    rep = compare(o, x, y.astype(np.float32), idx, w.astype(np.float32), "bf16")
    assert rep.near_ties == 1 and rep.set_mismatch_near == 0
    assert rep.rel_err < 1e-6 and rep.max_w_err < 1e-6
    assert_parity(rep, "bf16")
    assert_parity(rep, "f32")


def test_output_and_weight_errors_are_rejected():
    o, x, _, _ = _layer_with_near_tie()
    y, idx, w, _ = o.forward(x)
    for dtype in ("bf16", "f32"):
        bad_y = y.copy()
        bad_y[1, 3] += 1.5 * TOL_Y[dtype] * np.max(np.abs(y))
        with pytest.raises(AssertionError, match="output error"):
            assert_parity(compare(o, x, bad_y, idx, w, dtype), dtype)
        bad_w = w.copy()
        bad_w[1, 0] += 1.5 * TOL_W[dtype]
        with pytest.raises(AssertionError, match="weight error"):
            assert_parity(compare(o, x, y, idx, bad_w, dtype), dtype)


def test_swapped_set_on_a_clear_token_is_rejected():
    o, x, _, _ = _layer_with_near_tie()
    y, idx, w, _ = o.forward(x)
    bad = idx.copy()
    bad[1, K - 1] = next(e for e in range(E) if e not in idx[1])
    with pytest.raises(AssertionError, match="k-gap"):
        compare(o, x, y, bad, w, "bf16")


def test_near_tie_swap_is_accepted_only_with_its_own_output():
    o, x, a, b = _layer_with_near_tie()
    y, idx, w, _ = o.forward(x)
    alt = idx.copy()
    alt[0][list(idx[0]).index(a)] = b               # the (k+1)-th expert instead of the k-th
    y_alt, _, w_alt, _ = o.forward(x, forced_idx=alt)
    rep = compare(o, x, y_alt, alt, w_alt, "bf16")
    assert rep.set_mismatch_near == 1 and rep.rel_err < 1e-12 and rep.max_w_err < 1e-15
    assert_parity(rep, "f32")
    # the swapped set with the output of the original set is an output error
    with pytest.raises(AssertionError, match="output error"):
        assert_parity(compare(o, x, y, alt, w_alt, "f32"), "f32")


def test_near_tie_token_must_still_pick_a_valid_top_k():
    o, x, a, _ = _layer_with_near_tie()
    y, idx, w, _ = o.forward(x)
    lg = o.route(x)[0][0]
    worst = int(np.argmin(lg))                       # far below the k-th logit
    bad = idx.copy()
    bad[0][list(idx[0]).index(a)] = worst
    with pytest.raises(AssertionError, match="valid Top-k"):
        compare(o, x, y, bad, w, "bf16")

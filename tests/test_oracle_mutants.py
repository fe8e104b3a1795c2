"""Plant plausible mistakes in a copy of the C oracle; the pins must catch each.

Every mutant is the oracle source with one textual change (a dropped term, a
wrong sign, a wrong index, swapped operands...), compiled on the CPU into a
temporary library.  The test passes when at least one pin fails for it, which
shows the pins are sensitive to that class of slip.
"""
import os
import shutil
import tempfile

import pytest

import oracle
from tests import pins

MUTANTS = {
    "drop_shared_expert": ("for (int o = 0; o < H; ++o) acc[o] += eo[o];", ""),
    "silu_wrong_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "no_renormalisation": ("wsel[i] = p[sel[i]] / psum;", "wsel[i] = p[sel[i]];"),
    "ties_to_higher_index": ("(l[a] == l[b] && a < b)", "(l[a] == l[b] && a > b)"),
    "select_smallest": ("return l[a] > l[b] ||", "return l[a] < l[b] ||"),
    "gate_up_swapped": ("hbuf[i] = silu(g) * u;", "hbuf[i] = silu(u) * g;"),
    "down_of_next_expert": ("e * I, e * H, H, I", "e * I, ((e + 1) % E) * H, H, I"),
    "rms_sum_not_mean": ("ms /= (double)H;", ""),
    "kgap_wrong_pair": ("l[order[k - 1]] - l[order[k]]", "l[order[0]] - l[order[k]]"),
    "router_row_reversed": ("dot_row(w->w_router, c->dtype, (size_t)e, H, v)",
                            "dot_row(w->w_router, c->dtype, (size_t)(E - 1 - e), H, v)"),
    "residual_dropped": ("y[(size_t)t * H + o] = acc[o] + r;", "y[(size_t)t * H + o] = acc[o];"),
    "softmax_temperature": ("p[e] = exp(l[e] - m);", "p[e] = exp(2.0 * (l[e] - m));"),
    "routed_unweighted": ("acc[o] += ws[i] * eo[o];", "acc[o] += eo[o];"),
    "rms_eps_outside_sqrt": ("double r = sqrt(ms + c->rms_eps);",
                             "double r = sqrt(ms) + c->rms_eps;"),
    "rms_scale_dropped": ("v[j] = v[j] / r * load(w->rms_w, c->dtype, (size_t)j);",
                          "v[j] = v[j] / r;"),
    "shared_up_is_gate": ("swiglu(w->ws_gate, w->ws_up, w->ws_down,",
                          "swiglu(w->ws_gate, w->ws_gate, w->ws_down,"),
    "kgap_of_probabilities": ("l[order[k - 1]] - l[order[k]]", "p[order[k - 1]] - p[order[k]]"),
    "every_token_reads_row_0": ("v[j] = load(x, c->dtype, (size_t)t * H + j);",
                                "v[j] = load(x, c->dtype, (size_t)j);"),
    "down_rows_by_inter": ("e * I, e * H, H, I", "e * I, e * I, H, I"),
    "bf16_decoded_one_bit_low": ("uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;",
                                 "uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 15;"),
    "forced_sets_ignored": ("sel[i] = forced ? forced[i] : order[i];", "sel[i] = order[i];"),
    "forced_weights_from_own_sets": ("psum += p[sel[i]];", "psum += p[order[i]];"),
    "one_expert_short": ("for (int i = 0; i < k; ++i) psum += p[sel[i]];",
                         "for (int i = 0; i < k - 1; ++i) psum += p[sel[i]];"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, workdir):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.load_library(oracle.build(force=True, src=path,
                                           out=os.path.join(workdir, f"lib{name}.so")))
    make = lambda lw: oracle.Oracle(lw, lib=lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(make)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"

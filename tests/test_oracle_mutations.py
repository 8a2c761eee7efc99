"""Planted mistakes: each test builds a copy of the oracle with one plausible
bug (a dropped term, a wrong sign, index or operand) and shows that at least one
pin in test_oracle_pins.py fails against it.  Nothing here touches a GPU."""

import os
import subprocess

import pytest

import oracle as O
import test_oracle_backward_pins as bpins
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(O.__file__), "moe_oracle.c")

MUTATIONS = [
    ("tie to the higher index", "zt[e] > zt[best]) best = e;", "zt[e] >= zt[best]) best = e;",
     [pins.test_topk_ties_go_to_lower_index]),
    ("gate denominator drops a term", "for (int j = 0; j < k; ++j) den += exp",
     "for (int j = 0; j < 1; ++j) den += exp", [pins.test_gates_closed_forms]),
    ("capacity floors", "return (num + den - 1) / den;", "return num / den;",
     [pins.test_capacity_by_hand]),
    ("capacity adds one", "return (num + den - 1) / den;", "return num / den + 1;",
     [pins.test_capacity_by_hand]),
    ("silu sign", "a[i] / (1.0 + exp(-a[i]))", "a[i] / (1.0 + exp(a[i]))",
     [pins.test_ffn_silu_constant, pins.test_ffn_equals_library_composition]),
    ("gate and up swapped", "a[i] += xj * elem(w1, dtype, row + i);",
     "a[i] += xj * elem(w3, dtype, row + i);", [pins.test_ffn_silu_constant]),
    ("down projection transposed", "y[o] += a[i] * elem(w2, dtype, row + o);",
     "y[o] += a[i] * elem(w2, dtype, w_off2 + (int64_t)o * h + i);",
     [pins.test_ffn_equals_library_composition]),
    ("keeps one too many", "keep[t * k + j] = (r < C) ? 1 : 0;",
     "keep[t * k + j] = (r <= C) ? 1 : 0;", [pins.test_drops_match_queue_simulation]),
    ("aux not scaled by E", "out[0] = (double)E * aux;", "out[0] = aux;",
     [pins.test_aux_is_one_when_router_is_uniform]),
    ("aux uses kept counts", "double fe = (double)routed[e] /", "double fe = (double)kept[e] /",
     [pins.test_aux_uses_assignments_before_the_capacity_limit]),
    ("entropy in bits", "if (q > 0.0) ht -= q * log(q);", "if (q > 0.0) ht -= q * log2(q);",
     [pins.test_entropy_closed_form]),
    ("entropy sign", "if (q > 0.0) ht -= q * log(q);", "if (q > 0.0) ht += q * log(q);",
     [pins.test_aux_is_one_when_router_is_uniform]),
    ("bias ignored", "if (c->has_bias) s += (double)bias[e];", "",
     [pins.test_logits_equal_library_matmul]),
    ("gate not applied", "acc[o] += gate[t * k + j] * y[o];", "acc[o] += y[o];",
     [pins.test_identical_experts_return_that_expert]),
    ("shared experts skipped", "for (int s = 0; s < S; ++s) {", "for (int s = 0; s < 0; ++s) {",
     [pins.test_shared_experts_only]),
    ("dropped assignment still computed", "if (!keep[t * k + j]) continue;", "",
     [pins.test_fully_dropped_token_outputs_zero]),
    ("P averaged over experts", "Pe /= (double)T;", "Pe /= (double)E;",
     [pins.test_aux_is_one_when_assignment_is_uniform]),
    ("overflow counts kept", "dropped += (double)(routed[e] - kept[e]);",
     "dropped += (double)kept[e];", [pins.test_overflow_rate_closed_form]),
    ("reroute to the worst expert", "if (best < 0 || z[t * E + e] > z[t * E + best]) best = e;",
     "if (best < 0 || z[t * E + e] < z[t * E + best]) best = e;",
     [pins.test_reroute_hand_example]),
    ("reroute ignores capacity", "if (kept[e] >= C) continue;", "",
     [pins.test_reroute_matches_simulation_and_invariants]),
    ("reroute may reuse an expert", "if (used) continue;", "",
     [pins.test_reroute_matches_simulation_and_invariants]),
    # backward pass
    ("silu derivative drops a term", "sig * (1.0 + a[i] * (1.0 - sig))", "sig * (1.0 + a[i] * sig)",
     [bpins.test_backward_matches_finite_differences]),
    ("gate gradient sign", "dzt[it[j]] += gt[j] * (dgt[j] - m);",
     "dzt[it[j]] += gt[j] * (m - dgt[j]);", [bpins.test_backward_matches_finite_differences]),
    ("aux gradient misses the mean term", "dzt[e] += scale * p * (f[e] - q);",
     "dzt[e] += scale * p * f[e];", [bpins.test_backward_matches_finite_differences]),
    ("aux gradient not scaled by E", "const double scale = aux_coef * (double)E / (double)c->T;",
     "const double scale = aux_coef / (double)c->T;", [bpins.test_backward_matches_finite_differences]),
    ("output gradient not scaled by the gate", "const double dyo = g * elem(G, dtype, x_off + o);",
     "const double dyo = elem(G, dtype, x_off + o);", [bpins.test_backward_matches_finite_differences]),
    ("up gradient uses the gate pre-activation", "const double db = du[i] * silu;",
     "const double db = du[i] * a[i];", [bpins.test_backward_matches_finite_differences]),
    ("router term missing from dx",
     "            dxt[cc] += s;\n        }\n        for (int e = 0; e < E; ++e) db[e] += dzt[e];",
     "            (void)s;\n        }\n        for (int e = 0; e < E; ++e) db[e] += dzt[e];", [bpins.test_backward_matches_finite_differences]),
    ("dropped assignment differentiated",
     "            if (!keep[t * k + j]) continue;\n            const int64_t e = expert[t * k + j];\n"
     "            dg[j] = ffn_backward(d, h, c->dtype, x, t * d, G, gate[t * k + j], w1, w3, w2,\n"
     "                                 e * d * h, e * h * d, dw1,",
     "            const int64_t e = expert[t * k + j];\n"
     "            dg[j] = ffn_backward(d, h, c->dtype, x, t * d, G, gate[t * k + j], w1, w3, w2,\n"
     "                                 e * d * h, e * h * d, dw1,", [bpins.test_backward_matches_finite_differences]),
    ("gate gradient sent to the serving expert",
     "router_logit_grad(c, z + t * E, idx + t * k, gate + t * k, dg, f, aux_coef, dzt);\n"
     "        for (int cc = 0; cc < d; ++cc) {\n            const double xc",
     "router_logit_grad(c, z + t * E, expert + t * k, gate + t * k, dg, f, aux_coef, dzt);\n"
     "        for (int cc = 0; cc < d; ++cc) {\n            const double xc", [bpins.test_backward_matches_finite_differences]),
    ("router weight gradient transposed", "dWr[(int64_t)cc * E + e] += xc * dzt[e];",
     "dWr[(int64_t)e * d + cc] += xc * dzt[e];", [bpins.test_backward_matches_finite_differences]),
    ("down-projection gradient uses the gated input", "if (dw1) dw2[row + o] += u[i] * dyo;",
     "if (dw1) dw2[row + o] += a[i] * dyo;", [bpins.test_backward_matches_finite_differences]),
]


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    mut = src.replace(old, new, 1)
    cfile = tmp_path / f"{name}.c"
    cfile.write_text(mut)
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(so),
                           str(cfile), "-lm"])
    return str(so)


def _run(pin):
    params = getattr(pin, "pytestmark", [])
    names, args = None, []
    for m in params:
        if m.name == "parametrize":
            names, args = m.args[0], list(m.args[1])
    if args:
        multi = "," in names
        for a in args:
            if multi:
                pin(*a)
            else:
                pin(a)
    else:
        pin()


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(tmp_path, name, old, new, catchers):
    so = _build(tmp_path, name.replace(" ", "_"), old, new)
    caught = False
    with O.using_library(so):
        for pin in catchers:
            try:
                _run(pin)
            except AssertionError:
                caught = True
    assert caught, f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_the_same_pins(tmp_path):
    so = _build(tmp_path, "clean", "#include <math.h>", "#include <math.h>")
    with O.using_library(so):
        for _, _, _, catchers in MUTATIONS:
            for pin in catchers:
                _run(pin)

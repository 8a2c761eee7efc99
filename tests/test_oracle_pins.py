"""Pins for the fp64 oracle: each test checks the oracle against something other
than itself -- a value the pages print, a closed form, an invariant, a special
case that reduces to a library routine, or brute force on tiny inputs.

Page references: [Mixtral explained] "Mixtral 8x7B and MoE explained: sparse
mixture of experts, only 2 experts active per token"; [Routing explained]
"MoE routing fully explained: the expert-mixture structure Mixtral and DeepSeek
use, load balancing, capacity factor".
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from sparse_mixture_experts_22_b200 import inputs as I
from sparse_mixture_experts_22_b200.workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def rnd(shape, seed, std=1.0):
    return f32(np.random.default_rng(seed).standard_normal(shape) * std)


def np_silu(a):
    return a / (1.0 + np.exp(-a))


def np_ffn(x, w1, w3, w2):
    """Library composition of the SiLU-gated FFN (torch fp64 matmul + torch silu)."""
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    a = xt @ torch.from_numpy(np.asarray(w1, dtype=np.float64))
    b = xt @ torch.from_numpy(np.asarray(w3, dtype=np.float64))
    return ((torch.nn.functional.silu(a) * b) @ torch.from_numpy(
        np.asarray(w2, dtype=np.float64))).numpy()


def softmax(z):
    z = np.asarray(z, dtype=np.float64)
    return torch.softmax(torch.from_numpy(z), dim=-1).numpy()


def tiny_layer(T=16, d=24, h=40, E=6, k=2, cf=None, S=0, hs=0, seed=1, bias=None):
    cfg = O.make_cfg(T, d, h, E, k, S, hs, cf, "f32", bias is not None)
    inp = {
        "x": rnd((T, d), seed),
        "Wr": rnd((d, E), seed + 1, 1 / math.sqrt(d)),
        "bias": None if bias is None else f32(bias),
        "w1": rnd((E, d, h), seed + 2, 1 / math.sqrt(d)),
        "w3": rnd((E, d, h), seed + 3, 1 / math.sqrt(d)),
        "w2": rnd((E, h, d), seed + 4, 1 / math.sqrt(h)),
    }
    if S:
        inp["w1s"] = rnd((S, d, hs), seed + 5, 1 / math.sqrt(d))
        inp["w3s"] = rnd((S, d, hs), seed + 6, 1 / math.sqrt(d))
        inp["w2s"] = rnd((S, hs, d), seed + 7, 1 / math.sqrt(hs))
    return cfg, inp


# ---------------------------------------------------------------- capacity

def test_capacity_worked_example_from_page():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "capacity_worked_example.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows
    for T, E, k, num, den, C in (map(int, r) for r in rows):
        cfg = O.make_cfg(T, 8, 8, E, k, cf=(num, den))
        assert O.capacity(cfg) == C


def test_capacity_by_hand():
    # DeepSeek-style: 4096*6*1.5/160 = 230.4 -> 231 (a ceiling, not rounding)
    assert O.capacity(O.make_cfg(4096, 8, 8, 160, 6, cf=(3, 2))) == 231
    # 16384*2*1.5/8 = 6144 exactly: the ceiling must not add one
    assert O.capacity(O.make_cfg(16384, 8, 8, 8, 2, cf=(3, 2))) == 6144
    # no limit: at most T tokens can reach one expert
    assert O.capacity(O.make_cfg(77, 8, 8, 8, 2, cf=None)) == 77
    # the five workloads
    expect = {"prefill": 640, "deepseek": 231, "large": 6144}
    for name, C in expect.items():
        assert O.capacity(O.cfg_of(WORKLOADS[name])) == C


# ---------------------------------------------------------------- router

def test_logits_equal_library_matmul():
    cfg, inp = tiny_layer(T=20, d=33, E=7, bias=rnd(7, 9))
    z = O.logits(cfg, inp["x"], inp["Wr"], inp["bias"])
    ref = inp["x"].astype(np.float64) @ inp["Wr"].astype(np.float64) + inp["bias"]
    np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-12)


def test_logits_read_bf16_bytes():
    # bf16 input: the oracle must widen the raw bf16 bytes exactly
    xb = torch.randn(5, 16, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    Wr = rnd((16, 4), 4)
    cfg = O.make_cfg(5, 16, 8, 4, 1, dtype="bf16")
    z = O.logits(cfg, xb, Wr)
    ref = xb.double().numpy() @ Wr.astype(np.float64)
    np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("k", [1, 2, 3, 6])
def test_topk_equals_brute_force_subset(k):
    E, T = 6, 40
    z = np.random.default_rng(k).standard_normal((T, E))
    cfg = O.make_cfg(T, 4, 4, E, k)
    idx, gate = O.topk(cfg, z)
    for t in range(T):
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(z[t, list(s)]))
        assert sorted(idx[t]) == sorted(best)
        # descending-logit order
        assert all(z[t, idx[t, j]] >= z[t, idx[t, j + 1]] for j in range(k - 1))


def test_topk_ties_go_to_lower_index():
    z = np.array([[1.0, 3.0, 3.0, 0.5, 3.0],
                  [2.0, 2.0, 2.0, 2.0, 2.0],
                  [0.0, 1.0, 0.0, 1.0, -1.0]])
    cfg = O.make_cfg(3, 4, 4, 5, 2)
    idx, _ = O.topk(cfg, z)
    assert idx.tolist() == [[1, 2], [0, 1], [1, 3]]


def test_gates_closed_forms():
    # two kept logits ln 3 apart -> gates 3/4 and 1/4
    z = np.array([[0.0, math.log(3.0), -5.0, -6.0]])
    idx, gate = O.topk(O.make_cfg(1, 4, 4, 4, 2), z)
    assert idx.tolist() == [[1, 0]]
    np.testing.assert_allclose(gate, [[0.75, 0.25]], rtol=1e-14)
    # k = 1: the single gate is exactly 1 (Switch-style routing, "1-2 experts")
    z = np.random.default_rng(5).standard_normal((30, 8)) * 4
    _, g1 = O.topk(O.make_cfg(30, 4, 4, 8, 1), z)
    assert np.all(g1 == 1.0)
    # k = E: the gates are the full softmax, in top-k order
    idx, gE = O.topk(O.make_cfg(30, 4, 4, 8, 8), z)
    np.testing.assert_allclose(gE, np.take_along_axis(softmax(z), idx, 1), rtol=1e-13)
    # any k: gates sum to 1 and equal the renormalised full softmax
    idx, g3 = O.topk(O.make_cfg(30, 4, 4, 8, 3), z)
    np.testing.assert_allclose(g3.sum(1), 1.0, rtol=1e-14)
    p = np.take_along_axis(softmax(z), idx, 1)
    np.testing.assert_allclose(g3, p / p.sum(1, keepdims=True), rtol=1e-13)


def test_probs_are_library_softmax():
    z = np.random.default_rng(6).standard_normal((25, 9)) * 3
    cfg = O.make_cfg(25, 4, 4, 9, 2)
    np.testing.assert_allclose(O.probs(cfg, z), softmax(z), rtol=1e-13)
    zero = np.zeros((3, 9))
    np.testing.assert_allclose(O.probs(O.make_cfg(3, 4, 4, 9, 2), zero), 1 / 9, rtol=1e-15)


# ---------------------------------------------------------------- expert FFN

def test_ffn_one_hot_closed_form():
    # x = s * e_j and w2 = I  ->  y_i = silu(s * w1[j, i]) * s * w3[j, i]
    d = h = 8
    w1, w3 = rnd((d, h), 11), rnd((d, h), 12)
    w2 = f32(np.eye(h))
    for j, s in [(0, 1.0), (5, -2.0), (7, 0.5)]:
        x = np.zeros(d, dtype=np.float32)
        x[j] = s
        y = O.ffn(d, h, "f32", x, w1, w3, w2)
        a = torch.tensor(s * w1[j].astype(np.float64))
        ref = (torch.nn.functional.silu(a) * s * torch.tensor(w3[j].astype(np.float64)))
        np.testing.assert_allclose(y, ref.numpy(), rtol=1e-13, atol=1e-15)


def test_ffn_silu_constant():
    # silu(ln 3) = ln 3 / (1 + 1/3) = 0.75 ln 3; silu(0) = 0; gate is w1, up is w3
    d = h = 2
    w1 = f32([[math.log(3.0), 0.0], [0.0, 0.0]])
    w3 = f32([[2.0, 5.0], [0.0, 0.0]])
    w2 = f32(np.eye(2))
    y = O.ffn(d, h, "f32", f32([1.0, 0.0]), w1, w3, w2)
    # w1 holds ln 3 rounded to fp32, so the match is to fp32 resolution
    np.testing.assert_allclose(y, [0.75 * math.log(3.0) * 2.0, 0.0], rtol=1e-7, atol=0)
    # swapping the roles of w1 and w3 would give silu(2) * ln 3 instead
    assert abs(y[0] - 2.0 / (1.0 + math.exp(-2.0)) * math.log(3.0)) > 0.1


def test_ffn_equals_library_composition():
    d, h = 24, 40  # d != h so a transposed operand cannot pass
    x, w1, w3 = rnd(d, 1), rnd((d, h), 2, 0.2), rnd((d, h), 3, 0.2)
    w2 = rnd((h, d), 4, 0.2)
    y = O.ffn(d, h, "f32", x, w1, w3, w2)
    np.testing.assert_allclose(y, np_ffn(x[None], w1, w3, w2)[0], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- whole layer

def test_identical_experts_return_that_expert():
    # gates over the kept experts sum to 1, so identical experts give FFN(x)
    cfg, inp = tiny_layer(T=12, E=5, k=3)
    for n in ("w1", "w3", "w2"):
        inp[n] = f32(np.repeat(inp[n][:1], 5, axis=0))
    r = O.forward(cfg, inp)
    ref = np_ffn(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_k_equals_E_is_dense_softmax_mixture():
    cfg, inp = tiny_layer(T=10, E=4, k=4)
    r = O.forward(cfg, inp)
    z = inp["x"].astype(np.float64) @ inp["Wr"].astype(np.float64)
    p = softmax(z)
    ref = sum(p[:, e:e + 1] * np_ffn(inp["x"], inp["w1"][e], inp["w3"][e], inp["w2"][e])
              for e in range(4))
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_single_expert_is_gated_ffn():
    cfg, inp = tiny_layer(T=7, E=1, k=1)
    r = O.forward(cfg, inp)
    ref = np_ffn(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_layer_brute_force_over_subsets():
    E, k, T = 5, 2, 9
    cfg, inp = tiny_layer(T=T, E=E, k=k)
    r = O.forward(cfg, inp)
    z = inp["x"].astype(np.float64) @ inp["Wr"].astype(np.float64)
    Y = [np_ffn(inp["x"], inp["w1"][e], inp["w3"][e], inp["w2"][e]) for e in range(E)]
    for t in range(T):
        ref = np.zeros(cfg.d)
        for S in itertools.combinations(range(E), k):
            others = [e for e in range(E) if e not in S]
            if min(z[t, list(S)]) > max(z[t, others]):     # S is the top-k set
                w = softmax(z[t, list(S)])
                ref += sum(w[i] * Y[e][t] for i, e in enumerate(S))
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-11, atol=1e-13)


def test_unselected_experts_are_never_read():
    # "most experts are not even computed": NaN weights in unselected experts
    cfg, inp = tiny_layer(T=6, E=6, k=2, bias=[30.0, 30.0, 0, 0, 0, 0])
    for n in ("w1", "w3", "w2"):
        inp[n][2:] = np.nan
    r = O.forward(cfg, inp)
    assert set(np.unique(r["idx"])) == {0, 1}
    assert np.all(np.isfinite(r["out"]))


def test_shared_experts_only():
    # routed experts output zero -> the layer is the sum of the shared FFNs
    cfg, inp = tiny_layer(T=8, E=4, k=2, S=2, hs=16)
    inp["w2"][:] = 0
    r = O.forward(cfg, inp)
    ref = sum(np_ffn(inp["x"], inp["w1s"][s], inp["w3s"][s], inp["w2s"][s]) for s in range(2))
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_shared_plus_routed():
    cfg, inp = tiny_layer(T=8, E=4, k=4, S=2, hs=16)
    r = O.forward(cfg, inp)
    z = inp["x"].astype(np.float64) @ inp["Wr"].astype(np.float64)
    p = softmax(z)
    ref = sum(p[:, e:e + 1] * np_ffn(inp["x"], inp["w1"][e], inp["w3"][e], inp["w2"][e])
              for e in range(4))
    ref = ref + sum(np_ffn(inp["x"], inp["w1s"][s], inp["w3s"][s], inp["w2s"][s])
                    for s in range(2))
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_token_permutation_equivariance_without_capacity():
    cfg, inp = tiny_layer(T=14, E=5, k=2)
    r = O.forward(cfg, inp)
    perm = np.random.default_rng(3).permutation(14)
    inp2 = dict(inp)
    inp2["x"] = f32(inp["x"][perm])
    r2 = O.forward(cfg, inp2)
    np.testing.assert_allclose(r2["out"], r["out"][perm], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- capacity and drops

def queue_sim(idx, E, C):
    """Brute-force per-expert queues in token order."""
    routed = [0] * E
    keep = np.zeros(idx.shape, dtype=bool)
    for t in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            keep[t, j] = routed[e] < C
            routed[e] += 1
    return np.array(routed), keep


@pytest.mark.parametrize("cf", [(1, 2), (3, 4), (5, 4), (3, 2)])
def test_drops_match_queue_simulation(cf):
    T, E, k = 64, 5, 2
    cfg, inp = tiny_layer(T=T, E=E, k=k, cf=cf, bias=[1.5, 1.0, 0.5, 0.0, -0.5])
    r = O.forward(cfg, inp)
    C = math.ceil(T * k * cf[0] / (E * cf[1]))
    assert r["C"] == C
    routed, keep = queue_sim(r["idx"], E, C)
    assert r["routed"].tolist() == routed.tolist()
    assert r["kept"].tolist() == np.minimum(routed, C).tolist()
    assert r["routed"].sum() == T * k
    assert np.array_equal(r["keep"].astype(bool), keep)
    assert np.array_equal(r["keep"].astype(bool), r["rank"] < C)
    # output = sum over kept assignments only, gates not renormalised
    Y = [np_ffn(inp["x"], inp["w1"][e], inp["w3"][e], inp["w2"][e]) for e in range(E)]
    ref = np.zeros((T, cfg.d))
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                ref[t] += r["gate"][t, j] * Y[r["idx"][t, j]][t]
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_fully_dropped_token_outputs_zero():
    # every token prefers experts 0 and 1; C = 1 keeps only token 0
    T, E = 6, 4
    cfg, inp = tiny_layer(T=T, E=E, k=2, cf=(1, 6), bias=[40.0, 39.0, 0.0, 0.0])
    r = O.forward(cfg, inp)
    assert r["C"] == 1
    assert r["keep"].sum() == 2 and r["keep"][0].all()
    assert np.all(r["out"][1:] == 0.0)
    np.testing.assert_allclose(r["stats"]["overflow_rate"], (T * 2 - 2) / (T * 2))


def test_overflow_rate_closed_form():
    # T=8, E=2, k=1, all tokens to expert 0, cf=1/2 -> C=2: 6 of 8 dropped
    cfg, inp = tiny_layer(T=8, E=2, k=1, cf=(1, 2), bias=[50.0, 0.0])
    r = O.forward(cfg, inp)
    assert r["C"] == 2
    assert r["routed"].tolist() == [8, 0] and r["kept"].tolist() == [2, 0]
    assert r["stats"]["overflow_rate"] == 0.75


# ---------------------------------------------------------------- aux loss and entropy

def test_aux_is_one_when_router_is_uniform():
    # W_r = 0, no bias: P_e = 1/E whatever the hard routing -> aux = 1
    cfg, inp = tiny_layer(T=20, E=8, k=2)
    inp["Wr"][:] = 0
    r = O.forward(cfg, inp)
    assert r["routed"].tolist() == [20, 20, 0, 0, 0, 0, 0, 0]  # ties -> lower index
    assert abs(r["stats"]["aux_loss"] - 1.0) < 1e-14
    assert abs(r["stats"]["mean_entropy"] - math.log(8)) < 1e-14


def test_aux_is_one_when_assignment_is_uniform():
    # token t strongly prefers expert t mod E, so f_e = 1/E; P is far from uniform
    T, E = 24, 4
    cfg = O.make_cfg(T, E, 8, E, 1, dtype="f32")
    x = f32(np.stack([np.eye(E)[t % E] * (1.0 + 0.1 * (t % 3)) for t in range(T)]))
    Wr = f32(np.diag([2.0, 3.0, 1.0, 0.5]))
    r = O.route(cfg, x, Wr)
    assert r["routed"].tolist() == [6, 6, 6, 6]
    assert abs(r["stats"]["aux_loss"] - 1.0) < 1e-13
    assert r["stats"]["P"].std() > 0.01


def test_aux_collapse_reaches_E():
    # k=1, every token to expert 0 with near-one-hot probabilities -> aux -> E
    E, T = 8, 10
    cfg = O.make_cfg(T, 4, 4, E, 1, has_bias=True)
    x = np.zeros((T, 4), dtype=np.float32)
    b = f32([50.0] + [0.0] * (E - 1))
    r = O.route(cfg, x, np.zeros((4, E), dtype=np.float32), b)
    P0 = 1.0 / (1.0 + (E - 1) * math.exp(-50.0))
    assert abs(r["stats"]["aux_loss"] - E * P0) < 1e-12
    assert r["stats"]["mean_entropy"] < 1e-15


def test_aux_grows_with_skew():
    wl = WORKLOADS["prefill"].scaled(T=512, d=64, zipf_s=0.0)
    Wr = I.router_weights(wl)
    x, _ = I.tokens(wl, Wr=Wr, b=torch.zeros(wl.E))
    aux = []
    for s in (0.0, 1.0, 2.0):
        cfg = O.make_cfg(512, 64, 8, 8, 2, cf=None, dtype="bf16", has_bias=True)
        aux.append(O.route(cfg, x, Wr, I.zipf_bias(8, s))["stats"]["aux_loss"])
    assert aux[0] < aux[1] < aux[2]


def test_entropy_closed_form():
    # two experts with logits 0 and ln 3: p = (1/4, 3/4)
    cfg = O.make_cfg(1, 1, 4, 2, 1, has_bias=True)
    b = f32([0.0, math.log(3.0)])
    r = O.route(cfg, np.zeros((1, 1), dtype=np.float32), np.zeros((1, 2), np.float32), b)
    p1 = 1.0 / (1.0 + math.exp(float(b[1])))
    expect = -(p1 * math.log(p1) + (1 - p1) * math.log(1 - p1))
    assert abs(expect - 0.5623351446188083) < 1e-7  # -(1/4 ln 1/4 + 3/4 ln 3/4)
    assert abs(r["stats"]["mean_entropy"] - expect) < 1e-14
    # aux = E * (f0 P0 + f1 P1) with f = (0, 1): 2 * P1
    assert abs(r["stats"]["aux_loss"] - 2 * (1 - p1)) < 1e-14


def test_stats_of_empty_batch():
    cfg = O.make_cfg(0, 4, 4, 3, 2)
    r = O.route(cfg, np.zeros((0, 4), np.float32), np.zeros((4, 3), np.float32))
    assert r["routed"].tolist() == [0, 0, 0]
    assert r["stats"]["aux_loss"] == 0.0 and r["stats"]["overflow_rate"] == 0.0


# ---------------------------------------------------------------- generator

def test_generator_is_deterministic_and_tie_free():
    wl = WORKLOADS["deepseek"].scaled(T=256, d=128)
    a = I.layer_inputs(wl, weights=False)
    b = I.layer_inputs(wl, weights=False)
    assert torch.equal(a["x"], b["x"])
    z = a["x"].double() @ a["Wr"].double()
    top = torch.topk(z, wl.k + 1, dim=1).values
    assert torch.all(top[:, wl.k - 1] - top[:, wl.k] >= I.TIE_GAP)


def test_zipf_bias_values():
    b = I.zipf_bias(4, 1.2)
    np.testing.assert_allclose(b.numpy(), [0.0, -1.2 * math.log(2), -1.2 * math.log(3),
                                           -1.2 * math.log(4)], rtol=1e-6)


def test_aux_uses_assignments_before_the_capacity_limit():
    # f counts what the router assigned, so capacity (drops) cannot change aux,
    # while the overflow rate does change
    cfg_inf, inp = tiny_layer(T=48, E=4, k=2, bias=[2.0, 1.0, 0.0, -1.0])
    cfg_cap, _ = tiny_layer(T=48, E=4, k=2, cf=(1, 2), bias=[2.0, 1.0, 0.0, -1.0])
    a = O.route(cfg_inf, inp["x"], inp["Wr"], inp["bias"])
    b = O.route(cfg_cap, inp["x"], inp["Wr"], inp["bias"])
    assert b["stats"]["overflow_rate"] > 0.2 and a["stats"]["overflow_rate"] == 0.0
    assert a["stats"]["aux_loss"] == b["stats"]["aux_loss"]


# ---------------------------------------------------------------- overflow rerouted to a spare expert

def test_reroute_hand_example():
    # 4 tokens all preferring expert 0 (logits 3, 2, 1), k=1, C=1: token 0 keeps
    # expert 0, token 1 moves to expert 1, token 2 to expert 2, token 3 finds no room
    cfg = O.make_cfg(4, 3, 4, 3, 1, cf=(3, 4), has_bias=True, overflow="reroute")
    r = O.route(cfg, np.zeros((4, 3), np.float32), np.zeros((3, 3), np.float32),
                f32([3.0, 2.0, 1.0]))
    assert r["C"] == 1
    assert r["expert"][:, 0].tolist() == [0, 1, 2, 0]
    assert r["keep"][:, 0].tolist() == [1, 1, 1, 0]
    assert r["kept"].tolist() == [1, 1, 1] and r["routed"].tolist() == [4, 0, 0]
    assert r["stats"]["overflow_rate"] == 0.25


def reroute_sim(z, idx, E, C):
    """Brute-force arrival-order queues, then reroutes in token order."""
    T, k = idx.shape
    fill = [0] * E
    keep = np.zeros(idx.shape, bool)
    expert = idx.copy()
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            keep[t, j] = fill[e] < C
            fill[e] += 1
    fill = [min(f, C) for f in fill]
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                continue
            cands = [e for e in range(E) if fill[e] < C and e not in idx[t] and e not in expert[t]]
            if not cands:
                continue
            best = sorted(cands, key=lambda e: (-z[t, e], e))[0]
            expert[t, j] = best
            keep[t, j] = True
            fill[best] += 1
    return expert, keep, fill


@pytest.mark.parametrize("cf,k", [((1, 2), 2), ((3, 4), 2), ((1, 1), 1), ((5, 4), 3)])
def test_reroute_matches_simulation_and_invariants(cf, k):
    T, E = 48, 6
    cfg, inp = tiny_layer(T=T, E=E, k=k, cf=cf, bias=[2.0, 1.5, 1.0, 0.5, 0.0, -0.5])
    cfg.overflow = O.OVERFLOW["reroute"]
    r = O.forward(cfg, inp)
    expert, keep, fill = reroute_sim(r["z"], r["idx"], E, r["C"])
    assert np.array_equal(r["expert"], expert)
    assert np.array_equal(r["keep"].astype(bool), keep)
    assert r["kept"].tolist() == fill
    # no expert over capacity; no token uses an expert twice
    assert max(r["kept"]) <= r["C"]
    for t in range(T):
        served = [r["expert"][t, j] for j in range(k) if r["keep"][t, j]]
        assert len(served) == len(set(served))
    # an assignment left dropped had no free expert it could use
    for t in range(T):
        for j in range(k):
            if not r["keep"][t, j]:
                for e in range(E):
                    if e not in r["idx"][t] and e not in r["expert"][t]:
                        assert r["kept"][e] == r["C"]
    # the output sums the serving experts with the original gates
    Y = [np_ffn(inp["x"], inp["w1"][e], inp["w3"][e], inp["w2"][e]) for e in range(E)]
    ref = np.zeros((T, cfg.d))
    for t in range(T):
        for j in range(k):
            if r["keep"][t, j]:
                ref[t] += r["gate"][t, j] * Y[r["expert"][t, j]][t]
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-13)


def test_reroute_with_enough_room_drops_nothing():
    # k = 1 and E*C >= T: every overflowing token finds a spare expert
    cfg_d, inp = tiny_layer(T=40, E=4, k=1, cf=(1, 1), bias=[3.0, 0.0, 0.0, 0.0])
    cfg_r, _ = tiny_layer(T=40, E=4, k=1, cf=(1, 1), bias=[3.0, 0.0, 0.0, 0.0])
    cfg_r.overflow = O.OVERFLOW["reroute"]
    a = O.route(cfg_d, inp["x"], inp["Wr"], inp["bias"])
    b = O.route(cfg_r, inp["x"], inp["Wr"], inp["bias"])
    assert a["stats"]["overflow_rate"] > 0.3
    assert b["stats"]["overflow_rate"] == 0.0 and b["keep"].all()
    # aux counts the router's own choices, so rerouting leaves it unchanged
    assert a["stats"]["aux_loss"] == b["stats"]["aux_loss"]

"""Pins for the oracle's backward pass (oracle_backward and its sampled forms).

The backward is checked against things other than itself: central finite
differences of the oracle's own forward pass (the loss L = <G, out> + aux_coef
* aux, perturbing every input entry), torch autograd of closed forms the pages
fix (k = E without a capacity limit is the dense softmax mixture; E = 1 is the
plain SiLU-gated FFN), and closed forms of the load-balancing term (even
assignments give it zero gradient; identical experts give the gates none).

Page references: [Mixtral explained] "Mixtral 8x7B and MoE explained: sparse
mixture of experts, only 2 experts active per token"; [Routing explained]
"MoE routing fully explained: the expert-mixture structure Mixtral and DeepSeek
use, load balancing, capacity factor", "Easy explanation" ¶2-¶5.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O

EPS = 2.0 ** -14          # perturbation of one fp32 input entry
FD_ABS, FD_REL = 2e-7, 2e-6


def f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def rnd(shape, rng, std=1.0):
    return f32(rng.standard_normal(shape) * std)


def layer(T, d, h, E, k, S=0, hs=0, cf=None, bias=True, overflow="drop", seed=0, min_gap=0.02):
    """fp32 inputs whose sorted router logits are at least min_gap apart in
    every token (so the perturbations below never change the routing)."""
    for s in range(seed, seed + 1000):
        rng = np.random.default_rng(s)
        inp = {"x": rnd((T, d), rng), "Wr": rnd((d, E), rng, 1 / math.sqrt(d)),
               "bias": f32(-0.5 * np.log(np.arange(E) + 1.0)) if bias else None,
               "w1": rnd((E, d, h), rng, 1 / math.sqrt(d)),
               "w3": rnd((E, d, h), rng, 1 / math.sqrt(d)),
               "w2": rnd((E, h, d), rng, 1 / math.sqrt(h))}
        if S:
            inp["w1s"] = rnd((S, d, hs), rng, 1 / math.sqrt(d))
            inp["w3s"] = rnd((S, d, hs), rng, 1 / math.sqrt(d))
            inp["w2s"] = rnd((S, hs, d), rng, 1 / math.sqrt(hs))
        z = inp["x"].astype(np.float64) @ inp["Wr"].astype(np.float64)
        if bias:
            z = z + inp["bias"]
        srt = np.sort(z, axis=1)
        if E < 2 or (srt[:, 1:] - srt[:, :-1]).min() >= min_gap:
            cfg = O.make_cfg(T, d, h, E, k, S, hs, cf, "f32", bias, overflow)
            G = rnd((T, d), np.random.default_rng(s + 7919))
            return cfg, inp, G
    raise RuntimeError("no tie-free draw")


def loss(cfg, inp, G, alpha):
    r = O.forward(cfg, inp)
    L = float((G.astype(np.float64) * r["out"]).sum()) + alpha * r["stats"]["aux_loss"]
    return L, r


def same_routing(r0, r1):
    return (np.array_equal(r0["idx"], r1["idx"]) and np.array_equal(r0["keep"], r1["keep"])
            and np.array_equal(r0["expert"], r1["expert"]))


GRAD_OF = {"x": "dx", "Wr": "dWr", "bias": "db", "w1": "dw1", "w3": "dw3", "w2": "dw2",
           "w1s": "dw1s", "w3s": "dw3s", "w2s": "dw2s"}


def finite_difference_check(cfg, inp, G, alpha):
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g = O.backward(cfg, inp, r, G, alpha)
    L0, r0 = loss(cfg, inp, G, alpha)
    checked = 0
    worst = 0.0
    for name, gname in GRAD_OF.items():
        if inp.get(name) is None:
            continue
        base = inp[name]
        flat = base.reshape(-1)
        an = g[gname].reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            # fp32 steps: exact for |v| >= 2^-10; otherwise the rounded step is used
            up, dn = np.float32(v + np.float32(EPS)), np.float32(v - np.float32(EPS))
            flat[i] = up
            Lp, rp = loss(cfg, inp, G, alpha)
            flat[i] = dn
            Lm, rm = loss(cfg, inp, G, alpha)
            flat[i] = v
            assert same_routing(r0, rp) and same_routing(r0, rm), f"{name}[{i}] moved routing"
            fd = (Lp - Lm) / (float(up) - float(dn))
            err = abs(fd - an[i])
            worst = max(worst, err / (FD_ABS + FD_REL * abs(an[i])))
            assert err <= FD_ABS + FD_REL * abs(an[i]), (name, i, fd, an[i])
            checked += 1
    assert checked > 0
    return worst


# Small layers with capacity drops, shared experts, a router bias and a
# nonzero aux-loss weight; both overflow policies; k = 1 and k = 3.
FD_CASES = [
    dict(T=12, d=6, h=5, E=4, k=2, S=1, hs=3, cf=(1, 2), overflow="drop", alpha=0.7),
    dict(T=12, d=6, h=5, E=4, k=2, S=1, hs=3, cf=(1, 1), overflow="reroute", alpha=0.7),
    dict(T=10, d=5, h=4, E=5, k=3, cf=(3, 4), overflow="drop", alpha=1.3),
    dict(T=9, d=4, h=6, E=3, k=1, cf=None, overflow="drop", alpha=0.4),
]


@pytest.mark.parametrize("case", FD_CASES, ids=["drop", "reroute", "k3", "k1"])
def test_backward_matches_finite_differences(case):
    c = dict(case)
    alpha = c.pop("alpha")
    cfg, inp, G = layer(**c)
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    if cfg.cf_den:
        # the case must exercise the capacity rule
        assert int(r["keep"].sum()) < cfg.T * cfg.k or c["overflow"] == "reroute"
    finite_difference_check(cfg, inp, G, alpha)


def test_reroute_case_reroutes_something():
    cfg, inp, G = layer(**{k: v for k, v in FD_CASES[1].items() if k != "alpha"})
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    assert (r["expert"] != r["idx"]).any()


def _t(a):
    return torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)


def test_k_equals_E_is_dense_mixture_gradient():
    """k = E, no limit: out = sum_e softmax(z)_e FFN_e(x); every expert gets
    T/(T E) of the assignments, so the aux term is constant (zero gradient)."""
    cfg, inp, G = layer(T=7, d=5, h=6, E=3, k=3)
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g = O.backward(cfg, inp, r, G, 0.9)
    x, Wr, b = _t(inp["x"]), _t(inp["Wr"]), _t(inp["bias"])
    w1, w3, w2 = _t(inp["w1"]), _t(inp["w3"]), _t(inp["w2"])
    p = torch.softmax(x @ Wr + b, dim=-1)
    a = torch.einsum("td,edh->teh", x, w1)
    u = torch.nn.functional.silu(a) * torch.einsum("td,edh->teh", x, w3)
    y = torch.einsum("teh,ehd->ted", u, w2)
    out = torch.einsum("te,ted->td", p, y)
    (torch.from_numpy(G.astype(np.float64)) * out).sum().backward()
    for ref, name in ((x, "dx"), (Wr, "dWr"), (b, "db"), (w1, "dw1"), (w3, "dw3"), (w2, "dw2")):
        np.testing.assert_allclose(g[name], ref.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_single_expert_is_gated_ffn_gradient():
    """E = 1, k = 1: gate 1 and p = 1, so the router gets exactly zero gradient
    and the rest is the plain SiLU-gated FFN's."""
    cfg, inp, G = layer(T=6, d=5, h=7, E=1, k=1)
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g = O.backward(cfg, inp, r, G, 2.0)
    assert not g["dz"].any() and not g["dWr"].any() and not g["db"].any()
    x, w1, w3, w2 = _t(inp["x"]), _t(inp["w1"][0]), _t(inp["w3"][0]), _t(inp["w2"][0])
    out = (torch.nn.functional.silu(x @ w1) * (x @ w3)) @ w2
    (torch.from_numpy(G.astype(np.float64)) * out).sum().backward()
    np.testing.assert_allclose(g["dx"], x.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dw1"][0], w1.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dw3"][0], w3.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dw2"][0], w2.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_even_assignment_gives_aux_no_gradient():
    """f_e = 1/E for every expert: sum_e f_e P_e = 1/E whatever the router
    does, so the aux term's gradient is zero."""
    cfg, inp, G = layer(T=8, d=4, h=4, E=4, k=2)
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    r = dict(r)
    r["routed"] = np.full(cfg.E, cfg.T * cfg.k // cfg.E, dtype=np.int32)
    g = O.backward(cfg, inp, r, np.zeros_like(G), 5.0)
    assert np.abs(g["dz"]).max() < 1e-15


def test_identical_experts_give_gates_no_gradient():
    """All experts equal, no limit: every kept output is the same y, so
    dg_j = <G, y> for all j and the softmax-over-k gradient vanishes; dx is
    the single expert's."""
    cfg, inp, G = layer(T=6, d=5, h=4, E=4, k=2)
    for n in ("w1", "w3", "w2"):
        inp[n][:] = inp[n][0]
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g = O.backward(cfg, inp, r, G, 0.0)
    assert np.abs(g["dz"]).max() < 1e-13
    cfg1 = O.make_cfg(6, 5, 4, 1, 1, dtype="f32")
    one = {"x": inp["x"], "Wr": f32(np.zeros((5, 1))), "bias": None,
           "w1": inp["w1"][:1].copy(), "w3": inp["w3"][:1].copy(), "w2": inp["w2"][:1].copy()}
    r1 = O.route(cfg1, one["x"], one["Wr"])
    g1 = O.backward(cfg1, one, r1, G, 0.0)
    np.testing.assert_allclose(g["dx"], g1["dx"], rtol=1e-12, atol=1e-13)
    # the expert weights' gradient sums over experts to the single expert's
    np.testing.assert_allclose(g["dw1"].sum(0), g1["dw1"][0], rtol=1e-12, atol=1e-13)


def test_bf16_bytes_give_the_same_gradient():
    cfg, inp, G = layer(T=8, d=6, h=4, E=4, k=2, cf=(1, 1))
    # round every layer-dtype input to bf16 values, then compare the bf16-byte
    # and fp32 forms of the same numbers
    for n in ("x", "w1", "w3", "w2"):
        inp[n] = f32(torch.from_numpy(inp[n]).to(torch.bfloat16).float().numpy())
    Gr = f32(torch.from_numpy(G).to(torch.bfloat16).float().numpy())
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g32 = O.backward(cfg, inp, r, Gr, 0.3)
    cfgb = O.make_cfg(8, 6, 4, 4, 2, cf=(1, 1), dtype="bf16", has_bias=True)
    inb = dict(inp)
    for n in ("x", "w1", "w3", "w2"):
        inb[n] = torch.from_numpy(inp[n]).to(torch.bfloat16).contiguous()
    gb = O.backward(cfgb, inb, r, torch.from_numpy(Gr).to(torch.bfloat16).contiguous(), 0.3)
    for n in g32:
        np.testing.assert_array_equal(g32[n], gb[n])


def test_sampled_rows_and_blocks_equal_the_full_backward():
    """backward_rows / wgrad_block (used at full size) against the full pass."""
    for overflow in ("drop", "reroute"):
        cfg, inp, G = layer(T=14, d=6, h=5, E=4, k=2, S=2, hs=3, cf=(1, 2), overflow=overflow)
        r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
        g = O.backward(cfg, inp, r, G, 0.6)
        rows = [0, 3, 13, 7]
        s = O.backward_rows(cfg, inp, r, G, 0.6, rows)
        np.testing.assert_allclose(s["dx"], g["dx"][rows], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(s["dz"], g["dz"][rows], rtol=1e-12, atol=1e-14)
        hi, ci = [4, 0, 2], [5, 1]
        for e in range(cfg.E):
            b = O.wgrad_block(cfg, inp, r, G, e, hi, ci)
            np.testing.assert_allclose(b["dw1"], g["dw1"][e][np.ix_(ci, hi)].T, rtol=1e-12,
                                       atol=1e-14)
            np.testing.assert_allclose(b["dw3"], g["dw3"][e][np.ix_(ci, hi)].T, rtol=1e-12,
                                       atol=1e-14)
            np.testing.assert_allclose(b["dw2"], g["dw2"][e][np.ix_(hi, ci)], rtol=1e-12,
                                       atol=1e-14)
        for s_ in range(cfg.n_shared):
            b = O.wgrad_block(cfg, inp, r, G, s_, [2, 0], ci, shared=True)
            np.testing.assert_allclose(b["dw1"], g["dw1s"][s_][np.ix_(ci, [2, 0])].T,
                                       rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(b["dw2"], g["dw2s"][s_][np.ix_([2, 0], ci)],
                                       rtol=1e-12, atol=1e-14)


def test_router_gradient_rows_sum_to_zero():
    """Both the softmax-over-k and the full-softmax terms have zero sum over
    the experts, for every token (a property used at full size)."""
    cfg, inp, G = layer(T=11, d=6, h=4, E=5, k=2, cf=(1, 2))
    r = O.route(cfg, inp["x"], inp["Wr"], inp["bias"])
    g = O.backward(cfg, inp, r, G, 1.5)
    assert np.abs(g["dz"].sum(1)).max() < 1e-13
    assert np.abs(g["db"].sum()) < 1e-12
    assert np.abs(g["dWr"].sum(1)).max() < 1e-12


def test_empty_batch_backward():
    cfg, inp, G = layer(T=3, d=4, h=4, E=2, k=1)
    cfg0 = O.make_cfg(0, 4, 4, 2, 1, dtype="f32", has_bias=True)
    e = {"x": f32(np.zeros((0, 4))), "Wr": inp["Wr"], "bias": inp["bias"], "w1": inp["w1"],
         "w3": inp["w3"], "w2": inp["w2"]}
    r = O.route(cfg0, e["x"], e["Wr"], e["bias"])
    g = O.backward(cfg0, e, r, f32(np.zeros((0, 4))), 1.0)
    assert g["dx"].shape == (0, 4)
    assert not g["dWr"].any() and not g["dw1"].any() and not g["db"].any()

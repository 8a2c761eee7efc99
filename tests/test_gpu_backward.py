"""GPU parity of the backward pass (moe_backward) against the fp64 oracle.

The loss is L = <G, out> + aux_coef * aux with G seeded N(0, 1) in bf16.  The
library's gradients (fp32) are compared with oracle_backward on the same
inputs, element by element at small sizes (several tiles, ragged tails, both
overflow policies, shared experts, experts that receive no token) and on
sampled rows and weight-gradient blocks at full size.

Bar for every gradient: sum|gpu - ref| / sum|ref| <= BWD_REL_L1 and
max|gpu - ref| <= BWD_MAX_FRAC * max|ref|.  The bound comes from the bf16
operands of the backward GEMMs (unit roundoff u = 2^-8): on the path to dW13
and dx, dY = g G is rounded, the forward pre-activations a and b are stored
rounded, and dA, dB are rounded again; dW2 sees dY and the forward's H.  Each
rounding adds an independent relative error of about 1.1e-3 in the L1 sense
and the fp32 sums add nothing comparable, so up to four roundings give
~2.2e-3 and two ~1.6e-3; measured on the small cases: 1.6e-3 to 3.0e-3.
BWD_REL_L1 = 6e-3 is twice the worst of those.  The router gradient dz takes
its error from dg = <G, y> (y carries the forward's ~1.5e-3) and is held to
the same bar.  The bias gradient db_e = sum_t dz_te
is a sum over tokens whose terms largely cancel (sum_e db_e = 0), so its
error, which grows like the root-sum-square of the summands' errors, is
measured against sqrt(sum_t dz_te^2) per expert instead of |db_e|.
"""

import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_22_b200 as M
from layer_check import host_inputs, oracle_route, tile_rows
from sparse_mixture_experts_22_b200 import inputs as I
from sparse_mixture_experts_22_b200.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

BWD_REL_L1 = 6e-3
BWD_MAX_FRAC = 2e-2
AUX_COEF = 0.3

SMALL = {
    # token-major forward; h = 384 takes the 128-wide backward tiles
    "tok_cap": Workload("tok_cap", T=600, d=256, h=384, E=4, k=2, cf=(5, 4), zipf_s=0.7),
    # swapped forward tiles (few tokens per expert), split-K down projection
    "swap": Workload("swap", T=100, d=256, h=512, E=6, k=2),
    # shared experts beside routed top-4 of 16
    "shared": Workload("shared", T=300, d=256, h=256, E=16, k=4, n_shared=2, h_shared=128,
                       cf=(3, 2), zipf_s=0.3),
    # overflow rerouted to a spare expert
    "reroute": Workload("reroute", T=1000, d=256, h=256, E=8, k=2, cf=(1, 1), zipf_s=1.2,
                        overflow="reroute"),
    # top-1 routing, ragged token count
    "top1": Workload("top1", T=257, d=256, h=128, E=8, k=1, cf=(2, 1)),
    # collapsed routing: most experts get no token (their gradients are zero)
    "collapse": Workload("collapse", T=512, d=128, h=128, E=8, k=2, cf=(5, 4), zipf_s=12.0),
    # a single token
    "one_token": Workload("one_token", T=1, d=128, h=256, E=4, k=2),
    # experts that may keep 1024+ rows: the forward's GEMMs and the backward's dX
    # on CTA-pair tiles (a ragged last 256-row tile per expert)
    "pair_tok": Workload("pair_tok", T=1300, d=256, h=384, E=3, k=2, zipf_s=0.3),
    # the same with a hidden width that is a multiple of 256: dgate on CTA-pair
    # tiles as well
    "pair_tok_h512": Workload("pair_tok_h512", T=1300, d=256, h=512, E=3, k=2, zipf_s=0.3),
    # a shared expert over 1100 tokens (its dgate and dX on CTA-pair tiles too)
    "pair_shared": Workload("pair_shared", T=1100, d=256, h=128, E=8, k=2, n_shared=1,
                            h_shared=256, cf=(3, 2)),
}


def rel_l1(g, ref):
    den = np.abs(ref).sum()
    return float(np.abs(g - ref).sum() / den) if den > 0 else float(np.abs(g).sum())


def max_frac(g, ref):
    m = np.abs(ref).max() if ref.size else 0.0
    e = np.abs(g - ref).max() if ref.size else 0.0
    return float(e / m) if m > 0 else float(e)


def check(name, g, ref, report):
    g = np.asarray(g, dtype=np.float64)
    report[name] = (rel_l1(g, ref), max_frac(g, ref))


def check_token_sum(name, g, ref, summands, report):
    """A sum over tokens: error against the root-sum-square of its summands."""
    g = np.asarray(g, dtype=np.float64)
    rss = np.sqrt((summands ** 2).sum(0))
    err = np.abs(g - ref)
    report[name] = (float(err.sum() / rss.sum()), float(err.max() / rss.max()))


def assert_report(case, report):
    print(case, {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in report.items()})
    bad = {k: v for k, v in report.items() if v[0] > BWD_REL_L1 or v[1] > BWD_MAX_FRAC}
    assert not bad, (case, bad)


def unpack13(dW13: torch.Tensor, h: int):
    """[.., 2h, d] gate/up-interleaved rows -> (dw1, dw3) as [.., d, h]."""
    lead = dW13.shape[:-2]
    d = dW13.shape[-1]
    v = dW13.reshape(*lead, h // 128, 2, 128, d)
    g = v[..., 0, :, :].reshape(*lead, h, d).transpose(-1, -2)
    u = v[..., 1, :, :].reshape(*lead, h, d).transpose(-1, -2)
    return g, u


def device_backward(wl: Workload, inp, G, aux_coef):
    cfg = M.config_of(wl, train=True)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
    W13t, W2t = M.pack_weights_backward(cfg, g["w1"], g["w3"], g["w2"])
    W13s = W2s = W13st = W2st = None
    if wl.n_shared:
        W13s, W2s = M.pack_weights(cfg, g["w1s"], g["w3s"], g["w2s"], shared=True)
        W13st, W2st = M.pack_weights_backward(cfg, g["w1s"], g["w3s"], g["w2s"], shared=True)
    bufs = M.forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, W13s, W2s)
    Gd = G.cuda()
    grads = M.backward(cfg, Gd, aux_coef, g["x"], g["Wr"], g["bias"], W13t, W2t, W13st, W2st,
                       bufs)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(bufs["ws"]) == 0
    run = lambda: M.backward(cfg, Gd, aux_coef, g["x"], g["Wr"], g["bias"], W13t, W2t, W13st,
                             W2st, bufs)
    return cfg, grads, bufs, run


def gpu_math_layout(wl, grads):
    """The library's packed-layout gradients in the oracle's layouts (host fp64)."""
    out = {"dx": grads["dx"], "dWr": grads["dWr"], "dz": grads["dlogits"]}
    if wl.has_bias:
        out["db"] = grads["db"]
    dw1, dw3 = unpack13(grads["dW13"], wl.h)
    out.update({"dw1": dw1, "dw3": dw3, "dw2": grads["dW2p"].transpose(1, 2)})
    if wl.n_shared:
        S, hs = wl.n_shared, wl.h_shared
        g1, g3 = unpack13(grads["dW13s"], S * hs)       # [d, S hs]
        out["dw1s"] = g1.reshape(wl.d, S, hs).permute(1, 0, 2)
        out["dw3s"] = g3.reshape(wl.d, S, hs).permute(1, 0, 2)
        out["dw2s"] = grads["dW2s"].reshape(wl.d, S, hs).permute(1, 2, 0)
    return {k: v.double().cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_matches_oracle(name):
    wl = SMALL[name]
    inp = host_inputs(wl)
    G = I.grad_out(wl)
    cfg, grads, bufs, run = device_backward(wl, inp, G, AUX_COEF)
    r = oracle_route(wl, inp)
    ref = O.backward(O.cfg_of(wl), inp, r, G, AUX_COEF)
    got = gpu_math_layout(wl, grads)
    report = {}
    for key in got:
        if key == "db":
            check_token_sum("db", got["db"], ref["db"], ref["dz"], report)
        else:
            check(key, got[key], ref[key], report)
    assert_report(name, report)
    # a second call gives the same bits
    first = {k: v.clone() for k, v in grads.items() if k != "bws"}
    again = run()
    torch.cuda.synchronize()
    for k, v in first.items():
        if k == "db" and not wl.has_bias:
            continue
        assert torch.equal(v, again[k]), f"{k} differs between two calls"


def test_experts_without_tokens_get_zero_gradient():
    wl = SMALL["collapse"]
    inp = host_inputs(wl)
    cfg, grads, bufs, _ = device_backward(wl, inp, I.grad_out(wl), AUX_COEF)
    kept = bufs["kept"].cpu()
    idle = (kept == 0).nonzero().flatten().tolist()
    assert idle, "the collapsed workload should leave experts idle"
    for e in idle:
        assert not grads["dW13"][e].any() and not grads["dW2p"][e].any()


def test_backward_rejects_a_forward_without_train():
    wl = SMALL["swap"]
    cfg = M.config_of(wl)
    with pytest.raises(M.MoEError):
        M.moe_backward_workspace_size(cfg)


# ---------------------------------------------------------------- full size, sampled

FULL_ROWS = 6


@pytest.mark.parametrize("name", ["decode", "prefill", "deepseek", "large"])
def test_backward_full_size_sampled(name):
    """dx and dz on rows that reach every 128-row tile of every expert's queue
    (plus a few random ones), and a block of dw1, dw3, dw2 of every expert
    that kept tokens (and of the shared expert), against the oracle."""
    wl = WORKLOADS[name]
    inp = host_inputs(wl)
    G = I.grad_out(wl)
    cfg, grads, bufs, _ = device_backward(wl, inp, G, AUX_COEF)
    r = oracle_route(wl, inp)
    ocfg = O.cfg_of(wl)
    rng = np.random.default_rng(5)
    rows = tile_rows(r, FULL_ROWS, wl.T, seed=5)
    ref = O.backward_rows(ocfg, inp, r, G, AUX_COEF, rows)
    report = {}
    check("dx rows", grads["dx"][torch.from_numpy(rows).cuda()].double().cpu().numpy(),
          ref["dx"], report)
    check("dz rows", grads["dlogits"][torch.from_numpy(rows).cuda()].double().cpu().numpy(),
          ref["dz"], report)
    # a weight-gradient block of every expert that kept tokens
    kept = r["kept"]
    hi = sorted(rng.choice(wl.h, size=8, replace=False).tolist())
    ci = sorted(rng.choice(wl.d, size=16, replace=False).tolist())
    for e in [int(e) for e in np.nonzero(kept)[0]]:
        b = O.wgrad_block(ocfg, inp, r, G, e, hi, ci)
        W13 = grads["dW13"][e]
        rows1 = [256 * (i // 128) + i % 128 for i in hi]
        g1 = W13[rows1][:, ci].double().cpu().numpy()
        g3 = W13[[x + 128 for x in rows1]][:, ci].double().cpu().numpy()
        g2 = grads["dW2p"][e][ci][:, hi].T.double().cpu().numpy()
        check(f"dw1[{e}]", g1, b["dw1"], report)
        check(f"dw3[{e}]", g3, b["dw3"], report)
        check(f"dw2[{e}]", g2, b["dw2"], report)
    if wl.n_shared:
        hs = wl.h_shared
        b = O.wgrad_block(ocfg, inp, r, G, 0, hi, ci, shared=True)
        hi_s = list(hi)
        rows1 = [256 * (i // 128) + i % 128 for i in hi_s]
        g1 = grads["dW13s"][rows1][:, ci].double().cpu().numpy()
        g2 = grads["dW2s"][ci][:, hi_s].T.double().cpu().numpy()
        check("dw1s[0]", g1, b["dw1"], report)
        check("dw2s[0]", g2, b["dw2"], report)
    assert_report(name, report)
    # properties that hold at any size: both router terms sum to zero over experts
    dz = grads["dlogits"].double()
    scale = dz.abs().max().item()
    assert dz.sum(1).abs().max().item() <= 1e-4 * scale
    dWr = grads["dWr"].double()
    assert dWr.sum(1).abs().max().item() <= 1e-3 * dWr.abs().max().item()
    if wl.has_bias:
        db = grads["db"].double()
        assert abs(db.sum().item()) <= 1e-3 * db.abs().max().item()

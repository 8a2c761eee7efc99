"""Shared helpers of the GPU parity tests: run the layer through the C ABI and
compare every output with the fp64 oracle on the same seeded inputs.

Bars (the layer's stated tolerances):
  routing sets, counts, ranks, permutation, dropped set   bit-exact
  logits, gates                                          |err| <= 2.5e-5
  output    max|err| <= 1e-2 * max|ref|  and  sum|err| / sum|ref| <= 2e-3
            against the fp64 reference itself when H reaches the down
            projection as two bf16 parts (and for fp32 layers); with bf16 H
            alone the relative L1 bar holds against the reference rounded to
            the output dtype, and the unrounded figure is reported beside it
  aux loss  relative error <= 1e-5; overflow rate exact; entropy rel <= 1e-5
Why: storing the output in bf16 (unit roundoff 2^-8) alone leaves ~1.41e-3
relative L1 against the unrounded value; rounding H to bf16 adds ~0.8e-3 more
(2.2-2.3e-3 in all), while the two-part H (16 significant bits) adds ~1e-6.
The gate/up and down sums accumulate in fp32.
"""

import math
from typing import Dict, Optional

import numpy as np
import torch

import oracle as O
import sparse_mixture_experts_22_b200 as M
from sparse_mixture_experts_22_b200 import inputs as I
from sparse_mixture_experts_22_b200.workloads import Workload

MAX_ERR_FRAC = 1e-2
REL_L1 = 2e-3
AUX_REL = 1e-5
# The generator keeps the k-th and (k+1)-th fp64 logits of every token at
# least 1e-4 apart, so the expert set is unambiguous while every logit is off
# by less than 5e-5; the bar keeps a further factor of 2.  A gate moves by at
# most half the error of a logit difference, so the same bound covers gates.
LOGIT_ABS = 2.5e-5
GATE_ABS = 2.5e-5

_weight_cache: Dict = {}


def host_inputs(wl: Workload) -> Dict:
    """Seeded host inputs; expert weights cached across workloads of equal shape."""
    inp = I.layer_inputs(wl, weights=False)
    key = (wl.d, wl.h, wl.E, wl.n_shared, wl.h_shared, wl.dtype, wl.seed)
    if key not in _weight_cache:
        _weight_cache.clear()
        w = I.expert_weights(wl)
        if wl.n_shared:
            s = I.expert_weights(wl, shared=True)
            w.update({"w1s": s["w1"], "w3s": s["w3"], "w2s": s["w2"]})
        _weight_cache[key] = w
    inp.update(_weight_cache[key])
    return inp


def device_layer(wl: Workload, inp: Dict, dev="cuda", hidden: str = "auto"):
    cfg = M.config_of(wl, hidden=hidden)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
    W13s = W2s = None
    if wl.n_shared:
        W13s, W2s = M.pack_weights(cfg, g["w1s"], g["w3s"], g["w2s"], shared=True)
    return cfg, g, (W13, W2p, W13s, W2s)


def run_forward(cfg, g, W, bufs=None):
    W13, W2p, W13s, W2s = W
    bufs = M.forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, W13s, W2s, bufs=bufs)
    torch.cuda.synchronize()
    return bufs


def run_steps(cfg, g, W):
    """The same layer through the five step entry points."""
    W13, W2p, W13s, W2s = W
    dev = g["x"].device
    T, E, k, d = cfg.T, cfg.E, cfg.k, cfg.d
    rows = M.moe_perm_rows(cfg)
    splits = M.moe_ffn_splits(cfg)
    ws = torch.empty(max(M.moe_workspace_size(cfg), 256), dtype=torch.uint8, device=dev)
    b = {
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
        "topk_gate": torch.empty((T, k), dtype=torch.float32, device=dev),
        "routed": torch.empty(E, dtype=torch.int32, device=dev),
        "kept": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm_token": torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
        "slot_of": torch.empty((T, k), dtype=torch.int32, device=dev),
        "x_perm": torch.empty((max(rows, 1), d), dtype=g["x"].dtype, device=dev),
        "y_perm": torch.empty((splits, max(rows, 1), d), dtype=torch.float32, device=dev),
        "y_shared": torch.empty((T, d), dtype=torch.float32, device=dev) if cfg.n_shared else None,
        "out": torch.empty((T, d), dtype=g["x"].dtype, device=dev),
        "stats": torch.zeros(5, dtype=torch.float64, device=dev),
        "sums": torch.zeros(2 + 3 * E, dtype=torch.float64, device=dev),
        "stats2": torch.zeros(5, dtype=torch.float64, device=dev),
        "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
    }
    M.moe_route(cfg, g["x"], g["Wr"], g["bias"] if cfg.has_bias else None, b["topk_idx"],
                b["topk_gate"], ws, logits=b["logits"])
    M.moe_dispatch(cfg, b["topk_idx"], g["x"], b["routed"], b["kept"], b["offsets"],
                   b["perm_token"], b["slot_of"], b["x_perm"], ws)
    M.moe_expert_ffn(cfg, b["x_perm"], b["offsets"], b["kept"], W13, W2p, g["x"], W13s, W2s,
                     b["y_perm"], b["y_shared"], ws)
    M.moe_combine(cfg, b["y_perm"], b["slot_of"], b["topk_gate"], b["y_shared"], b["out"])
    M.moe_aux_stats(cfg, b["routed"], b["kept"], ws, b["stats"])
    M.moe_stats_sums(cfg, b["routed"], b["kept"], ws, b["sums"])
    M.moe_stats_finalize(cfg, b["sums"], b["stats2"])
    torch.cuda.synchronize()
    b["status"] = M.moe_read_device_status(ws)
    return b


def oracle_route(wl: Workload, inp: Dict) -> Dict:
    cfg = O.cfg_of(wl)
    return O.route(cfg, inp["x"], inp["Wr"], inp["bias"])


def oracle_rows(wl: Workload, inp: Dict, r: Dict, rows=None) -> np.ndarray:
    cfg = O.cfg_of(wl)
    return O.layer_rows(cfg, inp["x"], r["expert"], r["gate"], r["keep"], inp["w1"], inp["w3"],
                        inp["w2"], inp.get("w1s"), inp.get("w3s"), inp.get("w2s"), rows)


def check_routing(wl: Workload, r: Dict, b: Dict):
    T, k = wl.T, wl.k
    idx = b["topk_idx"].cpu().numpy()
    gate = b["topk_gate"].cpu().numpy()
    # kept-expert sets, bit-exact
    assert np.array_equal(np.sort(idx, axis=1), np.sort(r["idx"], axis=1)), "top-k sets differ"
    # gates per (t, e)
    order_g = np.argsort(idx, axis=1)
    order_o = np.argsort(r["idx"], axis=1)
    g_gpu = np.take_along_axis(gate, order_g, 1)
    g_ref = np.take_along_axis(r["gate"], order_o, 1)
    assert np.max(np.abs(g_gpu - g_ref)) <= GATE_ABS, np.max(np.abs(g_gpu - g_ref))
    # per-expert counts, bit-exact
    assert b["routed"].cpu().tolist() == r["routed"].tolist()
    assert b["kept"].cpu().tolist() == r["kept"].tolist()


def route_logits(cfg, g):
    """Router logits from moe_route (its optional output)."""
    T, E, k = cfg.T, cfg.E, cfg.k
    dev = g["x"].device
    ws = torch.empty(max(M.moe_workspace_size(cfg), 256), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    M.moe_route(cfg, g["x"], g["Wr"], g["bias"] if cfg.has_bias else None, idx, gate, ws,
                logits=logits)
    torch.cuda.synchronize()
    return logits


def check_logits(r: Dict, logits: torch.Tensor):
    z = logits.double().cpu().numpy()
    err = np.abs(z - r["z"]).max() if z.size else 0.0
    assert err <= LOGIT_ABS, f"router logits off by {err}"
    return float(err)


def check_slots(wl: Workload, r: Dict, b: Dict, offsets: np.ndarray,
                perm_token: Optional[np.ndarray] = None):
    """Dropped set, serving expert and rank of every assignment, bit-exact,
    matched per (token, expert the router chose)."""
    T, k = wl.T, wl.k
    idx = b["topk_idx"].cpu().numpy()
    slot = b["slot_of"].cpu().numpy()
    ref = {}
    for t in range(T):
        for j in range(k):
            ref[(t, int(r["idx"][t, j]))] = (int(r["keep"][t, j]), int(r["expert"][t, j]),
                                             int(r["rank"][t, j]))
    for t in range(T):
        for j in range(k):
            keep, ex, rank = ref[(t, int(idx[t, j]))]
            s = int(slot[t, j])
            if not keep:
                assert s == -1, (t, j, s)
            else:
                assert s == offsets[ex] + rank, (t, j, s, ex, offsets[ex], rank)
                if perm_token is not None:
                    assert perm_token[s] == t


def check_offsets(wl: Workload, r: Dict, offsets: np.ndarray, pad: int):
    o = 0
    for e in range(wl.E):
        assert offsets[e] == o
        o += (int(r["kept"][e]) + pad - 1) // pad * pad
    assert offsets[wl.E] == o


def strict_output(cfg) -> bool:
    """Whether the output bar holds against the unrounded fp64 reference:
    fp32 layers, and bf16 layers whose H reaches the down projection in two
    parts."""
    return cfg.act_dtype == M.MOE_F32 or M.moe_hidden_split(cfg)


def check_output(out_gpu: torch.Tensor, ref: np.ndarray, what: str = "out",
                 strict: bool = True):
    """max|err| against the fp64 reference.  Mean relative error (relative L1)
    against the unrounded fp64 reference when `strict`; always also against
    the correctly rounded result (the fp64 reference stored in the output
    dtype, round-to-nearest-even), which is the bar for bf16 H."""
    g = out_gpu.double().cpu().numpy()
    ref_q = torch.from_numpy(ref).to(out_gpu.dtype).double().numpy()
    err = np.abs(g - ref)
    scale = np.max(np.abs(ref))
    rel_l1 = np.abs(g - ref_q).sum() / max(np.abs(ref_q).sum(), 1e-300)
    rel_l1_raw = err.sum() / max(np.abs(ref).sum(), 1e-300)
    floor = np.abs(ref_q - ref).sum() / max(np.abs(ref).sum(), 1e-300)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    assert err.max() <= MAX_ERR_FRAC * scale, f"{what}: max|err| {err.max()} > 1e-2 * {scale}"
    if strict:
        assert rel_l1_raw <= REL_L1, (f"{what}: relative L1 {rel_l1_raw} against the unrounded "
                                      f"reference (storage floor {floor})")
    assert rel_l1 <= REL_L1, (f"{what}: relative L1 {rel_l1} against the rounded reference "
                              f"(vs unrounded {rel_l1_raw}, storage floor {floor})")
    return {"max_err_frac": float(err.max() / scale) if scale > 0 else 0.0,
            "rel_l1": float(rel_l1), "rel_l1_unrounded": float(rel_l1_raw),
            "storage_floor": float(floor), "strict": bool(strict)}


def check_stats(r: Dict, stats: torch.Tensor, T: int):
    s = M.stats_dict(stats)
    ref = r["stats"]
    assert s["tokens"] == T
    if T == 0:
        assert s["aux_loss"] == 0.0 and s["overflow_rate"] == 0.0
        return s
    assert abs(s["aux_loss"] - ref["aux_loss"]) <= AUX_REL * abs(ref["aux_loss"]), \
        (s["aux_loss"], ref["aux_loss"])
    assert s["overflow_rate"] == ref["overflow_rate"], (s["overflow_rate"], ref["overflow_rate"])
    assert abs(s["mean_entropy"] - ref["mean_entropy"]) <= 1e-5 * abs(ref["mean_entropy"]) + 1e-7
    return s


def sample_rows(T: int, n: int, seed: int = 0) -> np.ndarray:
    """n token rows spread over the batch: first, last and random ones."""
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    rest = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, T - 1], rest]))


def tile_rows(r: Dict, n_extra: int, T: int, seed: int = 0, tile: int = 128) -> np.ndarray:
    """Token rows that reach every tile of every expert: for each expert with
    kept rows, a token in each `tile`-row block of its queue (the blocks the
    GEMMs cut it into), the tokens at the head and at the tail of its queue
    (the ragged last tile), plus n_extra rows spread over the batch.  Built
    from the oracle's dispatch (serving expert and queue position of every
    kept assignment), which the GPU matches bit for bit."""
    keep, expert, rank = r["keep"], r["expert"], r["rank"]
    first: Dict = {}
    last: Dict = {}
    for t, j in zip(*np.nonzero(keep)):
        e, q = int(expert[t, j]), int(rank[t, j])
        key = (e, q // tile)
        if key not in first or q < first[key][0]:
            first[key] = (q, int(t))
        if e not in last or q > last[e][0]:
            last[e] = (q, int(t))
    rows = {t for _, t in first.values()} | {t for _, t in last.values()}
    rows |= set(sample_rows(T, n_extra, seed).tolist())
    return np.array(sorted(rows), dtype=np.int64)

"""GPU parity: the CUDA layer (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Small cases run the oracle on every token; they span several tensor-core
tiles and a ragged tail and reach both GEMM layouts (token-major when an
expert may hold more than 256 tokens, swapped otherwise), capacity drops,
shared experts, the fp32 path and the degenerate cases.  The full-size
workloads compare everything exactly except the expert outputs, which the
oracle computes for a sample of rows.
"""

import os

import numpy as np
import pytest
import torch

from layer_check import (check_logits, check_offsets, check_output, check_routing, check_slots,
                         check_stats, device_layer, host_inputs, oracle_route, oracle_rows,
                         route_logits, run_forward, run_steps, strict_output, tile_rows)
from sparse_mixture_experts_22_b200 import binding as B
from sparse_mixture_experts_22_b200.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

SMALL = {
    # token-major tiles (C = 375 > 256), 3 m-tiles with a ragged tail, drops
    "tok_cap": Workload("tok_cap", T=600, d=256, h=384, E=4, k=2, cf=(5, 4), zipf_s=0.7),
    # token-major without capacity, several experts of > 128 rows
    "tok_nocap": Workload("tok_nocap", T=700, d=384, h=256, E=3, k=2),
    # swapped tiles (no limit, T = 100 <= 256), split-K down projection
    "swap": Workload("swap", T=100, d=256, h=512, E=6, k=2),
    # swapped with drops (C = 250)
    "swap_cap": Workload("swap_cap", T=1000, d=256, h=256, E=8, k=2, cf=(1, 1), zipf_s=1.2),
    # shared + routed, top-4 of 16, cf 1.5 (C = 113), token-major shared expert (T > 256)
    "shared": Workload("shared", T=300, d=256, h=256, E=16, k=4, n_shared=2, h_shared=128,
                       cf=(3, 2)),
    # shared experts with a swapped shared GEMM (T <= 256)
    "shared_small": Workload("shared_small", T=40, d=128, h=128, E=5, k=2, n_shared=1,
                             h_shared=256),
    # fp32 throughout (the tiny workload)
    "tiny": WORKLOADS["tiny"],
    # fp32 with drops and shared experts
    "f32_shared": Workload("f32_shared", T=90, d=128, h=128, E=4, k=2, n_shared=2, h_shared=128,
                           cf=(1, 2), dtype="f32", zipf_s=1.0),
    # degenerate: one token; one expert; k = E; heavy skew
    "one_token": Workload("one_token", T=1, d=128, h=128, E=8, k=2),
    # shared expert on 200 tokens: one swapped gate/up tile of 208 token columns
    "shared_swap64": Workload("shared_swap64", T=200, d=256, h=256, E=8, k=2, n_shared=1,
                              h_shared=256, cf=(1, 1)),
    "one_expert": Workload("one_expert", T=130, d=128, h=256, E=1, k=1),
    "k_equals_E": Workload("k_equals_E", T=64, d=128, h=128, E=4, k=4),
    "top1": Workload("top1", T=257, d=256, h=128, E=8, k=1, cf=(2, 1)),
    "collapse": Workload("collapse", T=512, d=128, h=128, E=8, k=2, cf=(5, 4), zipf_s=12.0),
    # overflow rerouted to a spare expert: swapped and token-major tiles, top-1, many experts
    "reroute_swap": Workload("reroute_swap", T=1000, d=256, h=256, E=8, k=2, cf=(1, 1),
                             zipf_s=1.2, overflow="reroute"),
    "reroute_tok": Workload("reroute_tok", T=600, d=256, h=384, E=4, k=2, cf=(5, 4), zipf_s=0.7,
                            overflow="reroute"),
    "reroute_top1": Workload("reroute_top1", T=300, d=128, h=128, E=8, k=1, cf=(1, 1),
                             zipf_s=2.0, overflow="reroute"),
    "reroute_wide": Workload("reroute_wide", T=300, d=256, h=128, E=40, k=4, cf=(1, 2),
                             zipf_s=0.5, overflow="reroute"),
    "reroute_f32": Workload("reroute_f32", T=90, d=128, h=128, E=4, k=2, cf=(1, 2), dtype="f32",
                            zipf_s=1.0, overflow="reroute"),
    # one warp per token above 32 experts, four top-k CTAs per 128-token block:
    # the last block holds 44 tokens (CTAs of 32, 12, 0 and 0 tokens)
    "wide_sub": Workload("wide_sub", T=300, d=128, h=128, E=64, k=3, cf=(5, 4), zipf_s=0.5),
    "wide_sub_reroute": Workload("wide_sub_reroute", T=300, d=128, h=128, E=64, k=3, cf=(1, 1),
                                 zipf_s=1.5, overflow="reroute"),
    # logits past 256 experts live in global scratch; k at its limit of 8
    "wide_zbuf": Workload("wide_zbuf", T=400, d=128, h=128, E=512, k=8, cf=(1, 1)),
    # the largest expert count, one routing block (fused top-k and dispatch)
    "max_experts": Workload("max_experts", T=64, d=128, h=128, E=1024, k=8),
    # experts of up to 219 tokens (C): swapped tiles on CTA pairs for both GEMMs,
    # groups of 16..219 rows, three 128-feature gate/up units and two 256-wide
    # down units per expert
    "pair_tiles": Workload("pair_tiles", T=700, d=512, h=384, E=8, k=2, cf=(5, 4),
                           zipf_s=0.8),
    # pair tiles with shared experts (a dense group of 200 tokens) and drops
    "pair_shared": Workload("pair_shared", T=200, d=256, h=256, E=4, k=2, n_shared=2,
                            h_shared=128, cf=(1, 1), zipf_s=0.5),
    # experts of over 1024 tokens: token-major tiles of 256 tokens on CTA pairs,
    # ragged last tiles (an expert's second CTA half partly or wholly past its rows)
    "pair_tok": Workload("pair_tok", T=1300, d=256, h=384, E=3, k=2, zipf_s=0.3),
    # a model width that is not a multiple of 256: the down projection on
    # 128-wide output tiles (three of them), swapped and token-major
    "d384_swap": Workload("d384_swap", T=300, d=384, h=256, E=6, k=2, cf=(5, 4), zipf_s=0.5),
    "d384_tok": Workload("d384_tok", T=1000, d=384, h=256, E=4, k=2, cf=(1, 1), zipf_s=0.5),
    # swapped gate/up tiles of up to 256 token columns (C = 250) with a model
    # width of 384: the token rows arrive in boxes of 64, and a group's last box
    # runs into the next group's rows (or past the tensor's end)
    "d384_swap_wide": Workload("d384_swap_wide", T=600, d=384, h=256, E=6, k=2, cf=(5, 4),
                               zipf_s=0.5),
}


def _pad(cfg):
    return 128 if B.moe_perm_rows(cfg) and _path(cfg) == "tok" else 16


def _path(cfg):
    C = B.moe_capacity(cfg)
    nmax = min(C, cfg.T)
    if cfg.act_dtype == B.MOE_F32:
        return "f32"
    return "swap" if nmax <= 256 else "tok"


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_matches_oracle(name):
    wl = SMALL[name]
    inp = host_inputs(wl)
    r = oracle_route(wl, inp)
    ref = oracle_rows(wl, inp, r)
    cfg, g, W = device_layer(wl, inp)
    b = run_forward(cfg, g, W)
    check_routing(wl, r, b)
    s = run_steps(cfg, g, W)
    assert s["status"] == 0
    zerr = check_logits(r, s["logits"])
    offsets = s["offsets"].cpu().numpy()
    check_offsets(wl, r, offsets, _pad(cfg))
    check_slots(wl, r, s, offsets, s["perm_token"].cpu().numpy())
    check_slots(wl, r, b, offsets)
    e = check_output(b["out"], ref, strict=strict_output(cfg))
    print(f"{name}: {e} logit_err={zerr:.2e}")
    check_stats(r, b["stats"], wl.T)
    check_stats(r, s["stats"], wl.T)
    check_stats(r, s["stats2"], wl.T)
    # the step entry points run the same kernels as moe_forward
    assert torch.equal(s["out"], b["out"])
    assert torch.equal(s["slot_of"], b["slot_of"])


BF16_SMALL = [n for n, w in SMALL.items() if w.dtype == "bf16"]


@pytest.mark.parametrize("name", BF16_SMALL)
def test_small_layer_other_hidden_mode(name):
    """Each bf16 case with H fed to the down projection the other way: two
    bf16 parts where the default rounds it to bf16 (the output then meets the
    relative-L1 bar against the unrounded fp64 reference), bf16 alone where the
    default splits it.  Routing is the same in both."""
    wl = SMALL[name]
    inp = host_inputs(wl)
    r = oracle_route(wl, inp)
    ref = oracle_rows(wl, inp, r)
    auto_split = B.moe_hidden_split(B.config_of(wl))
    cfg, g, W = device_layer(wl, inp, hidden="bf16" if auto_split else "split")
    assert B.moe_hidden_split(cfg) != auto_split
    b = run_steps(cfg, g, W)
    assert b["status"] == 0
    check_routing(wl, r, b)
    offsets = b["offsets"].cpu().numpy()
    check_offsets(wl, r, offsets, _pad(cfg))
    check_slots(wl, r, b, offsets)
    e = check_output(b["out"], ref, strict=strict_output(cfg))
    print(f"{name} ({'split' if not auto_split else 'bf16'} H): {e}")
    check_stats(r, b["stats"], wl.T)


def test_empty_batch():
    wl = Workload("empty", T=0, d=128, h=128, E=4, k=2, cf=(5, 4))
    cfg = B.config_of(wl)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((128, 4), dtype=torch.float32, device="cuda")
    w1 = torch.zeros((4, 128, 128), dtype=torch.bfloat16, device="cuda")
    W13, W2p = B.pack_weights(cfg, w1, w1, w1)
    bufs = B.alloc_layer(cfg)
    bufs["routed"].fill_(7)
    B.forward(cfg, x, Wr, None, W13, W2p, bufs=bufs)
    torch.cuda.synchronize()
    assert bufs["routed"].tolist() == [0, 0, 0, 0]
    st = B.stats_dict(bufs["stats"])
    assert st["tokens"] == 0 and st["aux_loss"] == 0.0
    assert B.moe_read_device_status(bufs["ws"]) == 0


def test_repeatable_bitwise():
    wl = SMALL["swap_cap"]
    inp = host_inputs(wl)
    cfg, g, W = device_layer(wl, inp)
    a = run_forward(cfg, g, W)
    out1 = a["out"].clone()
    slot1 = a["slot_of"].clone()
    stats1 = a["stats"].clone()
    for _ in range(3):
        run_forward(cfg, g, W, bufs=a)
        assert torch.equal(a["out"], out1)
        assert torch.equal(a["slot_of"], slot1)
        assert torch.equal(a["stats"], stats1)


def test_bad_workspace_is_rejected():
    wl = SMALL["swap"]
    cfg = B.config_of(wl)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    x = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((wl.d, wl.E), dtype=torch.float32, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoEError) as e:
        B.moe_route(cfg, x, Wr, None, idx, gate, small)
    assert e.value.code == 5


# ---------------------------------------------------------------- full-size workloads

FULL = dict(WORKLOADS)
FULL["prefill_reroute"] = WORKLOADS["prefill"].scaled(name="prefill_reroute", overflow="reroute")
# random rows added to those that reach every 128-row tile of every expert
FULL_EXTRA = {"decode": 32, "prefill": 16, "deepseek": 8, "large": 16, "prefill_reroute": 16}
FULL_CASES = [("decode", "auto"), ("decode", "bf16"), ("prefill", "auto"), ("prefill", "split"),
              ("deepseek", "auto"), ("deepseek", "split"), ("large", "auto"), ("large", "split"),
              ("prefill_reroute", "auto"), ("prefill_reroute", "split")]
_full_ref: dict = {}


@pytest.mark.parametrize("name,hidden", FULL_CASES)
def test_full_size_workload(name, hidden):
    """A full-size workload: routing, ranks, dropped set and statistics
    compared in full; the layer output on rows that reach every 128-row tile
    of every expert's queue (its first and last rows included) plus random
    ones, computed one by one by the oracle."""
    wl = FULL[name]
    inp = host_inputs(wl)
    if name not in _full_ref:
        _full_ref.clear()
        r = oracle_route(wl, inp)
        rows = tile_rows(r, FULL_EXTRA[name], wl.T, seed=1)
        _full_ref[name] = (r, rows, oracle_rows(wl, inp, r, rows))
    r, rows, ref = _full_ref[name]
    cfg, g, W = device_layer(wl, inp, hidden=hidden)
    b = run_forward(cfg, g, W)
    assert B.moe_read_device_status(b["ws"]) == 0
    check_routing(wl, r, b)
    check_stats(r, b["stats"], wl.T)
    zerr = check_logits(r, route_logits(cfg, g))
    # dropped set and ranks for every assignment (offsets rebuilt from the oracle's kept counts)
    pad = _pad(cfg)
    offsets = np.zeros(wl.E + 1, dtype=np.int64)  # from the oracle's final kept counts
    for e in range(wl.E):
        offsets[e + 1] = offsets[e] + (int(r["kept"][e]) + pad - 1) // pad * pad
    check_slots(wl, r, b, offsets)
    e = check_output(b["out"][torch.as_tensor(rows, device="cuda")], ref,
                     f"{name} sampled rows", strict=strict_output(cfg))
    print(f"{name} ({hidden} H, {len(rows)} rows): {e} logit_err={zerr:.2e}")


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("name", ["pair_tiles", "pair_shared", "swap_cap", "pair_tok"])
def test_pair_tiles_match_single_sm_tiles(name, mode):
    """Experts of more than 128 tokens run their GEMMs on CTA pairs (mode 1:
    token-major pair tiles; mode 2: the swapped pair tiles too); the same layer
    with one SM per tile gives the same routing and the same output bit for bit
    (the fp32 sums run in the same order), within the bar of the oracle."""
    wl = SMALL[name]
    inp = host_inputs(wl)
    r = oracle_route(wl, inp)
    ref = oracle_rows(wl, inp, r)
    cfg, g, W = device_layer(wl, inp)
    try:
        B.moe_set_pair_tiles(mode)
        a = run_forward(cfg, g, W)
        out_pair = a["out"].clone()
        B.moe_set_pair_tiles(0)
        b = run_forward(cfg, g, W)
    finally:
        B.moe_set_pair_tiles(1)
    assert B.moe_read_device_status(b["ws"]) == 0
    assert torch.equal(a["slot_of"], b["slot_of"])
    e1 = check_output(out_pair, ref, strict=strict_output(cfg))
    e2 = check_output(b["out"], ref, strict=strict_output(cfg))
    d = (out_pair.float() - b["out"].float()).abs().max().item()
    print(f"{name} mode {mode}: pair {e1} single {e2} max|pair - single| {d:.3e}")
    assert torch.equal(out_pair, b["out"])


@pytest.mark.parametrize("name", ["shared", "shared_small", "pair_shared", "shared_swap64"])
def test_shared_overlap_gives_identical_bits(name):
    """Shared experts on a second stream beside the routed ones, or after them
    on one stream: the same bits; and the overlapped run matches the oracle."""
    wl = SMALL[name]
    inp = host_inputs(wl)
    cfg, g, W = device_layer(wl, inp)
    B.moe_set_shared_overlap(True)
    a = run_forward(cfg, g, W)
    out_on = a["out"].clone()
    try:
        B.moe_set_shared_overlap(False)
        b = run_forward(cfg, g, W)
    finally:
        B.moe_set_shared_overlap(True)
    assert torch.equal(out_on, b["out"])
    assert B.moe_read_device_status(b["ws"]) == 0
    # SMs set aside for the shared experts: the grids change, the bits do not
    try:
        B.moe_set_shared_sms(24)
        c = run_forward(cfg, g, W)
    finally:
        B.moe_set_shared_sms(0)
    assert torch.equal(out_on, c["out"])
    assert B.moe_read_device_status(c["ws"]) == 0
    r = oracle_route(wl, inp)
    check_output(out_on, oracle_rows(wl, inp, r), strict=strict_output(cfg))


@pytest.mark.parametrize("name", ["swap", "tok_cap", "shared"])
def test_dependent_launch_gives_identical_bits(name):
    """The forward chain launched with and without programmatic dependent
    launch (and the gate/up weight prefetch it enables) gives the same bits."""
    wl = SMALL[name]
    inp = host_inputs(wl)
    cfg, g, W = device_layer(wl, inp)
    B.moe_set_pdl(True)
    a = run_forward(cfg, g, W)
    out_on = a["out"].clone()
    try:
        B.moe_set_pdl(False)
        b = run_forward(cfg, g, W)
    finally:
        B.moe_set_pdl(True)
    assert torch.equal(out_on, b["out"])
    assert B.moe_read_device_status(b["ws"]) == 0


@pytest.mark.parametrize("name", ["wide_sub", "wide_zbuf", "max_experts"])
def test_first_call_in_a_fresh_process(name):
    """A layer whose routing kernels need a shared-memory opt-in (their static
    arrays plus the dynamic buffer exceed 48 KB) works as the first call of a
    process, whatever ran before it elsewhere."""
    import subprocess
    import sys
    HERE = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import torch\n"
        "from test_gpu_parity import SMALL\n"
        "from layer_check import device_layer, host_inputs, run_forward\n"
        "import sparse_mixture_experts_22_b200 as M\n"
        "wl = SMALL[%r]\n"
        "cfg, g, W = device_layer(wl, host_inputs(wl))\n"
        "b = run_forward(cfg, g, W)\n"
        "assert M.moe_read_device_status(b['ws']) == 0\n"
        "assert torch.isfinite(b['out'].float()).all()\n"
    ) % (HERE, os.path.dirname(HERE), name)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]

"""Expert parallelism on the GPU: G ranks emulated by one process on one
device (the same phases rank by rank, the exchanges as copies -- no kernel
ever waits on another), against the fp64 oracle on the concatenated batch.

The G ranks must reproduce the single-GPU layer on the concatenation of their
batches: the routing sets, the rows every expert keeps under the global
capacity (bit-exact), the output (the layer's bars) and the statistics.  The
peer-memory form (rows stored into, and read from, the owners' buffers by the
dispatch and combine kernels) must give the exchange form's output bit for
bit."""

import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_22_b200 as M
from layer_check import check_output, check_stats, host_inputs, strict_output
from sparse_mixture_experts_22_b200 import ep
from sparse_mixture_experts_22_b200.workloads import Workload

pytestmark = pytest.mark.gpu

CASES = {
    # 200 tokens per rank: swapped tiles; capacity binds on the skewed experts
    "g2_swap": (Workload("ep_swap", T=400, d=256, h=256, E=8, k=2, cf=(5, 4), zipf_s=0.8), 2),
    # 600 tokens per rank, groups up to 300 rows: token-major tiles, h = 384
    "g2_tok": (Workload("ep_tok", T=1200, d=256, h=384, E=8, k=2, cf=(1, 1), zipf_s=1.0), 2),
    # four ranks of 4 experts each, top-4
    "g4": (Workload("ep_g4", T=512, d=128, h=256, E=16, k=4, cf=(3, 2), zipf_s=0.5), 4),
    # no capacity limit
    "g2_nocap": (Workload("ep_nocap", T=300, d=128, h=128, E=4, k=2), 2),
    # one rank: the plain layer through the expert-parallel calls
    "g1": (Workload("ep_g1", T=256, d=128, h=256, E=8, k=2, cf=(5, 4)), 1),
    # eight ranks of two experts each, a skewed router: some owners receive
    # nothing from some sources
    "g8": (Workload("ep_g8", T=512, d=128, h=128, E=16, k=2, cf=(5, 4), zipf_s=1.5), 8),
    # top-8 of 16 over two ranks, no limit
    "g2_k8": (Workload("ep_k8", T=192, d=128, h=128, E=16, k=8), 2),
}


def run_emulated(wl, G, inp):
    dev = torch.device("cuda")
    cfg = M.config_of(wl)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
    T_loc, E_loc = wl.T // G, wl.E // G
    ranks = [ep.Rank(wl, r, G, g["x"][r * T_loc:(r + 1) * T_loc].contiguous(), g["Wr"],
                     g["bias"], W13[r * E_loc:(r + 1) * E_loc], W2p[r * E_loc:(r + 1) * E_loc])
             for r in range(G)]
    outs, stats, plan = ep.forward_emulated(ranks, wl.T)
    torch.cuda.synchronize()
    return ranks, torch.cat(outs), stats, plan


@pytest.mark.parametrize("name", list(CASES))
def test_emulated_ranks_match_the_layer_on_the_concatenated_batch(name):
    wl, G = CASES[name]
    inp = host_inputs(wl)
    ranks, out, stats, plan = run_emulated(wl, G, inp)
    for r in ranks:
        assert M.moe_read_device_status(r.b["ws"]) == 0
        if hasattr(r, "ffn_ws"):
            assert M.moe_read_device_status(r.ffn_ws) == 0
    ref = O.forward(O.cfg_of(wl), inp)
    T_loc = wl.T // G
    # routing sets, bit-exact
    idx = torch.cat([r.b["topk_idx"] for r in ranks]).cpu().numpy()
    assert np.array_equal(np.sort(idx, 1), np.sort(ref["idx"], 1))
    # rows kept per (rank, expert): the plan, the device and the oracle agree
    for r in ranks:
        np.testing.assert_array_equal(r.b["kept"].cpu().numpy(), plan.kept[r.rank])
        kr = ref["keep"][r.rank * T_loc:(r.rank + 1) * T_loc]
        ir = ref["idx"][r.rank * T_loc:(r.rank + 1) * T_loc]
        for e in range(wl.E):
            assert plan.kept[r.rank, e] == int(kr[ir == e].sum())
    np.testing.assert_array_equal(plan.kept.sum(0), ref["kept"])
    if wl.cf is not None and name != "g1":
        assert ref["kept"].sum() < wl.T * wl.k, "the case should drop some assignments"
    check_output(out, ref["out"], name, strict=strict_output(ranks[0].cfg))
    check_stats(ref, stats, wl.T)


def run_emulated_peers(wl, G, inp, bound=None):
    dev = torch.device("cuda")
    cfg = M.config_of(wl)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
    T_loc, E_loc = wl.T // G, wl.E // G
    ranks = [ep.Rank(wl, r, G, g["x"][r * T_loc:(r + 1) * T_loc].contiguous(), g["Wr"],
                     g["bias"], W13[r * E_loc:(r + 1) * E_loc], W2p[r * E_loc:(r + 1) * E_loc])
             for r in range(G)]
    outs, stats, plan = ep.forward_emulated_peers(ranks, wl.T, bound=bound)
    torch.cuda.synchronize()
    return ranks, torch.cat([o.clone() for o in outs]), stats, plan


@pytest.mark.parametrize("name", list(CASES))
def test_peer_stores_and_loads_give_the_exchange_path_bit_for_bit(name):
    """The dispatch that stores rows into the owners' buffers and the combine
    that loads them from there reproduce the all-to-all path exactly, and so
    the oracle."""
    wl, G = CASES[name]
    inp = host_inputs(wl)
    _, out_x, stats_x, plan_x = run_emulated(wl, G, inp)
    ranks, out_p, stats_p, plan_p = run_emulated_peers(wl, G, inp)
    for r in ranks:
        assert M.moe_read_device_status(r.b["ws"]) == 0
    np.testing.assert_array_equal(plan_p.kept, plan_x.kept)
    assert torch.equal(out_p, out_x)
    assert torch.equal(stats_p, stats_x)
    ref = O.forward(O.cfg_of(wl), inp)
    check_output(out_p, ref["out"], name, strict=strict_output(ranks[0].cfg))


def _ranks(wl, G, inp):
    dev = torch.device("cuda")
    cfg = M.config_of(wl)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
    T_loc, E_loc = wl.T // G, wl.E // G
    return [ep.Rank(wl, r, G, g["x"][r * T_loc:(r + 1) * T_loc].contiguous(), g["Wr"],
                    g["bias"], W13[r * E_loc:(r + 1) * E_loc], W2p[r * E_loc:(r + 1) * E_loc])
            for r in range(G)]


@pytest.mark.parametrize("name", list(CASES))
def test_device_plan_equals_the_host_plan(name):
    """moe_ep_plan on the gathered counts gives every rank exactly the host
    plan: its caps, where its rows start at each owner, and the groups it
    receives (rows, first row, expert) with their total."""
    wl, G = CASES[name]
    inp = host_inputs(wl)
    ranks = _ranks(wl, G, inp)
    counts = [r.route().clone() for r in ranks]
    host = ep.make_plan(np.stack([c.cpu().numpy() for c in counts]).astype(np.int64), wl.T, wl.k,
                        wl.E, wl.cf, ranks[0].pad)
    counts_all = torch.cat(counts)
    C = ep.capacity(wl.T, wl.k, wl.E, wl.cf)
    for r in ranks:
        d = ep.device_plan(r, counts_all, C)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(d["cap"].cpu().numpy(),
                                      host.cap[r.rank].clip(max=2 ** 31 - 1))
        np.testing.assert_array_equal(d["row_start"].cpu().numpy(),
                                      ep.peer_row_starts(host, r.rank))
        rows, off, wi = host.groups(r.rank)
        np.testing.assert_array_equal(d["group_rows"].cpu().numpy(), rows)
        np.testing.assert_array_equal(d["group_off"].cpu().numpy(), off)
        np.testing.assert_array_equal(d["group_weight"].cpu().numpy(), wi)
        assert int(d["recv_rows"].item()) == int(host.recv_rows(r.rank).sum())


@pytest.mark.parametrize("name", list(CASES))
def test_device_plan_step_matches_the_host_plan_step(name):
    """The peer-memory step with the plan on the device (nothing read back to
    the host) gives the host-planned step's output and statistics bit for
    bit (the host-planned step given the same static bound on a group's rows,
    min(C, T_all), which picks the GEMM layout)."""
    wl, G = CASES[name]
    inp = host_inputs(wl)
    bound = min(ep.capacity(wl.T, wl.k, wl.E, wl.cf), wl.T)
    _, out_h, stats_h, _ = run_emulated_peers(wl, G, inp, bound=bound)
    ranks = _ranks(wl, G, inp)
    pad = ranks[0].pad
    timer = ep.StepTimer()
    outs, stats_d, _ = ep.forward_emulated_peers_device(ranks, wl.T, wl.T * wl.k + wl.E * pad,
                                                        timer=timer)
    torch.cuda.synchronize()
    m4 = timer.share()
    assert 0.0 < m4["dispatch_share"] < 1.0, m4
    print(f"{name}: dispatch-time share {m4}")
    for r in ranks:
        assert M.moe_read_device_status(r.b["ws"]) == 0
        assert M.moe_read_device_status(r.ffn_ws_dev) == 0
    out_d = torch.cat([o.clone() for o in outs])
    assert torch.equal(out_d, out_h)
    assert torch.equal(stats_d, stats_h)


def test_grouped_ffn_flags_an_oversized_group():
    """A group longer than max_group_rows is clamped and MOE_ERR_SHAPE
    recorded; the call itself completes."""
    wl = Workload("ep_guard", T=64, d=128, h=128, E=2, k=1)
    cfg = M.config_of(wl)
    dev = torch.device("cuda")
    inp = host_inputs(wl)
    W13, W2p = M.pack_weights(cfg, inp["w1"].to(dev), inp["w3"].to(dev), inp["w2"].to(dev))
    x = inp["x"].to(dev)
    rows = torch.tensor([48, 16], dtype=torch.int32, device=dev)
    off = torch.tensor([0, 48], dtype=torch.int32, device=dev)
    wi = torch.tensor([1, 0], dtype=torch.int32, device=dev)
    y = torch.zeros((64, 128), dtype=torch.float32, device=dev)
    ws = torch.empty(M.moe_grouped_workspace_size(cfg, 64, 32), dtype=torch.uint8, device=dev)
    M.moe_expert_ffn_grouped(cfg, x, 64, rows, off, wi, 32, W13, W2p, y, ws)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(ws) == 2  # MOE_ERR_SHAPE
    # the in-bound group (16 rows of expert 0) is computed as the oracle says
    ocfg = O.cfg_of(wl)
    ref = np.stack([O.ffn(128, 128, "bf16", inp["x"][48 + i].contiguous(), inp["w1"][0],
                          inp["w3"][0], inp["w2"][0]) for i in range(16)])
    got = y[48:64].double().cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-2 * np.abs(ref).max()

"""Data-parallel host logic on CPU ranks (gloo, world size 2): every rank routes
its own batch, the additive statistics sums are all-reduced with the same
helper the benchmark uses, and the result must equal the statistics of the
two batches routed as one (no capacity limit, so per-rank routing equals the
global one)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _sums_from_oracle(r, T, E):
    st = r["stats"]
    return torch.tensor([T, T * st["mean_entropy"], *(T * st["P"]), *r["routed"], *r["kept"]],
                        dtype=torch.float64)


def _rank(rank, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle as O
    from sparse_mixture_experts_22_b200 import dp
    from sparse_mixture_experts_22_b200 import inputs as I
    from sparse_mixture_experts_22_b200.workloads import Workload
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        wl = Workload("dp", T=40, d=64, h=128, E=8, k=2, zipf_s=0.8)
        Wr, b = I.router_weights(wl), I.router_bias(wl)
        x, _ = I.tokens(wl, Wr=Wr, b=b, stream=dp.token_stream(rank))
        r = O.route(O.cfg_of(wl), x, Wr, b)
        sums = _sums_from_oracle(r, wl.T, wl.E)
        assert sums.numel() == dp.sums_len(wl.E)
        dp.allreduce_sums(sums)
        out[rank] = sums.numpy().copy()
    finally:
        dist.destroy_process_group()


def test_stats_sums_all_reduce_over_gloo_ranks():
    import oracle as O
    from sparse_mixture_experts_22_b200 import dp
    from sparse_mixture_experts_22_b200 import inputs as I
    from sparse_mixture_experts_22_b200.workloads import Workload

    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    a, b = out[0], out[1]
    assert np.array_equal(a, b)

    # the two batches routed as one
    wl = Workload("dp", T=40, d=64, h=128, E=8, k=2, zipf_s=0.8)
    Wr, bias = I.router_weights(wl), I.router_bias(wl)
    xs = [I.tokens(wl, Wr=Wr, b=bias, stream=dp.token_stream(r))[0] for r in range(WORLD)]
    xg = torch.cat(xs)
    wg = wl.scaled(T=WORLD * wl.T)
    rg = O.route(O.cfg_of(wg), xg, Wr, bias)
    ref = _sums_from_oracle(rg, wg.T, wg.E).numpy()
    E = wl.E
    assert a[0] == ref[0]
    np.testing.assert_array_equal(a[2 + E:], ref[2 + E:])  # counts: exact
    np.testing.assert_allclose(a[:2 + E], ref[:2 + E], rtol=1e-12)
    # the global load-balancing loss follows from the summed parts
    T, k = a[0], wl.k
    aux = E * np.sum(a[2 + E:2 + 2 * E] / (T * k) * a[2:2 + E] / T)
    assert abs(aux - rg["stats"]["aux_loss"]) < 1e-12

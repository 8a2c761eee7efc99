"""Expert parallelism across two GPUs, one process per GPU (skipped unless two
GPUs are visible).  Each rank holds half of the experts and half of the batch
and runs the peer-memory step (forward_dist_peers: rows stored into, and read
from, the owners' symmetric-memory buffers, stream-ordered barriers between the
phases, the plan computed on the device) twice in a row.  The two steps must
give the same bits, and the outputs of both ranks together must match the
oracle on the concatenated batch (the layer's bars) with the statistics.

The ranks run as spawned child processes with NVLS off and a short process-group
timeout, so that a rank that fails ends the others' next collective with an
error instead of leaving them waiting."""

import datetime
import os
import queue
import socket
import traceback

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = [
    pytest.mark.gpu,
    pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs"),
]

WL_ARGS = dict(name="ep2_gpu", T=1200, d=256, h=384, E=8, k=2, cf=(1, 1), zipf_s=1.0)
WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), NCCL_NVLS_ENABLE="0")
    import torch.distributed as dist

    import sparse_mixture_experts_22_b200 as M
    from layer_check import host_inputs
    from sparse_mixture_experts_22_b200 import ep
    from sparse_mixture_experts_22_b200.workloads import Workload

    dev = torch.device("cuda", rank)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        wl = Workload(**WL_ARGS)
        inp = host_inputs(wl)
        cfg = M.config_of(wl)
        g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        W13, W2p = M.pack_weights(cfg, g["w1"], g["w3"], g["w2"])
        T_loc, E_loc = wl.T // WORLD, wl.E // WORLD
        r = ep.Rank(wl, rank, WORLD, g["x"][rank * T_loc:(rank + 1) * T_loc].contiguous(),
                    g["Wr"], g["bias"], W13[rank * E_loc:(rank + 1) * E_loc],
                    W2p[rank * E_loc:(rank + 1) * E_loc])
        out1, stats1, _ = ep.forward_dist_peers(r, wl.T)
        out1 = out1.clone()
        out2, stats2, _ = ep.forward_dist_peers(r, wl.T)
        torch.cuda.synchronize(dev)
        same = bool(torch.equal(out1, out2) and torch.equal(stats1, stats2))
        status = M.moe_read_device_status(r.b["ws"])
        parts = [torch.empty_like(out2) for _ in range(WORLD)]
        dist.all_gather(parts, out2.contiguous())
        torch.cuda.synchronize(dev)
        if rank == 0:
            results.put(("ok", rank, same, status, torch.cat(parts).cpu(), stats2.cpu()))
        else:
            results.put(("ok", rank, same, status, None, None))
    except Exception:  # reported to the parent, which fails the test
        results.put(("error", rank, traceback.format_exc()))
    finally:
        dist.destroy_process_group()


def test_two_gpus_peer_memory_step_matches_the_oracle():
    import oracle as O
    from layer_check import check_output, check_stats, host_inputs, strict_output

    import sparse_mixture_experts_22_b200 as M
    from sparse_mixture_experts_22_b200.workloads import Workload

    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(rank, port, results)) for rank in range(WORLD)]
    for p in procs:
        p.start()
    got = []
    try:
        for _ in range(WORLD):
            got.append(results.get(timeout=600))
    except queue.Empty:
        pass
    for p in procs:
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
            p.join()
    errors = [g for g in got if g[0] == "error"]
    assert not errors, errors
    assert len(got) == WORLD, f"only {len(got)} of {WORLD} ranks reported"
    for _, rank, same, status, _, _ in got:
        assert same, f"rank {rank}: two steps in a row gave different bits"
        assert status == 0, f"rank {rank}: device status {status}"
    out, stats = next((g[4], g[5]) for g in got if g[1] == 0)
    wl = Workload(**WL_ARGS)
    inp = host_inputs(wl)
    ref = O.forward(O.cfg_of(wl), inp)
    cfg_loc = M.make_config(wl.T // WORLD, wl.d, wl.h, wl.E, wl.k, dtype=wl.dtype,
                            has_bias=wl.has_bias)
    check_output(out.cuda(), ref["out"], "two GPUs", strict=strict_output(cfg_loc))
    check_stats(ref, stats.cuda(), wl.T)

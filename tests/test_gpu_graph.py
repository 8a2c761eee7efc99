"""The forward layer captured in a CUDA graph and replayed.

moe_forward issues its kernels, the zeroing of the CTA-pair work counters and
the fork and join of the shared experts' stream without reading anything back
to the host, so one call can be captured whole (programmatic dependent launch
edges included) and replayed.  Every replay must give the eager call's output,
statistics and routing bit for bit on the same inputs, and leave the device
status clean."""

import pytest
import torch

import sparse_mixture_experts_22_b200 as M
from layer_check import device_layer, host_inputs, run_forward
from sparse_mixture_experts_22_b200.workloads import Workload

pytestmark = pytest.mark.gpu

CASES = {
    # at most 128 tokens: fused routing and dispatch, swapped GEMMs, split-K down
    "swap": Workload("g_swap", T=100, d=256, h=512, E=6, k=2),
    # token-major one-SM tiles, capacity binding, router bias
    "tok_cap": Workload("g_tok_cap", T=600, d=256, h=384, E=4, k=2, cf=(5, 4), zipf_s=0.7),
    # shared experts on their own stream beside the routed ones
    "shared": Workload("g_shared", T=200, d=256, h=256, E=4, k=2, n_shared=2, h_shared=256,
                       cf=(3, 2)),
    # token-major tiles on SM pairs (work counters zeroed inside the graph)
    "pair_tok": Workload("g_pair_tok", T=1300, d=256, h=384, E=3, k=2, zipf_s=0.3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_gives_the_eager_bits(name):
    wl = CASES[name]
    inp = host_inputs(wl)
    cfg, g, W = device_layer(wl, inp)
    W13, W2p, W13s, W2s = W
    eager = run_forward(cfg, g, W)
    keys = ("out", "stats", "topk_idx", "topk_gate", "kept", "slot_of")
    ref = {k: eager[k].clone() for k in keys}

    bufs = M.alloc_layer(cfg, g["x"].device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        # one call on the capturing stream first (lazy set-up: kernel attributes,
        # the shared experts' stream and its events)
        M.forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, W13s, W2s, bufs=bufs)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            M.forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, W13s, W2s, bufs=bufs)
    torch.cuda.synchronize()
    for _ in range(2):
        for k in keys:
            bufs[k].zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert M.moe_read_device_status(bufs["ws"]) == 0
        for k in keys:
            assert torch.equal(bufs[k], ref[k]), k
    del graph

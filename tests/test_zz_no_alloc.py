"""moe_route_static: routing for callers that cannot allocate device memory
(a workspace-free variant of moe_route whose scratch is a fixed device array
inside the library).  Called through the C ABI, it must give what moe_route
gives on the same batch, and what the fp64 oracle's routing gives (the same
expert sets, gates within the parity tests' bound), on two calls in a row with
different batches (so a stale result left in the shared array would be
caught).

This file is collected last on purpose; it runs alone as well.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O

from sparse_mixture_experts_22_b200 import binding as B
from sparse_mixture_experts_22_b200 import inputs as I
from sparse_mixture_experts_22_b200.workloads import Workload

pytestmark = pytest.mark.gpu

GATE_ABS = 2.5e-5  # the gate tolerance of the parity tests


def _lib():
    L = B.load()
    fn = L.moe_route_static
    fn.argtypes = [ctypes.POINTER(B.MoEConfig)] + [ctypes.c_void_p] * 6
    fn.restype = ctypes.c_int
    return fn


def _route_with_workspace(cfg, x, Wr, bias):
    T, k = cfg.T, cfg.k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(B.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    B.moe_route(cfg, x, Wr, bias, idx, gate, ws)
    return idx, gate


def _route_static(fn, cfg, x, Wr, bias):
    T, k = cfg.T, cfg.k
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = fn(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(Wr.data_ptr()),
            ctypes.c_void_p(bias.data_ptr()) if bias is not None else None,
            ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(gate.data_ptr()),
            ctypes.c_void_p(stream))
    assert rc == 0, B.load().moe_last_error().decode()
    return idx, gate


@pytest.mark.parametrize("wl", [
    # Mixtral-shaped decode batch with a Zipf-skewed router
    Workload("decode_zipf", T=32, d=4096, h=128, E=8, k=2, zipf_s=1.0),
    # many experts, top-6, 256 tokens (the limit), fp32 tokens
    Workload("wide_f32", T=256, d=256, h=128, E=160, k=6, dtype="f32"),
])
def test_static_route_matches_workspace_route_twice(wl):
    fn = _lib()
    cfg = B.config_of(wl)
    Wr = I.router_weights(wl).cuda()
    bias = I.router_bias(wl)
    bias = bias.cuda() if bias is not None else None
    for call in range(2):
        x, _ = I.tokens(wl, Wr=Wr.cpu(), b=bias.cpu() if bias is not None else None,
                        stream=f"x.static{call}")
        x_host = x.clone()
        x = x.cuda()
        idx_s, gate_s = _route_static(fn, cfg, x, Wr, bias)
        idx_w, gate_w = _route_with_workspace(cfg, x, Wr, bias)
        torch.cuda.synchronize()
        assert torch.equal(idx_s, idx_w), f"call {call}: top-k differs"
        err = (gate_s - gate_w).abs().max().item()
        assert err <= GATE_ABS, f"call {call}: gates differ by {err}"
        # against the fp64 oracle: expert sets bit-exact, gates per (token, expert)
        r = O.route(O.cfg_of(wl), x_host, Wr.cpu(), bias.cpu() if bias is not None else None)
        idx = idx_s.cpu().numpy()
        gate = gate_s.cpu().numpy()
        assert np.array_equal(np.sort(idx, 1), np.sort(r["idx"], 1)), f"call {call}: sets"
        g_gpu = np.take_along_axis(gate, np.argsort(idx, 1), 1)
        g_ref = np.take_along_axis(r["gate"], np.argsort(r["idx"], 1), 1)
        oerr = np.abs(g_gpu - g_ref).max()
        assert oerr <= GATE_ABS, f"call {call}: gates off the oracle by {oerr}"


def test_static_route_rejects_oversized_batches():
    fn = _lib()
    cfg = B.make_config(257, 128, 128, 8, 2)
    x = torch.zeros((257, 128), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((128, 8), dtype=torch.float32, device="cuda")
    idx = torch.empty((257, 2), dtype=torch.int32, device="cuda")
    gate = torch.empty((257, 2), dtype=torch.float32, device="cuda")
    rc = fn(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(Wr.data_ptr()),
            None, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(gate.data_ptr()), None)
    assert rc == 2
    assert b"MOE_ROUTE_STATIC_MAX_T" in B.load().moe_last_error()

"""Failure detection without a GPU fault: every wait of the tensor-core kernels
is bounded.  The test hook makes the epilogue that takes work unit 0 wait on a
signal that is never sent; with a 5 ms bound the wait runs out, and the kernels must record
MOE_ERR_TIMEOUT in the device status word, let their in-flight copies and MMAs
finish, release tensor memory and return, leaving the context usable -- the
next call with the hook off gives the normal result bit for bit."""

import pytest
import torch

from layer_check import device_layer, host_inputs, run_forward
from sparse_mixture_experts_22_b200 import binding as B
from sparse_mixture_experts_22_b200.workloads import Workload

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000
SHORT_LIMIT_NS = 5_000_000


@pytest.mark.parametrize("wl", [
    Workload("swap_timeout", T=100, d=256, h=512, E=6, k=2),            # swapped GEMMs
    Workload("tok_timeout", T=600, d=256, h=384, E=4, k=2, cf=(5, 4)),  # token-major GEMMs
    # CTA-pair GEMMs: swapped tiles (experts of up to 219 tokens) and token-major
    # tiles of 256 tokens (experts of over 1024 tokens)
    Workload("pair_swap_timeout", T=700, d=512, h=384, E=8, k=2, cf=(5, 4), zipf_s=0.8),
    Workload("pair_tok_timeout", T=1300, d=256, h=384, E=3, k=2, zipf_s=0.3),
])
def test_wait_bound_reports_timeout_and_context_survives(wl):
    inp = host_inputs(wl)
    cfg, g, W = device_layer(wl, inp)
    ref = run_forward(cfg, g, W)
    assert B.moe_read_device_status(ref["ws"]) == 0
    out_ref = ref["out"].clone()

    B.moe_set_wait_limit_ns(SHORT_LIMIT_NS)
    B.moe_set_test_stall(True)
    B.moe_set_pair_tiles(2)  # the swapped pair tiles too
    try:
        bad = run_forward(cfg, g, W)
        status = B.moe_read_device_status(bad["ws"])
    finally:
        B.moe_set_test_stall(False)
        B.moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
        B.moe_set_pair_tiles(1)
    assert status == 7  # MOE_ERR_TIMEOUT

    # the context still works and the layer gives the same bits again
    again = run_forward(cfg, g, W)
    assert B.moe_read_device_status(again["ws"]) == 0
    assert torch.equal(again["out"], out_ref)

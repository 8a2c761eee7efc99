"""Host-side checks of the C ABI: the library loads, exports every entry point
include/moe.h declares, and its host-only calls (capacity, workspace size,
argument checks) behave, without touching a GPU."""

import ctypes
import os
import re

import pytest

import sparse_mixture_experts_22_b200 as M
from sparse_mixture_experts_22_b200 import binding as B
from sparse_mixture_experts_22_b200 import build as build_mod
from sparse_mixture_experts_22_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build_mod.build()


def declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt)
    return names


def test_every_declared_symbol_is_exported():
    names = declared()
    assert len(names) >= 18
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(B.EXPORTS) <= set(names)


def test_capacity_matches_the_worked_example():
    # batch 2048, 8 experts, top-2, capacity factor 1.25 -> 640 per expert
    assert M.moe_capacity(M.make_config(2048, 4096, 14336, 8, 2, cf=(5, 4))) == 640
    assert M.moe_capacity(M.config_of(WORKLOADS["deepseek"])) == 231
    assert M.moe_capacity(M.config_of(WORKLOADS["large"])) == 6144
    assert M.moe_capacity(M.config_of(WORKLOADS["decode"])) == 32  # no limit: T


def test_workspace_and_perm_rows():
    for name, wl in WORKLOADS.items():
        cfg = M.config_of(wl)
        ws = M.moe_workspace_size(cfg)
        rows = M.moe_perm_rows(cfg)
        splits = M.moe_ffn_splits(cfg)
        assert rows >= min(wl.T * wl.k, wl.E * M.moe_capacity(cfg))
        assert ws >= rows * wl.d * (2 if wl.dtype == "bf16" else 4) * 2
        assert 1 <= splits <= 8
    # decode streams the weights with a split-K down projection
    assert M.moe_ffn_splits(M.config_of(WORKLOADS["decode"])) > 1
    assert M.moe_workspace_size(M.make_config(0, 128, 128, 4, 2)) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(T=8, d=100, h=128, E=4, k=2), 2),          # d not a multiple of 128
    (dict(T=8, d=128, h=200, E=4, k=2), 2),          # h not a multiple of 128
    (dict(T=8, d=128, h=128, E=4, k=5), 2),          # k > E
    (dict(T=8, d=128, h=128, E=16, k=9), 2),         # k > 8
    (dict(T=8, d=128, h=128, E=0, k=1), 2),          # no experts
    (dict(T=-1, d=128, h=128, E=4, k=2), 2),         # negative T
    (dict(T=8, d=128, h=128, E=4, k=2, cf=(0, 4)), 1),  # zero capacity factor
    (dict(T=8, d=128, h=128, E=4, k=2, n_shared=2, h_shared=100), 2),
])
def test_invalid_configs_are_rejected(kw, code):
    with pytest.raises(B.MoEError) as e:
        M.moe_workspace_size(M.make_config(**kw))
    assert e.value.code == code
    assert "invalid config" in str(e.value)


def test_bad_dtype_is_rejected():
    cfg = M.make_config(8, 128, 128, 4, 2)
    cfg.act_dtype = 7
    with pytest.raises(B.MoEError) as e:
        M.moe_capacity(cfg)
    assert e.value.code == 3


def test_null_config_is_rejected():
    lib = B.load()
    v = ctypes.c_int64()
    assert lib.moe_capacity(None, ctypes.byref(v)) == 1
    assert b"NULL" in lib.moe_last_error()


def test_training_workspaces():
    for name, wl in WORKLOADS.items():
        if wl.dtype != "bf16":
            continue
        inf = M.moe_workspace_size(M.config_of(wl))
        tr = M.config_of(wl, train=True)
        # the forward keeps the gate/up pre-activations (bf16 [perm_rows][2h])
        assert M.moe_workspace_size(tr) >= inf + M.moe_perm_rows(tr) * 2 * wl.h * 2
        assert M.moe_backward_workspace_size(tr) > 0
    # fp32 layers have no backward pass; train must be 0 or 1
    with pytest.raises(B.MoEError) as e:
        M.moe_workspace_size(M.make_config(8, 128, 128, 4, 2, dtype="f32", train=True))
    assert e.value.code == 8
    cfg = M.make_config(8, 128, 128, 4, 2)
    cfg.train = 2
    with pytest.raises(B.MoEError) as e:
        M.moe_workspace_size(cfg)
    assert e.value.code == 1
    # the backward workspace exists only for a training config
    with pytest.raises(B.MoEError) as e:
        M.moe_backward_workspace_size(M.make_config(8, 128, 128, 4, 2))
    assert e.value.code == 1


def _peer_call_codes(cfg, world, ptrs):
    """Return codes of the two peer entry points for fake (never dereferenced)
    addresses; every case here fails in the host-side checks."""
    lib = B.load()
    fake = ctypes.c_void_p(0x100000)
    ws_bytes = M.moe_workspace_size(cfg)
    arr = (ctypes.c_void_p * max(len(ptrs), 1))(*[ctypes.c_void_p(p) if p else None
                                                  for p in ptrs])
    d = lib.moe_dispatch_peers(ctypes.byref(cfg), fake, fake, fake, world, arr, None, fake, fake,
                               fake, None, fake, fake, ws_bytes, None)
    c = lib.moe_combine_peers(ctypes.byref(cfg), world, arr, None, fake, fake, fake, fake, None,
                              fake, None)
    return d, c


@pytest.mark.parametrize("kw,world,ptrs,code", [
    (dict(), 0, [], 1),                                  # no ranks
    (dict(), 65, [0x200000] * 65, 1),                    # above MOE_MAX_PEERS
    (dict(), 3, [0x200000] * 3, 2),                      # 8 experts over 3 ranks
    (dict(), 2, [0x200000, 0x200008], 4),                # a row pointer off 16 bytes
    (dict(), 2, [0x200000, 0], 1),                       # a NULL row pointer
    (dict(overflow="reroute", cf=(1, 1)), 2, [0x200000] * 2, 8),  # drop policy only
])
def test_peer_calls_check_their_arguments(kw, world, ptrs, code):
    cfg = M.make_config(64, 128, 128, 8, 2, **kw)
    d, c = _peer_call_codes(cfg, world, ptrs)
    assert d == code, B.load().moe_last_error()
    assert c == code, B.load().moe_last_error()


@pytest.mark.parametrize("world,rank,C,code", [
    (0, 0, 10, 1),     # no ranks
    (65, 0, 10, 1),    # above MOE_MAX_PEERS
    (3, 0, 10, 2),     # 8 experts over 3 ranks
    (2, 2, 10, 1),     # rank out of range
    (2, -1, 10, 1),
    (2, 0, -1, 1),     # negative capacity
])
def test_ep_plan_checks_its_arguments(world, rank, C, code):
    cfg = M.make_config(64, 128, 128, 8, 2)
    fake = ctypes.c_void_p(0x100000)
    rc = B.load().moe_ep_plan(ctypes.byref(cfg), world, rank, fake, C, fake, fake, fake, fake,
                              fake, fake, None)
    assert rc == code, B.load().moe_last_error()


def test_peer_dispatch_is_bf16_only():
    cfg = M.make_config(64, 128, 128, 8, 2, dtype="f32")
    d, _ = _peer_call_codes(cfg, 2, [0x200000] * 2)
    assert d == 3


def test_binding_refuses_host_and_strided_tensors():
    import torch
    with pytest.raises(ValueError):
        B._p(torch.zeros(4))
    assert B._p(None) is None


def test_pair_tile_mode_is_checked():
    lib = B.load()
    assert lib.moe_set_pair_tiles(3) == 1
    assert lib.moe_set_pair_tiles(-1) == 1
    assert lib.moe_set_pair_tiles(1) == 0  # the default, restored


def test_shared_sm_budget_is_checked():
    lib = B.load()
    assert lib.moe_set_shared_sms(3) == 1      # odd: SMs go in pairs
    assert lib.moe_set_shared_sms(-2) == 1
    assert lib.moe_set_shared_sms(2048) == 1
    assert lib.moe_set_shared_sms(24) == 0
    assert lib.moe_set_shared_sms(0) == 0      # the default, restored


def test_hidden_mode_is_checked_and_reported():
    cfg = M.make_config(64, 128, 128, 8, 2)
    assert M.moe_hidden_split(cfg)          # auto: every expert keeps <= 128 rows
    cfg_big = M.make_config(4096, 128, 128, 8, 2)
    assert not M.moe_hidden_split(cfg_big)  # auto: experts of up to 4096 rows
    assert M.moe_hidden_split(M.make_config(4096, 128, 128, 8, 2, hidden="split"))
    assert not M.moe_hidden_split(M.make_config(64, 128, 128, 8, 2, hidden="bf16"))
    assert not M.moe_hidden_split(M.make_config(64, 128, 128, 8, 2, dtype="f32",
                                                hidden="split"))
    cfg.hidden_mode = 3
    with pytest.raises(B.MoEError) as e:
        M.moe_workspace_size(cfg)
    assert e.value.code == 1
    # the split doubles the hidden activations' share of the workspace
    a = M.moe_workspace_size(M.make_config(4096, 128, 256, 8, 2, hidden="bf16"))
    b = M.moe_workspace_size(M.make_config(4096, 128, 256, 8, 2, hidden="split"))
    rows = M.moe_perm_rows(M.make_config(4096, 128, 256, 8, 2))
    assert b - a >= rows * 256 * 2

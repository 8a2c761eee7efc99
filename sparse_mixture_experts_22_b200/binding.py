"""Python binding of libmoe_b200.so (include/moe.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their device pointers and the
current CUDA stream to the C ABI of the same name, and raises MoEError when
the library returns a non-zero status.  No step of the layer runs here; the
library must be present (build it with sparse_mixture_experts_22_b200/build.py)
and the calls fail loudly without it.
"""

import ctypes
import os
from typing import Dict, List, Optional, Tuple

import torch

from .workloads import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_ARG", 2: "MOE_ERR_SHAPE", 3: "MOE_ERR_DTYPE",
          4: "MOE_ERR_ALIGN", 5: "MOE_ERR_WORKSPACE", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_TIMEOUT",
          8: "MOE_ERR_UNSUPPORTED"}

EXPORTS = ["moe_capacity", "moe_workspace_size", "moe_perm_rows", "moe_ffn_splits",
           "moe_last_error", "moe_pack_weights", "moe_route", "moe_dispatch", "moe_expert_ffn",
           "moe_combine", "moe_aux_stats", "moe_stats_sums", "moe_stats_finalize", "moe_forward",
           "moe_read_device_status", "moe_set_wait_limit_ns", "moe_set_test_stall",
           "moe_trace_begin", "moe_trace_end", "moe_backward_workspace_size", "moe_backward",
           "moe_launch_count", "moe_segment_pad", "moe_route_counts", "moe_dispatch_capped",
           "moe_grouped_workspace_size", "moe_expert_ffn_grouped", "moe_combine_rows", "moe_set_pdl",
           "moe_dispatch_peers", "moe_combine_peers", "moe_hidden_split", "moe_set_pair_tiles",
           "moe_ep_plan", "moe_set_shared_overlap", "moe_set_shared_sms"]

MOE_MAX_PEERS = 64


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class MoEConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("d", ctypes.c_int32),
        ("h", ctypes.c_int32),
        ("E", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("n_shared", ctypes.c_int32),
        ("h_shared", ctypes.c_int32),
        ("cf_num", ctypes.c_int64),
        ("cf_den", ctypes.c_int64),
        ("act_dtype", ctypes.c_int32),
        ("has_bias", ctypes.c_int32),
        ("overflow", ctypes.c_int32),
        ("train", ctypes.c_int32),
        ("hidden_mode", ctypes.c_int32),
    ]


STATS_FIELDS = ["aux_loss", "overflow_rate", "mean_entropy", "tokens", "dropped"]

_lib = None


def load() -> ctypes.CDLL:
    """Load the C-ABI library; raise if it is missing (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "python sparse_mixture_experts_22_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        C = ctypes.POINTER(MoEConfig)
        sig = {
            "moe_capacity": [C, P],
            "moe_workspace_size": [C, P],
            "moe_perm_rows": [C, P],
            "moe_ffn_splits": [C, P],
            "moe_hidden_split": [C, P],
            "moe_pack_weights": [C, I, P, P, P, P, P, P],
            "moe_route": [C, P, P, P, P, P, P, P, S, P],
            "moe_dispatch": [C, P, P, P, P, P, P, P, P, P, S, P],
            "moe_expert_ffn": [C, P, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_combine": [C, P, P, P, P, P, P],
            "moe_aux_stats": [C, P, P, P, S, P, P],
            "moe_stats_sums": [C, P, P, P, S, P, P],
            "moe_stats_finalize": [C, P, P, P],
            "moe_forward": [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_read_device_status": [P, P, P],
            "moe_set_wait_limit_ns": [ctypes.c_uint64],
            "moe_set_test_stall": [I],
            "moe_trace_begin": [I, ctypes.c_char_p],
            "moe_trace_end": [P, P, P, I, P],
            "moe_backward_workspace_size": [C, P],
            "moe_launch_count": [P],
            "moe_segment_pad": [C, P],
            "moe_route_counts": [C, P, S, P, P],
            "moe_dispatch_capped": [C, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_grouped_workspace_size": [C, ctypes.c_int64, ctypes.c_int32, P],
            "moe_combine_rows": [C, P, P, P, P, P, P],
            "moe_dispatch_peers": [C, P, P, P, ctypes.c_int32, P, P, P, P, P, P, P, P, S, P],
            "moe_combine_peers": [C, ctypes.c_int32, P, P, P, P, P, P, P, P, P],
            "moe_ep_plan": [C, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_int64, P, P, P, P, P,
                            P, P],
            "moe_set_pdl": [I],
            "moe_set_pair_tiles": [I],
            "moe_set_shared_overlap": [I],
            "moe_set_shared_sms": [I],
            "moe_expert_ffn_grouped": [C, P, ctypes.c_int64, ctypes.c_int32, P, P, P,
                                       ctypes.c_int32, P, P, P, P, S, P],
            "moe_backward": [C, P, ctypes.c_float, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P,
                             P, P, P, P, P, P, P, P, S, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise MoEError(rc, load().moe_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


# ---------------------------------------------------------------- config

OVERFLOW = {"drop": 0, "reroute": 1}
HIDDEN = {"auto": 0, "split": 1, "bf16": 2}


def make_config(T, d, h, E, k, n_shared=0, h_shared=0, cf=None, dtype="bf16",
                has_bias=False, overflow="drop", train=False, hidden="auto") -> MoEConfig:
    num, den = (0, 0) if cf is None else cf
    return MoEConfig(T, d, h, E, k, n_shared, h_shared, num, den,
                     MOE_BF16 if dtype == "bf16" else MOE_F32, 1 if has_bias else 0,
                     OVERFLOW[overflow], 1 if train else 0, HIDDEN[hidden])


def config_of(wl: Workload, T: Optional[int] = None, train: bool = False,
              hidden: str = "auto") -> MoEConfig:
    return make_config(wl.T if T is None else T, wl.d, wl.h, wl.E, wl.k, wl.n_shared,
                       wl.h_shared, wl.cf, wl.dtype, wl.has_bias, wl.overflow, train, hidden)


def moe_hidden_split(cfg: MoEConfig) -> bool:
    """Whether this config feeds H to the down projection as two bf16 parts."""
    v = ctypes.c_int32()
    _check(load().moe_hidden_split(ctypes.byref(cfg), ctypes.byref(v)))
    return bool(v.value)


def act_dtype(cfg: MoEConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.act_dtype == MOE_BF16 else torch.float32


# ---------------------------------------------------------------- host helpers

def moe_capacity(cfg: MoEConfig) -> int:
    v = ctypes.c_int64()
    _check(load().moe_capacity(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


def moe_workspace_size(cfg: MoEConfig) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


def moe_perm_rows(cfg: MoEConfig) -> int:
    v = ctypes.c_int64()
    _check(load().moe_perm_rows(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


def moe_ffn_splits(cfg: MoEConfig) -> int:
    v = ctypes.c_int32()
    _check(load().moe_ffn_splits(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


# ---------------------------------------------------------------- steps

def moe_pack_weights(cfg, which, w1, w3, w2, W13, W2p, stream=None):
    _check(load().moe_pack_weights(ctypes.byref(cfg), which, _p(w1), _p(w3), _p(w2), _p(W13),
                                   _p(W2p), _stream(stream)))


def moe_route(cfg, x, Wr, bias, topk_idx, topk_gate, ws, logits=None, stream=None):
    _check(load().moe_route(ctypes.byref(cfg), _p(x), _p(Wr), _p(bias), _p(topk_idx),
                            _p(topk_gate), _p(logits), _p(ws), ws.numel() * ws.element_size(),
                            _stream(stream)))


def moe_dispatch(cfg, topk_idx, x, routed, kept, offsets, perm_token, slot_of, x_perm, ws,
                 stream=None):
    _check(load().moe_dispatch(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(routed), _p(kept),
                               _p(offsets), _p(perm_token), _p(slot_of), _p(x_perm), _p(ws),
                               ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_ffn(cfg, x_perm, offsets, kept, W13, W2p, x, W13s, W2s, y_perm, y_shared, ws,
                   stream=None):
    _check(load().moe_expert_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(kept), _p(W13),
                                 _p(W2p), _p(x), _p(W13s), _p(W2s), _p(y_perm), _p(y_shared),
                                 _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_combine(cfg, y_perm, slot_of, topk_gate, y_shared, out, stream=None):
    _check(load().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(slot_of), _p(topk_gate),
                              _p(y_shared), _p(out), _stream(stream)))


def moe_aux_stats(cfg, routed, kept, ws, stats, stream=None):
    _check(load().moe_aux_stats(ctypes.byref(cfg), _p(routed), _p(kept), _p(ws),
                                ws.numel() * ws.element_size(), _p(stats), _stream(stream)))


def moe_stats_sums(cfg, routed, kept, ws, sums, stream=None):
    _check(load().moe_stats_sums(ctypes.byref(cfg), _p(routed), _p(kept), _p(ws),
                                 ws.numel() * ws.element_size(), _p(sums), _stream(stream)))


def moe_stats_finalize(cfg, sums, stats, stream=None):
    _check(load().moe_stats_finalize(ctypes.byref(cfg), _p(sums), _p(stats), _stream(stream)))


def moe_forward(cfg, x, Wr, bias, W13, W2p, W13s, W2s, out, topk_idx, topk_gate, routed, kept,
                slot_of, stats, ws, stream=None):
    _check(load().moe_forward(ctypes.byref(cfg), _p(x), _p(Wr), _p(bias), _p(W13), _p(W2p),
                              _p(W13s), _p(W2s), _p(out), _p(topk_idx), _p(topk_gate),
                              _p(routed), _p(kept), _p(slot_of), _p(stats), _p(ws),
                              ws.numel() * ws.element_size(), _stream(stream)))


def moe_backward_workspace_size(cfg: MoEConfig) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


def moe_backward(cfg, grad_out, aux_coef, x, Wr, bias, W13t, W2t, W13st, W2st, topk_idx,
                 topk_gate, routed, kept, slot_of, ws, dx, dWr, db, dW13, dW2p, dW13s, dW2s,
                 dlogits, bws, stream=None):
    _check(load().moe_backward(
        ctypes.byref(cfg), _p(grad_out), float(aux_coef), _p(x), _p(Wr), _p(bias), _p(W13t),
        _p(W2t), _p(W13st), _p(W2st), _p(topk_idx), _p(topk_gate), _p(routed), _p(kept),
        _p(slot_of), _p(ws), ws.numel() * ws.element_size(), _p(dx), _p(dWr), _p(db), _p(dW13),
        _p(dW2p), _p(dW13s), _p(dW2s), _p(dlogits), _p(bws), bws.numel() * bws.element_size(),
        _stream(stream)))


def moe_read_device_status(ws, stream=None) -> int:
    v = ctypes.c_int32()
    _check(load().moe_read_device_status(_p(ws), ctypes.byref(v), _stream(stream)))
    return v.value


def moe_segment_pad(cfg: MoEConfig) -> int:
    v = ctypes.c_int32()
    _check(load().moe_segment_pad(ctypes.byref(cfg), ctypes.byref(v)))
    return v.value


def moe_route_counts(cfg, ws, counts, stream=None):
    _check(load().moe_route_counts(ctypes.byref(cfg), _p(ws), ws.numel() * ws.element_size(),
                                   _p(counts), _stream(stream)))


def moe_dispatch_capped(cfg, topk_idx, x, cap, routed, kept, offsets, perm_token, slot_of,
                        x_perm, ws, stream=None):
    _check(load().moe_dispatch_capped(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(cap),
                                      _p(routed), _p(kept), _p(offsets), _p(perm_token),
                                      _p(slot_of), _p(x_perm), _p(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)))


def moe_grouped_workspace_size(cfg, rows: int, max_group_rows: int) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_grouped_workspace_size(ctypes.byref(cfg), int(rows), int(max_group_rows),
                                             ctypes.byref(v)))
    return v.value


def moe_expert_ffn_grouped(cfg, x_rows, rows, group_rows, group_off, group_weight,
                           max_group_rows, W13, W2p, y_rows, ws, stream=None):
    _check(load().moe_expert_ffn_grouped(
        ctypes.byref(cfg), _p(x_rows), int(rows), int(group_rows.numel()), _p(group_rows),
        _p(group_off), _p(group_weight), int(max_group_rows), _p(W13), _p(W2p), _p(y_rows),
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_combine_rows(cfg, y_rows, slot_of, topk_gate, y_shared, out, stream=None):
    _check(load().moe_combine_rows(ctypes.byref(cfg), _p(y_rows), _p(slot_of), _p(topk_gate),
                                   _p(y_shared), _p(out), _stream(stream)))


def _ptr_array(ptrs):
    """A host array of device addresses (ints) for the peer entry points."""
    return (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(int(p)) for p in ptrs])


def moe_dispatch_peers(cfg, topk_idx, x, cap, dst_rows, routed, kept, offsets, perm_token,
                       slot_of, ws, dst_row_start=None, stream=None):
    """dst_rows: one device address per rank (ints), each rank's receive
    buffer; this rank's rows begin at row dst_row_start[q] there (device
    int32 [world]) or, when it is None, at dst_rows[q] itself."""
    arr = _ptr_array(dst_rows)
    _check(load().moe_dispatch_peers(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(cap),
                                     len(dst_rows), arr, _p(dst_row_start), _p(routed),
                                     _p(kept), _p(offsets), _p(perm_token), _p(slot_of), _p(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def moe_combine_peers(cfg, y_rows, topk_idx, offsets, slot_of, topk_gate, y_shared, out,
                      y_row_start=None, stream=None):
    """y_rows: one device address per rank (ints), each rank's fp32 output
    rows; this rank's rows begin at row y_row_start[q] (device int32
    [world]) or, when it is None, at y_rows[q] itself."""
    arr = _ptr_array(y_rows)
    _check(load().moe_combine_peers(ctypes.byref(cfg), len(y_rows), arr, _p(y_row_start),
                                    _p(topk_idx), _p(offsets), _p(slot_of), _p(topk_gate),
                                    _p(y_shared), _p(out), _stream(stream)))


def moe_ep_plan(cfg, world: int, rank: int, counts, C: int, cap, row_start, group_rows,
                group_off, group_weight, recv_rows, stream=None):
    """The expert-parallel plan of `rank` on the device (see include/moe.h)."""
    _check(load().moe_ep_plan(ctypes.byref(cfg), int(world), int(rank), _p(counts), int(C),
                              _p(cap), _p(row_start), _p(group_rows), _p(group_off),
                              _p(group_weight), _p(recv_rows), _stream(stream)))


def moe_launch_count() -> int:
    v = ctypes.c_uint64()
    _check(load().moe_launch_count(ctypes.byref(v)))
    return v.value


def moe_set_pdl(on: bool):
    _check(load().moe_set_pdl(1 if on else 0))


def moe_set_pair_tiles(mode):
    """0 none, 1 token-major pair tiles (default), 2 also swapped pair tiles;
    True means 2 (every pair tile), False 0."""
    if mode is True:
        mode = 2
    elif mode is False:
        mode = 0
    _check(load().moe_set_pair_tiles(int(mode)))


def moe_set_shared_overlap(on: bool):
    _check(load().moe_set_shared_overlap(1 if on else 0))


def moe_set_shared_sms(sms: int):
    """SMs set aside for the shared experts beside the routed ones (0: none)."""
    _check(load().moe_set_shared_sms(int(sms)))


def moe_set_wait_limit_ns(ns: int):
    _check(load().moe_set_wait_limit_ns(int(ns)))


def moe_set_test_stall(on: bool):
    _check(load().moe_set_test_stall(1 if on else 0))


def moe_trace_begin(max_calls: int, only: Optional[str] = None):
    _check(load().moe_trace_begin(max_calls, only.encode() if only else None))


def moe_trace_end(cap: int = 64) -> List[Tuple[str, int, float]]:
    names = (ctypes.c_char * 32 * cap)()
    launches = (ctypes.c_int * cap)()
    ms = (ctypes.c_double * cap)()
    n = ctypes.c_int()
    _check(load().moe_trace_end(names, launches, ms, cap, ctypes.byref(n)))
    return [(bytes(names[i]).split(b"\0")[0].decode(), launches[i], ms[i]) for i in range(n.value)]


# ---------------------------------------------------------------- buffers (device memory plumbing)

def stats_dict(stats: torch.Tensor) -> Dict[str, float]:
    v = stats.cpu().tolist()
    return dict(zip(STATS_FIELDS, v))


def alloc_layer(cfg: MoEConfig, device="cuda") -> Dict[str, torch.Tensor]:
    """Outputs and workspace of one moe_forward call, allocated by torch."""
    T, E, k, d = cfg.T, cfg.E, cfg.k, cfg.d
    return {
        "out": torch.empty((T, d), dtype=act_dtype(cfg), device=device),
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=device),
        "topk_gate": torch.empty((T, k), dtype=torch.float32, device=device),
        "routed": torch.empty(E, dtype=torch.int32, device=device),
        "kept": torch.empty(E, dtype=torch.int32, device=device),
        "slot_of": torch.empty((T, k), dtype=torch.int32, device=device),
        "stats": torch.zeros(len(STATS_FIELDS), dtype=torch.float64, device=device),
        "ws": torch.empty(max(moe_workspace_size(cfg), 256), dtype=torch.uint8, device=device),
    }


def pack_weights(cfg: MoEConfig, w1, w3, w2, shared: bool = False, stream=None):
    """Packs [n, d, hid] / [n, hid, d] device weights into (W13, W2p)."""
    n, d, hid = w1.shape
    if shared:
        W13 = torch.empty((2 * n * hid, d), dtype=w1.dtype, device=w1.device)
        W2p = torch.empty((d, n * hid), dtype=w1.dtype, device=w1.device)
    else:
        W13 = torch.empty((n, 2 * hid, d), dtype=w1.dtype, device=w1.device)
        W2p = torch.empty((n, d, hid), dtype=w1.dtype, device=w1.device)
    moe_pack_weights(cfg, 1 if shared else 0, w1, w3, w2, W13, W2p, stream)
    return W13, W2p


def forward(cfg: MoEConfig, x, Wr, bias, W13, W2p, W13s=None, W2s=None, bufs=None,
            with_stats: bool = True, stream=None) -> Dict[str, torch.Tensor]:
    """One moe_forward call; returns the buffers dict (allocated if not given)."""
    if bufs is None:
        bufs = alloc_layer(cfg, x.device)
    moe_forward(cfg, x, Wr, bias if cfg.has_bias else None, W13, W2p, W13s, W2s, bufs["out"],
                bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                bufs["slot_of"], bufs["stats"] if with_stats else None, bufs["ws"], stream)
    return bufs


def pack_weights_backward(cfg: MoEConfig, w1, w3, w2, shared: bool = False, stream=None):
    """Backward-layout copies (W13t, W2t) of [n, d, hid] / [n, hid, d] weights."""
    n, d, hid = w1.shape
    if shared:
        W13t = torch.empty((d, 2 * n * hid), dtype=w1.dtype, device=w1.device)
        W2t = torch.empty((n * hid, d), dtype=w1.dtype, device=w1.device)
    else:
        W13t = torch.empty((n, d, 2 * hid), dtype=w1.dtype, device=w1.device)
        W2t = torch.empty((n, hid, d), dtype=w1.dtype, device=w1.device)
    moe_pack_weights(cfg, 3 if shared else 2, w1, w3, w2, W13t, W2t, stream)
    return W13t, W2t


def alloc_grads(cfg: MoEConfig, device="cuda") -> Dict[str, torch.Tensor]:
    """Gradient outputs and backward workspace of one moe_backward call."""
    T, E, d, h = cfg.T, cfg.E, cfg.d, cfg.h
    f32 = dict(dtype=torch.float32, device=device)
    g = {
        "dx": torch.empty((T, d), **f32),
        "dWr": torch.empty((d, E), **f32),
        "db": torch.empty(E, **f32),
        "dW13": torch.empty((E, 2 * h, d), **f32),
        "dW2p": torch.empty((E, d, h), **f32),
        "dlogits": torch.empty((T, E), **f32),
        "bws": torch.empty(max(moe_backward_workspace_size(cfg), 256), dtype=torch.uint8,
                           device=device),
    }
    if cfg.n_shared:
        hsum = cfg.n_shared * cfg.h_shared
        g["dW13s"] = torch.empty((2 * hsum, d), **f32)
        g["dW2s"] = torch.empty((d, hsum), **f32)
    return g


def backward(cfg: MoEConfig, grad_out, aux_coef, x, Wr, bias, W13t, W2t, W13st, W2st, bufs,
             grads=None, stream=None) -> Dict[str, torch.Tensor]:
    """One moe_backward call after forward(...) filled `bufs` (cfg.train = 1)."""
    if grads is None:
        grads = alloc_grads(cfg, x.device)
    moe_backward(cfg, grad_out, aux_coef, x, Wr, bias if cfg.has_bias else None, W13t, W2t,
                 W13st, W2st, bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                 bufs["slot_of"], bufs["ws"], grads["dx"], grads["dWr"], grads["db"],
                 grads["dW13"], grads["dW2p"], grads.get("dW13s"), grads.get("dW2s"),
                 grads["dlogits"], grads["bws"], stream)
    return grads

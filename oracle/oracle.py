"""ctypes front end of the fp64 oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY.  Inputs are host torch tensors or numpy arrays in
the layer's own layouts (x [T, d]; W_r [d, E]; w1, w3 [E, d, h]; w2 [E, h, d];
shared experts [S, d, hs] / [S, hs, d]); bf16 tensors are passed as their raw
bytes and widened to double inside the oracle.  Every result is fp64 (or an
integer array).
"""

import ctypes
import os
from typing import Dict, Optional

import numpy as np
import torch

from .build import build

_F32, _BF16 = 0, 1


class OracleCfg(ctypes.Structure):
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
        ("dtype", ctypes.c_int32),
        ("has_bias", ctypes.c_int32),
        ("overflow", ctypes.c_int32),
    ]


_lib = None


def _bind(path: str):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    C = ctypes.POINTER(OracleCfg)
    L.oracle_capacity.argtypes = [C]
    L.oracle_capacity.restype = ctypes.c_int64
    L.oracle_logits.argtypes = [C, P, P, P, P]
    L.oracle_topk.argtypes = [C, P, P, P]
    L.oracle_probs.argtypes = [C, P, P]
    L.oracle_dispatch.argtypes = [C, P, ctypes.c_int64, P, P, P, P]
    L.oracle_stats.argtypes = [C, P, P, P, P]
    L.oracle_reroute.argtypes = [C, P, P, ctypes.c_int64, P, P, P, P]
    L.oracle_ffn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
    L.oracle_layer_rows.argtypes = [C, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_int64, P]
    L.oracle_threads.restype = ctypes.c_int
    L.oracle_backward.argtypes = [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                  ctypes.c_double, P, P, P, P, P, P, P, P, P, P]
    L.oracle_backward_rows.argtypes = [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                       ctypes.c_double, P, ctypes.c_int64, P, P]
    L.oracle_wgrad_block.argtypes = [C, P, P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                     P, ctypes.c_int, P, ctypes.c_int, P, P, P]
    return L


class using_library:
    """Temporarily route every oracle call through another build of the oracle
    (the mutation tests use this to show that a planted mistake fails a pin)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def threads() -> int:
    return lib().oracle_threads()


OVERFLOW = {"drop": 0, "reroute": 1}


def make_cfg(T, d, h, E, k, n_shared=0, h_shared=0, cf=None, dtype="bf16",
             has_bias=False, overflow="drop") -> OracleCfg:
    num, den = (0, 0) if cf is None else cf
    return OracleCfg(T, d, h, E, k, n_shared, h_shared, num, den,
                     _BF16 if dtype == "bf16" else _F32, 1 if has_bias else 0,
                     OVERFLOW[overflow])


def cfg_of(wl, T: Optional[int] = None) -> OracleCfg:
    return make_cfg(wl.T if T is None else T, wl.d, wl.h, wl.E, wl.k, wl.n_shared,
                    wl.h_shared, wl.cf, wl.dtype, wl.has_bias, wl.overflow)


def _ptr(a):
    """Address of a host array (torch tensor or numpy), which must be contiguous."""
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        assert a.device.type == "cpu" and a.is_contiguous()
        return ctypes.c_void_p(a.data_ptr())
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def capacity(cfg: OracleCfg) -> int:
    return int(lib().oracle_capacity(ctypes.byref(cfg)))


def logits(cfg: OracleCfg, x, Wr, bias=None) -> np.ndarray:
    z = np.empty((cfg.T, cfg.E), dtype=np.float64)
    lib().oracle_logits(ctypes.byref(cfg), _ptr(x), _ptr(Wr), _ptr(bias), _ptr(z))
    return z


def topk(cfg: OracleCfg, z: np.ndarray):
    idx = np.empty((cfg.T, cfg.k), dtype=np.int32)
    gate = np.empty((cfg.T, cfg.k), dtype=np.float64)
    lib().oracle_topk(ctypes.byref(cfg), _ptr(np.ascontiguousarray(z)), _ptr(idx), _ptr(gate))
    return idx, gate


def probs(cfg: OracleCfg, z: np.ndarray) -> np.ndarray:
    p = np.empty((cfg.T, cfg.E), dtype=np.float64)
    lib().oracle_probs(ctypes.byref(cfg), _ptr(np.ascontiguousarray(z)), _ptr(p))
    return p


def dispatch(cfg: OracleCfg, idx: np.ndarray, C: int):
    routed = np.empty(cfg.E, dtype=np.int32)
    kept = np.empty(cfg.E, dtype=np.int32)
    rank = np.empty((cfg.T, cfg.k), dtype=np.int32)
    keep = np.empty((cfg.T, cfg.k), dtype=np.int8)
    lib().oracle_dispatch(ctypes.byref(cfg), _ptr(np.ascontiguousarray(idx, dtype=np.int32)),
                          C, _ptr(routed), _ptr(kept), _ptr(rank), _ptr(keep))
    return routed, kept, rank, keep


def reroute(cfg: OracleCfg, z: np.ndarray, idx: np.ndarray, C: int, kept, rank, keep):
    """Second pass of the reroute policy (updates kept, rank, keep in place);
    returns the expert serving each assignment."""
    expert = np.empty((cfg.T, cfg.k), dtype=np.int32)
    lib().oracle_reroute(ctypes.byref(cfg), _ptr(np.ascontiguousarray(z)),
                         _ptr(np.ascontiguousarray(idx, dtype=np.int32)), C, _ptr(kept),
                         _ptr(rank), _ptr(keep), _ptr(expert))
    return expert


def stats(cfg: OracleCfg, p: np.ndarray, routed: np.ndarray, kept: np.ndarray) -> Dict:
    out = np.empty(3 + cfg.E, dtype=np.float64)
    lib().oracle_stats(ctypes.byref(cfg), _ptr(np.ascontiguousarray(p)), _ptr(routed),
                       _ptr(kept), _ptr(out))
    return {"aux_loss": out[0], "overflow_rate": out[1], "mean_entropy": out[2],
            "P": out[3:].copy()}


def ffn(d: int, h: int, dtype: str, x_row, w1, w3, w2) -> np.ndarray:
    y = np.empty(d, dtype=np.float64)
    lib().oracle_ffn(d, h, _BF16 if dtype == "bf16" else _F32, _ptr(x_row), _ptr(w1),
                     _ptr(w3), _ptr(w2), _ptr(y))
    return y


def layer_rows(cfg: OracleCfg, x, expert, gate, keep, w1, w3, w2, w1s=None, w3s=None,
               w2s=None, rows=None) -> np.ndarray:
    """Layer output rows; `expert` is the expert serving each assignment (the
    router's choice, or the spare expert under the reroute policy)."""
    if rows is None:
        n = cfg.T
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows_arr.shape[0]
    out = np.empty((n, cfg.d), dtype=np.float64)
    lib().oracle_layer_rows(ctypes.byref(cfg), _ptr(x), _ptr(expert), _ptr(gate), _ptr(keep),
                            _ptr(w1), _ptr(w3), _ptr(w2), _ptr(w1s), _ptr(w3s), _ptr(w2s),
                            _ptr(rows_arr), n, _ptr(out))
    return out


def route(cfg: OracleCfg, x, Wr, bias=None) -> Dict:
    """Router, top-k, gates, full softmax, capacity, dispatch and statistics."""
    z = logits(cfg, x, Wr, bias if cfg.has_bias else None)
    idx, gate = topk(cfg, z)
    p = probs(cfg, z)
    C = capacity(cfg)
    routed, kept, rank, keep = dispatch(cfg, idx, C)
    if cfg.overflow == OVERFLOW["reroute"]:
        expert = reroute(cfg, z, idx, C, kept, rank, keep)
    else:
        expert = idx.copy()
    st = stats(cfg, p, routed, kept)
    return {"z": z, "idx": idx, "gate": gate, "p": p, "C": C, "routed": routed,
            "kept": kept, "rank": rank, "keep": keep, "expert": expert, "stats": st}


def forward(cfg: OracleCfg, inp: Dict, rows=None) -> Dict:
    """The whole layer; out holds the rows listed in `rows` (all tokens if None)."""
    r = route(cfg, inp["x"], inp["Wr"], inp.get("bias"))
    r["out"] = layer_rows(cfg, inp["x"], r["expert"], r["gate"], r["keep"], inp["w1"],
                          inp["w3"], inp["w2"], inp.get("w1s"), inp.get("w3s"),
                          inp.get("w2s"), rows)
    return r


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def backward(cfg: OracleCfg, inp: Dict, r: Dict, G, aux_coef: float = 0.0) -> Dict:
    """Gradients of L = <G, out> + aux_coef * aux (see oracle_backward).

    `r` is the routing of the same inputs (route()); G [T, d] in the layer
    dtype.  Returns fp64 arrays dx, dWr, db, dz, dw1, dw3, dw2 (and dw1s,
    dw3s, dw2s with shared experts) in the layer's own layouts."""
    T, d, h, E, k = cfg.T, cfg.d, cfg.h, cfg.E, cfg.k
    S, hs = cfg.n_shared, cfg.h_shared
    out = {"dx": np.empty((T, d)), "dWr": np.empty((d, E)), "db": np.empty(E),
           "dz": np.empty((T, E)), "dw1": np.empty((E, d, h)), "dw3": np.empty((E, d, h)),
           "dw2": np.empty((E, h, d))}
    if S:
        out.update({"dw1s": np.empty((S, d, hs)), "dw3s": np.empty((S, d, hs)),
                    "dw2s": np.empty((S, hs, d))})
    z = _c(r["z"], np.float64)
    idx = _c(r["idx"], np.int32)
    expert = _c(r["expert"], np.int32)
    gate = _c(r["gate"], np.float64)
    keep = _c(r["keep"], np.int8)
    routed = _c(r["routed"], np.int32)
    lib().oracle_backward(
        ctypes.byref(cfg), _ptr(inp["x"]), _ptr(inp["Wr"]), _ptr(z), _ptr(idx), _ptr(expert),
        _ptr(gate), _ptr(keep), _ptr(routed), _ptr(inp["w1"]), _ptr(inp["w3"]), _ptr(inp["w2"]),
        _ptr(inp.get("w1s")), _ptr(inp.get("w3s")), _ptr(inp.get("w2s")), _ptr(G),
        float(aux_coef), _ptr(out["dx"]), _ptr(out["dWr"]), _ptr(out["db"]), _ptr(out["dz"]),
        _ptr(out["dw1"]), _ptr(out["dw3"]), _ptr(out["dw2"]), _ptr(out.get("dw1s")),
        _ptr(out.get("dw3s")), _ptr(out.get("dw2s")))
    return out


def backward_rows(cfg: OracleCfg, inp: Dict, r: Dict, G, aux_coef: float, rows) -> Dict:
    """dx and dz rows of the listed tokens only (see oracle_backward_rows)."""
    rows_arr = _c(rows, np.int64)
    n = rows_arr.shape[0]
    dx = np.empty((n, cfg.d))
    dz = np.empty((n, cfg.E))
    lib().oracle_backward_rows(
        ctypes.byref(cfg), _ptr(inp["x"]), _ptr(inp["Wr"]), _ptr(_c(r["z"], np.float64)),
        _ptr(_c(r["idx"], np.int32)), _ptr(_c(r["expert"], np.int32)),
        _ptr(_c(r["gate"], np.float64)), _ptr(_c(r["keep"], np.int8)),
        _ptr(_c(r["routed"], np.int32)), _ptr(inp["w1"]), _ptr(inp["w3"]), _ptr(inp["w2"]),
        _ptr(inp.get("w1s")), _ptr(inp.get("w3s")), _ptr(inp.get("w2s")), _ptr(G),
        float(aux_coef), _ptr(rows_arr), n, _ptr(dx), _ptr(dz))
    return {"dx": dx, "dz": dz}


def wgrad_block(cfg: OracleCfg, inp: Dict, r: Dict, G, e: int, hi, ci,
                shared: bool = False) -> Dict:
    """dw1[ci, hi], dw3[ci, hi] and dw2[hi, ci] of one routed (or shared) expert,
    each returned as [len(hi), len(ci)] (see oracle_wgrad_block)."""
    hi_a = _c(hi, np.int32)
    ci_a = _c(ci, np.int32)
    ni, nc = hi_a.shape[0], ci_a.shape[0]
    o1, o3, o2 = np.empty((ni, nc)), np.empty((ni, nc)), np.empty((ni, nc))
    if shared:
        w1, w3, w2 = inp["w1s"], inp["w3s"], inp["w2s"]
    else:
        w1, w3, w2 = inp["w1"], inp["w3"], inp["w2"]
    lib().oracle_wgrad_block(
        ctypes.byref(cfg), _ptr(inp["x"]), _ptr(_c(r["expert"], np.int32)),
        _ptr(_c(r["gate"], np.float64)), _ptr(_c(r["keep"], np.int8)), _ptr(w1), _ptr(w3),
        _ptr(w2), _ptr(G), 1 if shared else 0, int(e), _ptr(hi_a), ni, _ptr(ci_a), nc,
        _ptr(o1), _ptr(o3), _ptr(o2))
    return {"dw1": o1, "dw3": o3, "dw2": o2}

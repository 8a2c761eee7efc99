#!/usr/bin/env python
"""Throughput of the sparse top-k MoE layer on B200.

One step = one pass of the whole layer (router, top-k, capacity dispatch,
expert FFNs, combine, statistics) over one batch of synthetic tokens, through
the library's public call (moe_forward).  Default workload: the large
Mixtral-shaped prefill layer (T=16384 tokens, d=4096, h=14336, 8 experts,
top-2, cf 1.5, Zipf(1.2) router bias, bf16), tensor-core bound; on one GPU the
same process then times the T=32 decode layer (weight streaming, HBM-bound) and
reports it under the line's "decode" key.  Under torchrun every rank runs its
own batch (weak scaling; weights replicated) and the per-rank routing
statistics are summed across ranks with one NCCL all-reduce.

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
instead, on a bounded sample of the same workload.  `--backward` (1 GPU) times
a training step instead: moe_forward with the pre-activations kept, then
moe_backward (gradients of <G, out> + 0.01 aux for every input and weight).
"""

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_22_b200 import binding as B  # noqa: E402
from sparse_mixture_experts_22_b200 import dp  # noqa: E402
from sparse_mixture_experts_22_b200 import inputs as I  # noqa: E402
from sparse_mixture_experts_22_b200.workloads import WORKLOADS  # noqa: E402

METRIC = "MoE-layer tokens/s (1xB200) and % of roofline (BF16 TC / HBM)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILES = os.path.join(ROOT, "profiles")
GEMM_SRCS = [os.path.join(ROOT, "sparse_mixture_experts_22_b200", "csrc", n)
             for n in ("gemm_tc.cu", "gemm_pair.cu", "common.cuh")]


def parse():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="large", choices=list(WORKLOADS))
    p.add_argument("--hidden-mode", default="auto", choices=["auto", "split", "bf16"],
                   help="how H reaches the down projection (moe_config.hidden_mode)")
    p.add_argument("--no-decode", action="store_true",
                   help="skip the decode layer timed after the main workload")
    p.add_argument("--no-split-line", action="store_true",
                   help="skip the same workload timed with H split (when the run's H is bf16)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="budget of the CPU-baseline sample")
    p.add_argument("--no-trace", action="store_true",
                   help="skip the per-kernel CUDA events in the timed region")
    p.add_argument("--trace-all", action="store_true",
                   help="time every kernel (one event after each launch) instead of only "
                        "the gate/up GEMM")
    p.add_argument("--overflow", default=None, choices=["drop", "reroute"],
                   help="capacity overflow policy (default: the workload's, drop)")
    p.add_argument("--hidden", type=int, default=0,
                   help="override the expert hidden width (small profiling cases only)")
    p.add_argument("--graph", action="store_true",
                   help="capture one step in a CUDA graph and replay it (1 GPU)")
    p.add_argument("--no-pdl", action="store_true",
                   help="launch the forward chain without programmatic dependent launch")
    p.add_argument("--pair", type=int, default=1, choices=[0, 1, 2],
                   help="CTA-pair GEMM tiles: 0 none, 1 token-major (default), 2 also swapped")
    p.add_argument("--no-overlap", action="store_true",
                   help="shared experts after the routed ones on one stream")
    p.add_argument("--shared-sms", type=int, default=-1,
                   help="SMs set aside for the shared experts beside the routed ones "
                        "(-1: the library's default)")
    p.add_argument("--backward", action="store_true",
                   help="time forward + backward (a training step) instead of the forward (1 GPU)")
    return p.parse_args()


AUX_COEF = 0.01


# ---------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_label(wl):
    return f"{wl.name}: {wl.describe()}"


def algorithmic(wl, kept):
    """Algorithmic FLOPs and bytes of one layer pass (kept assignments only;
    experts with no token are not read)."""
    d, h, E = wl.d, wl.h, wl.E
    ab = 2 if wl.dtype == "bf16" else 4
    N = int(sum(kept))
    active = sum(1 for n in kept if n > 0)
    T = wl.T
    flops = 2 * T * d * E + 6 * d * h * N + wl.n_shared * 6 * d * wl.h_shared * T
    wbytes = active * 3 * d * h * ab + wl.n_shared * 3 * d * wl.h_shared * ab
    byt = T * d * ab + 4 * d * E + wbytes + T * d * ab
    return flops, byt, N, active


def backward_algorithmic(wl, kept):
    """Algorithmic FLOPs and bytes of one backward pass: the backward GEMMs
    (12 N d h, shared 12 T d S hs), the router's two products (4 T d E); the
    bytes read (the backward-layout weights of active experts, G, x) and
    written (fp32 gradients of every weight, dx)."""
    d, h, E, T = wl.d, wl.h, wl.E, wl.T
    N = int(sum(kept))
    active = sum(1 for n in kept if n > 0)
    hs = wl.n_shared * wl.h_shared
    flops = 12.0 * N * d * h + 12.0 * T * d * hs + 4.0 * T * d * E
    byt = (active * 3 * d * h * 2 + 3 * d * hs * 2 + 2 * T * d * 2
           + E * 3 * d * h * 4 + 3 * d * hs * 4 + d * E * 4 + T * d * 4)
    return flops, byt


def kernel_work(name, wl, kept, splits):
    """Algorithmic work of one launch of a GEMM kernel: (bound, amount, unit)."""
    d, h = wl.d, wl.h
    ab = 2 if wl.dtype == "bf16" else 4
    N = int(sum(kept))
    active = sum(1 for n in kept if n > 0)
    E = wl.E
    # backward GEMMs (token-major tiles): the binding one of FLOPs and bytes
    kt = N + 63 * active
    bwd = {
        "gemm_dgate": (2.0 * N * d * h, active * h * d * 2 + N * d * 2 + 4 * N * 2 * h),
        "gemm_dx": (4.0 * N * d * h, active * 2 * h * d * 2 + N * 2 * h * 2 + N * d * 4),
        "gemm_dw2": (2.0 * N * d * h, E * d * h * 4 + (d + h) * kt * 2),
        "gemm_dw13": (4.0 * N * d * h, E * 2 * h * d * 4 + (2 * h + d) * kt * 2),
    }
    if name in bwd:
        fl, by = bwd[name]
        pk, _ = peaks()
        if fl / (pk["bf16_tflops"] * 1e12) >= by / (pk["hbm_gbs"] * 1e9):
            return "tensor", fl, "flops"
        return "hbm", by, "bytes"
    C = min(B.moe_capacity(B.config_of(wl)), wl.T)
    swapped = C <= 256
    if name == "gemm_gateup":
        if swapped:
            return "hbm", active * 2 * h * d * ab + N * d * ab + N * h * ab, "bytes"
        return "tensor", 4.0 * N * d * h, "flops"
    if name == "gemm_down":
        if swapped:
            return "hbm", active * d * h * ab + N * h * ab + splits * N * d * 4, "bytes"
        return "tensor", 2.0 * N * d * h, "flops"
    return None


def tile_stats(wl, kept, sms):
    """Token-major tile bookkeeping from the run's kept counts: the rows the
    128- and 256-row m tiles cover over the kept rows (padding), and the
    gate/up work units (m tiles x 128-wide hidden blocks) in waves of the SMs
    (one tile per SM, or per SM pair for 256-row tiles)."""
    N = max(int(sum(kept)), 1)
    out = {}
    for m, per in ((128, 1), (256, 2)):
        tiles = sum(-(-int(n) // m) for n in kept if n > 0)
        units = tiles * (wl.h // 128)
        out[f"m{m}"] = {"m_tiles": tiles, "padded_rows_frac": tiles * m / N,
                        "gateup_units": units, "waves": units / (sms // per)}
    return out


def dominant_roofline(trace, wl, cfg, kept):
    """Roofline of the dominant GEMM among the traced kernels: its algorithmic
    work per launch over its mean CUDA-event duration, against the measured
    HBM copy bandwidth (weight-streaming GEMMs) or the measured bf16 tensor
    rate (sustained for a kernel inside a long step; the burst figure beside)."""
    pk, pk_kind = peaks()
    splits = B.moe_ffn_splits(cfg)
    known = [r for r in trace if kernel_work(r[0], wl, kept, splits)]
    if not known:
        return None
    name, launches, tot_ms = max(known, key=lambda r: r[2])
    per = tot_ms / launches / 1000.0
    bound, amount, _ = kernel_work(name, wl, kept, splits)
    if bound == "hbm":
        ach, peak, unit = amount / per / 1e9, pk["hbm_gbs"], "GB/s"
        extra = {}
    else:
        ach, unit = amount / per / 1e12, "TFLOP/s"
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        extra = {"peak_kind": "bf16 sustained", "peak_burst": pk["bf16_tflops"],
                 "frac_burst": ach / pk["bf16_tflops"]}
    out = {"kernel": name, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
           "frac": ach / peak, "peak_source": pk_kind, "algorithmic_per_launch": amount,
           "launch_us": per * 1e6, "traffic": traffic_from_profile(name, wl.name)}
    out.update(extra)
    return out


def decode_line(args, dev, stream, wl_main, W_main):
    """The T=32 decode layer timed in the same process after the main workload
    (inputs resident in HBM; its 2.82 GB of expert weights stream from HBM each
    step), with its own dominant-kernel and layer rooflines."""
    wl = WORKLOADS["decode"]
    cfg = B.config_of(wl, hidden=args.hidden_mode)
    Wr = I.router_weights(wl)
    bias = I.router_bias(wl)
    x, _ = I.tokens(wl, Wr=Wr, b=bias)
    same = (wl.d, wl.h, wl.E, wl.seed, wl.dtype) == (wl_main.d, wl_main.h, wl_main.E,
                                                     wl_main.seed, wl_main.dtype)
    if same:  # the expert weights depend on the shape and the seed only
        W13, W2p = W_main[0], W_main[1]
    else:
        w = I.expert_weights(wl)
        W13, W2p = B.pack_weights(cfg, *(w[k].to(dev) for k in ("w1", "w3", "w2")))
    g = {"x": x.to(dev), "Wr": Wr.to(dev), "bias": bias.to(dev) if bias is not None else None}
    bufs = B.alloc_layer(cfg, dev)

    def step():
        B.moe_forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, None, None, bufs["out"],
                      bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                      bufs["slot_of"], bufs["stats"], bufs["ws"])

    steps = max(args.steps, 200)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    B.moe_trace_begin(steps, "gemm_gateup")
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    trace = B.moe_trace_end()
    ms = ev0.elapsed_time(ev1)
    status = B.moe_read_device_status(bufs["ws"])
    kept = bufs["kept"].cpu().tolist()
    pk, _ = peaks()
    flops, byts, N, active = algorithmic(wl, kept)
    t_step = ms / 1000.0 / steps
    roof_t = max(flops / (pk["bf16_tflops"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    return {"workload": workload_label(wl), "value": wl.T * steps / (ms / 1000.0),
            "unit": UNIT, "steps": steps, "ms_per_step": ms / steps,
            "hidden": "split" if B.moe_hidden_split(cfg) else "bf16",
            "roofline": dominant_roofline(trace, wl, cfg, kept),
            "layer_roofline": {"flops": flops, "bytes": byts, "time_us": roof_t * 1e6,
                               "frac": roof_t / t_step, "kept_assignments": N,
                               "active_experts": active},
            "clocks": clk, "device_status": status}


def split_line(args, dev, stream, wl, g, W):
    """The same workload timed with H fed to the down projection as two bf16
    parts (the mode whose output meets the relative-L1 bar against the
    unrounded fp64 reference), same inputs and weights, device-resident."""
    cfg = B.config_of(wl, hidden="split")
    W13, W2p, W13s, W2s = W
    bufs = B.alloc_layer(cfg, dev)

    def step():
        B.moe_forward(cfg, g["x"], g["Wr"], g["bias"], W13, W2p, W13s, W2s, bufs["out"],
                      bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                      bufs["slot_of"], bufs["stats"], bufs["ws"])

    steps = max(5, min(args.steps, 20))
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    kept = bufs["kept"].cpu().tolist()
    pk, _ = peaks()
    flops, byts, N, active = algorithmic(wl, kept)
    t_step = ms / 1000.0 / steps
    roof_t = max(flops / (pk["bf16_tflops"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    status = B.moe_read_device_status(bufs["ws"])
    del bufs
    return {"hidden": "split", "value": wl.T * steps / (ms / 1000.0), "unit": UNIT,
            "steps": steps, "ms_per_step": ms / steps,
            "layer_roofline": {"frac": roof_t / t_step, "time_us": roof_t * 1e6},
            "clocks": clk, "device_status": status}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"samples": 0, "note": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                power.append(float(r[3]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def traffic_from_profile(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current GEMM sources; None otherwise.  A summary of a smaller case
    of the workload (`<kernel>_<workload>_h<width>.ncu.txt`, the hidden width
    cut) records `scale_to_full`, the factor by which the launch's work units
    (and so its traffic) grow at full size."""
    cands = [os.path.join(PROFILES, f"{kernel}_{workload}.ncu.txt")]
    cands += sorted(glob.glob(os.path.join(PROFILES, f"{kernel}_{workload}_h*.ncu.txt")))
    for path in cands:
        if not os.path.exists(path):
            continue
        vals = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.startswith("#"):
                    k, v = line.split("=", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("gemm_source_sha256") != gemm_sources_sha():
            continue
        try:
            return float(vals["dram_bytes_per_launch"]) * float(vals.get("scale_to_full", 1))
        except (KeyError, ValueError):
            continue
    return None


def gemm_sources_sha():
    """SHA-256 over the tensor-core GEMM sources (one-SM and CTA-pair kernels)."""
    h = hashlib.sha256()
    for path in GEMM_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ---------------------------------------------------------------- inputs

def build_inputs(wl, rank, world, dev, keep_host, train=False, hidden="auto"):
    """Per-rank tokens; expert weights drawn on rank 0 and broadcast.  With
    train, also the backward-layout weights (one GPU)."""
    Wr = I.router_weights(wl)
    bias = I.router_bias(wl)
    x, _ = I.tokens(wl, Wr=Wr, b=bias, stream=dp.token_stream(rank))
    cfg = B.config_of(wl, train=train, hidden=hidden)
    Wb = (None, None, None, None)
    host = {"x": x, "Wr": Wr, "bias": bias}
    dt = I.torch_dtype(wl.dtype)
    if rank == 0:
        w = I.expert_weights(wl)
        w1, w3, w2 = (w[k].to(dev) for k in ("w1", "w3", "w2"))
        W13, W2p = B.pack_weights(cfg, w1, w3, w2)
        if train:
            Wb = B.pack_weights_backward(cfg, w1, w3, w2) + (None, None)
        del w1, w3, w2
        if keep_host:
            host.update(w)
        W13s = W2s = None
        if wl.n_shared:
            s = I.expert_weights(wl, shared=True)
            s1, s3, s2 = (s[k].to(dev) for k in ("w1", "w3", "w2"))
            W13s, W2s = B.pack_weights(cfg, s1, s3, s2, shared=True)
            if train:
                Wb = Wb[:2] + B.pack_weights_backward(cfg, s1, s3, s2, shared=True)
            del s1, s3, s2
            if keep_host:
                host.update({"w1s": s["w1"], "w3s": s["w3"], "w2s": s["w2"]})
    else:
        W13 = torch.empty((wl.E, 2 * wl.h, wl.d), dtype=dt, device=dev)
        W2p = torch.empty((wl.E, wl.d, wl.h), dtype=dt, device=dev)
        W13s = W2s = None
        if wl.n_shared:
            hs = wl.n_shared * wl.h_shared
            W13s = torch.empty((2 * hs, wl.d), dtype=dt, device=dev)
            W2s = torch.empty((wl.d, hs), dtype=dt, device=dev)
    if world > 1:
        dp.broadcast_weights([W13, W2p, W13s, W2s], src=0)
    torch.cuda.synchronize()
    dev_in = {"x": x.to(dev), "Wr": Wr.to(dev), "bias": bias.to(dev) if bias is not None else None}
    if train:
        dev_in["G"] = I.grad_out(wl).to(dev)
    return cfg, host, dev_in, (W13, W2p, W13s, W2s), Wb


# ---------------------------------------------------------------- CPU oracle timing

def oracle_row_seconds(O, cfg, x, r, host, T):
    """Seconds of oracle work per layer-output row: one untimed call first (its
    first-call costs: thread start-up, first touch of the weights), then a
    timed probe of a few rows per host thread."""
    import numpy as np
    w = (host["w1"], host["w3"], host["w2"], host.get("w1s"), host.get("w3s"), host.get("w2s"))
    O.layer_rows(cfg, x, r["expert"], r["gate"], r["keep"], *w, [0])
    probe = max(1, min(T, 2 * O.threads()))
    t0 = time.perf_counter()
    O.layer_rows(cfg, x, r["expert"], r["gate"], r["keep"], *w, np.arange(probe))
    return max((time.perf_counter() - t0) / probe, 1e-6)


def time_oracle(wl, host, budget_s):
    """Oracle on the host cores: routing of the whole batch plus the expert
    FFN rows of as many tokens as fit in about budget_s seconds."""
    import numpy as np
    import oracle as O
    cfg = O.cfg_of(wl)
    t0 = time.perf_counter()
    r = O.route(cfg, host["x"], host["Wr"], host["bias"])
    t_route = time.perf_counter() - t0
    t_row = oracle_row_seconds(O, cfg, host["x"], r, host, wl.T)
    rows_per_pass = max(1, min(wl.T, int(max(budget_s - t_route, 0.0) / t_row)))
    done, elapsed, passes = 0, 0.0, 0
    while elapsed < budget_s or passes == 0:
        t0 = time.perf_counter()
        r = O.route(cfg, host["x"], host["Wr"], host["bias"])
        O.layer_rows(cfg, host["x"], r["expert"], r["gate"], r["keep"], host["w1"], host["w3"],
                     host["w2"], host.get("w1s"), host.get("w3s"), host.get("w2s"),
                     np.arange(rows_per_pass))
        elapsed += time.perf_counter() - t0
        done += rows_per_pass
        passes += 1
        if rows_per_pass < wl.T:
            break
    sample = (f"{passes} pass(es): fp64 routing, capacity dispatch and statistics of the whole "
              f"T={wl.T} batch plus the layer output of {rows_per_pass} token row(s) per pass")
    return {"value": done / elapsed, "unit": UNIT, "cores": O.threads(), "kind": "oracle",
            "sample": sample, "seconds": elapsed}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    Wr = I.router_weights(wl)
    bias = I.router_bias(wl)
    x, _ = I.tokens(wl, Wr=Wr, b=bias)
    host = {"x": x, "Wr": Wr, "bias": bias}
    host.update(I.expert_weights(wl))
    if wl.n_shared:
        s = I.expert_weights(wl, shared=True)
        host.update({"w1s": s["w1"], "w3s": s["w3"], "w2s": s["w2"]})
    import numpy as np
    import oracle as O
    cfg = O.cfg_of(wl)
    # each step: the whole batch routed, and the outputs of a bounded row sample;
    # the sample is sized so that the whole run (warm-up and timed steps) takes
    # about REF_BUDGET_S: rows per step, or one row every `every` steps when even
    # one row per step would overrun
    REF_BUDGET_S = 120.0
    t0 = time.perf_counter()
    r0 = O.route(cfg, x, Wr, bias)
    t_route = time.perf_counter() - t0
    t_row = oracle_row_seconds(O, cfg, x, r0, host, wl.T)
    nsteps = max(1, args.steps + args.warmup)
    per_step = max(REF_BUDGET_S / nsteps - t_route, 0.0)
    rows, every = max(1, min(wl.T, int(min(0.5, per_step) / t_row))), 1
    if per_step < t_row:
        every = int(np.ceil(t_row / max(per_step, 1e-6)))
    sample_rows = np.arange(rows)
    count = [0]

    def step(i):
        r = O.route(cfg, x, Wr, bias)
        if i % every == 0:
            O.layer_rows(cfg, x, r["expert"], r["gate"], r["keep"], host["w1"], host["w3"],
                         host["w2"], host.get("w1s"), host.get("w3s"), host.get("w2s"),
                         sample_rows)
            count[0] += rows

    for i in range(args.warmup):
        step(i)
    count[0] = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = max(count[0], 1) / el
    if every == 1:
        sample = (f"each step: fp64 routing, dispatch and statistics of the whole T={wl.T} batch "
                  f"plus the layer output of {rows} token row(s)")
    else:
        sample = (f"each step: fp64 routing, dispatch and statistics of the whole T={wl.T} batch; "
                  f"one step in {every} also the layer output of {rows} token row(s)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(wl), "global_batch": wl.T, "tokens_per_step": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": O.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    wl = WORKLOADS[args.workload]
    if args.hidden:
        wl = wl.scaled(h=args.hidden, name=f"{wl.name}_h{args.hidden}")
    if args.overflow:
        wl = wl.scaled(overflow=args.overflow)
    if args.backward and world > 1:
        raise SystemExit("--backward runs on one GPU")
    B.moe_set_pdl(not args.no_pdl)
    B.moe_set_pair_tiles(args.pair)
    B.moe_set_shared_overlap(not args.no_overlap)
    if args.shared_sms >= 0:
        B.moe_set_shared_sms(args.shared_sms)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline and not args.backward
    cfg, host, g, W, Wb = build_inputs(wl, rank, world, dev, keep_host=want_cpu,
                                       train=args.backward, hidden=args.hidden_mode)
    W13, W2p, W13s, W2s = W
    W13t, W2t, W13st, W2st = Wb
    bufs = B.alloc_layer(cfg, dev)
    grads = B.alloc_grads(cfg, dev) if args.backward else None
    sums = torch.zeros(dp.sums_len(wl.E), dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def layer(x, out, stats, G=None, dx=None):
        """One step of the public API on the given input and output buffers."""
        if world == 1:
            B.moe_forward(cfg, x, g["Wr"], g["bias"], W13, W2p, W13s, W2s, out,
                          bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                          bufs["slot_of"], stats, bufs["ws"])
            if args.backward:
                gr = dict(grads)
                gr["dx"] = dx
                B.backward(cfg, G, AUX_COEF, x, g["Wr"], g["bias"], W13t, W2t, W13st, W2st, bufs,
                           gr)
        else:
            B.moe_forward(cfg, x, g["Wr"], g["bias"], W13, W2p, W13s, W2s, out,
                          bufs["topk_idx"], bufs["topk_gate"], bufs["routed"], bufs["kept"],
                          bufs["slot_of"], None, bufs["ws"])
            dp.global_stats(cfg, bufs["routed"], bufs["kept"], bufs["ws"], sums, stats)

    def step():
        layer(g["x"], bufs["out"], bufs["stats"], g.get("G"),
              grads["dx"] if args.backward else None)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    c0 = B.moe_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = B.moe_launch_count() - c0
    status = B.moe_read_device_status(bufs["ws"])
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")

    graph = None
    if args.graph and world == 1:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
            torch.cuda.synchronize()
            with torch.cuda.graph(graph, stream=side):
                step()
        torch.cuda.synchronize()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    run = graph.replay if graph is not None else step
    trace_on = not args.no_trace and graph is None
    calls = 2 if args.backward else 1  # library calls per step that launch kernels

    # ------------------------------------------------ timed region (device resident)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if trace_on:
        # bracket only the dominant kernel (the one the roofline is quoted on)
        only = None if (args.trace_all or args.backward) else "gemm_gateup"
        B.moe_trace_begin(args.steps * calls, only)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    n0 = B.moe_launch_count()
    ev0.record(stream)
    for _ in range(args.steps):
        run()
    ev1.record(stream)
    torch.cuda.synchronize()
    # kernels launched in the timed region (a replayed graph launches its captured step)
    launched = (B.moe_launch_count() - n0) if graph is None else launches_per_step * args.steps
    if dist:
        dist.barrier()
    clk = clocks.stop()
    trace = B.moe_trace_end() if trace_on else []
    ms = ev0.elapsed_time(ev1)
    ms_t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if dist:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    status = B.moe_read_device_status(bufs["ws"])

    # ------------------------------------------------ end to end (host buffers, copies timed)
    # Every step copies its batch in from pinned host memory and its output and
    # statistics (and, training, dx) back, all inside the timed region.  The
    # copies run on their own streams with two sets of device buffers, so step
    # i + 1's input travels while step i computes and step i's output travels
    # while step i + 1 computes -- the pipelining a user of the API would do.
    e2e = None
    if not args.no_e2e:
        NB = 2
        xs = [g["x"], torch.empty_like(g["x"])]
        outs = [bufs["out"], torch.empty_like(bufs["out"])]
        sts = [bufs["stats"], torch.zeros_like(bufs["stats"])]
        x_h = g["x"].cpu().pin_memory()
        out_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        st_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in sts]
        Gs = dxs = G_h = dx_h = None
        if args.backward:
            Gs = [g["G"], torch.empty_like(g["G"])]
            dxs = [grads["dx"], torch.empty_like(grads["dx"])]
            G_h = g["G"].cpu().pin_memory()
            dx_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dxs]
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(NB)]    # input of the buffer copied in
        ev_done = [torch.cuda.Event() for _ in range(NB)]  # compute done with the buffer
        ev_out = [torch.cuda.Event() for _ in range(NB)]   # output of the buffer copied out

        def issue_input(i, start=None):
            b = i % NB
            with torch.cuda.stream(cin):
                if start is not None:
                    cin.wait_event(start)
                cin.wait_event(ev_done[b])   # step i - 2 no longer reads this buffer
                xs[b].copy_(x_h, non_blocking=True)
                if args.backward:
                    Gs[b].copy_(G_h, non_blocking=True)
                ev_in[b].record(cin)

        def run(i):
            b = i % NB
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])     # step i - 2's output has left this buffer
            layer(xs[b], outs[b], sts[b], Gs[b] if Gs else None, dxs[b] if dxs else None)
            ev_done[b].record(stream)
            with torch.cuda.stream(cout):
                cout.wait_event(ev_done[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                st_h[b].copy_(sts[b], non_blocking=True)
                if args.backward:
                    dx_h[b].copy_(dxs[b], non_blocking=True)
                ev_out[b].record(cout)

        def e2e_steps(n, start=None):
            issue_input(0, start)
            for i in range(n):
                if i + 1 < n:
                    issue_input(i + 1)
                run(i)
            stream.wait_event(ev_out[(n - 1) % NB])

        e2e_steps(3)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_steps(args.steps, start=e0)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if dist:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        h2d = x_h.numel() * x_h.element_size()
        d2h = out_h[0].numel() * out_h[0].element_size() + st_h[0].numel() * st_h[0].element_size()
        if args.backward:
            h2d += G_h.numel() * G_h.element_size()
            d2h += dx_h[0].numel() * dx_h[0].element_size()
        e2e = {"value": world * wl.T * args.steps / (float(e_ms.item()) / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "input of step i+1 and output of step i copied while step i computes"}

    # ------------------------------------------------ report
    kept = bufs["kept"].cpu().tolist()
    stats = B.stats_dict(bufs["stats"])
    pk, pk_kind = peaks()
    flops, byts, N, active = algorithmic(wl, kept)
    if args.backward:
        bf, bb = backward_algorithmic(wl, kept)
        flops, byts = flops + bf, byts + bb
    t_step = ms_max / 1000.0 / args.steps
    roof_t = max(flops / (pk["bf16_tflops"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    kernels = {n: {"launches": c, "ms_per_launch": t / c} for n, c, t in trace}
    roofline = dominant_roofline(trace, wl, cfg, kept)
    line = {
        "metric": METRIC if not args.backward else METRIC + ", training step (forward + backward)",
        "value": world * wl.T * args.steps / (ms_max / 1000.0),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic",
        "config": {"workload": workload_label(wl), "global_batch": world * wl.T,
                   "tokens_per_rank": wl.T,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "hidden": "split" if B.moe_hidden_split(cfg) else "bf16",
                   **({"shared_sms": args.shared_sms}
                      if wl.n_shared and args.shared_sms >= 0 else {}),
                   "l2": ("inputs larger than L2: the active expert weights "
                          f"({active * 3 * wl.d * wl.h * 2 / 1e9:.2f} GB) stream from HBM "
                          "every step")},
        "roofline": roofline,
        "layer_roofline": {"flops": flops, "bytes": byts, "time_us": roof_t * 1e6,
                           "frac": roof_t / t_step, "kept_assignments": N,
                           "active_experts": active, "peaks": "bf16 burst, HBM copy"},
        "tiles": tile_stats(wl, kept, torch.cuda.get_device_properties(dev).multi_processor_count),
        "kernels": kernels,
        "gpu_launches": launched,
        "clocks": clk,
        "e2e": e2e,
        "stats": stats,
        "device_status": status,
    }
    if want_cpu:
        line["cpu_baseline"] = time_oracle(wl, host, args.cpu_seconds)
    if (world == 1 and not args.backward and not args.no_decode and wl.name != "decode"
            and not args.graph and not args.hidden):
        line["decode"] = decode_line(args, dev, stream, wl, W)
    if (world == 1 and not args.backward and not args.no_split_line and not args.graph
            and not B.moe_hidden_split(cfg) and wl.dtype == "bf16"):
        line["split_hidden"] = split_line(args, dev, stream, wl, g, W)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

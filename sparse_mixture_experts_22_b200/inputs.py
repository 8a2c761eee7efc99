"""Seeded synthetic inputs for the MoE layer, shared by the oracle tests, the GPU
parity tests and the benchmark.

This module draws random tensors and nothing else of the layer's arithmetic.
The one computation it does is the input-validity filter that keeps routing
well defined: a token whose k-th and (k+1)-th router logits (fp64, from the
rounded inputs) differ by less than 1e-4 is redrawn, so that an fp32 router and
an fp64 one must pick the same expert set.  The filter uses a library matmul and
sort; the layer's own routing lives in the oracle and in the CUDA library.

Recipe (every tensor from its own torch CPU generator, seeded from the workload
seed and the tensor's name, so any tensor can be regenerated alone):

  x      ~ N(0, 1)            [T, d]      rounded to the workload dtype
  W_r    ~ N(0, 1/d)          [d, E]      fp32 (router weights, z = x @ W_r + b)
  b_e    = -s * ln(e + 1)     [E]         fp32, only for Zipf(s) workloads
  w1, w3 ~ N(0, 1/d)          [E, d, h]   gate and up projections
  w2     ~ N(0, 1/h)          [E, h, d]   down projection
  shared experts: w1s, w3s [S, d, hs] ~ N(0, 1/d); w2s [S, hs, d] ~ N(0, 1/hs)
  G      ~ N(0, 1)            [T, d]      gradient of the loss w.r.t. the layer
                                          output (backward pass), workload dtype
"""

import hashlib
import math
from typing import Dict, Optional

import torch

from .workloads import Workload

TIE_GAP = 1e-4


def _seed(base: int, name: str) -> int:
    h = hashlib.sha256(f"{base}:{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(base: int, name: str) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(_seed(base, name))


def torch_dtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def normal(shape, std: float, gen: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded (round-to-nearest-even) to dtype."""
    return (torch.randn(*shape, generator=gen) * std).to(dtype)


def zipf_bias(E: int, s: float) -> torch.Tensor:
    """Router bias whose softmax is the Zipf(s) pmf over experts 0..E-1.

    ln of the pmf is -s*ln(e+1) - ln(H_{E,s}); the constant cancels in both the
    top-k choice and every softmax, so it is left out.  Expert 0 is the most
    popular.
    """
    return torch.tensor([-s * math.log(e + 1) for e in range(E)], dtype=torch.float32)


def router_weights(wl: Workload) -> torch.Tensor:
    return normal((wl.d, wl.E), 1.0 / math.sqrt(wl.d), generator(wl.seed, "W_r"),
                  torch.float32)


def router_bias(wl: Workload) -> Optional[torch.Tensor]:
    return zipf_bias(wl.E, wl.zipf_s) if wl.zipf_s is not None else None


def _near_tie_rows(x: torch.Tensor, Wr: torch.Tensor, b: Optional[torch.Tensor],
                   k: int, all_gaps: bool = False) -> torch.Tensor:
    """Indices of rows whose k-th and (k+1)-th largest fp64 logits are < TIE_GAP
    apart (with all_gaps: any two neighbouring logits in sorted order)."""
    E = Wr.shape[1]
    if (k >= E and not all_gaps) or x.shape[0] == 0 or E < 2:
        return torch.zeros(0, dtype=torch.long)
    z = x.double() @ Wr.double()
    if b is not None:
        z = z + b.double()
    if all_gaps:
        srt = torch.sort(z, dim=1, descending=True).values
        gap = (srt[:, :-1] - srt[:, 1:]).min(dim=1).values
    else:
        top = torch.topk(z, k + 1, dim=1).values
        gap = top[:, k - 1] - top[:, k]
    return torch.nonzero(gap < TIE_GAP).flatten()


def tokens(wl: Workload, T: Optional[int] = None, Wr: Optional[torch.Tensor] = None,
           b: Optional[torch.Tensor] = None, stream: str = "x") -> (torch.Tensor, int):
    """x [T, d] in the workload dtype, with near-tie rows redrawn.

    Under the reroute policy a spare expert is chosen among all experts, so
    there every pair of neighbouring sorted logits is kept TIE_GAP apart.
    Returns (x, number of rows redrawn).  Redrawn rows come from the same
    generator stream, continuing, so the result is a pure function of the seed.
    """
    T = wl.T if T is None else T
    dt = torch_dtype(wl.dtype)
    g = generator(wl.seed, stream)
    x = normal((T, wl.d), 1.0, g, dt)
    if Wr is None:
        Wr = router_weights(wl)
    if b is None:
        b = router_bias(wl)
    redrawn = 0
    for _ in range(1000):
        bad = _near_tie_rows(x, Wr, b, wl.k, all_gaps=wl.overflow == "reroute")
        if bad.numel() == 0:
            return x, redrawn
        redrawn += bad.numel()
        x[bad] = normal((bad.numel(), wl.d), 1.0, g, dt)
    raise RuntimeError("near-tie resampling did not converge")


def expert_weights(wl: Workload, shared: bool = False) -> Dict[str, torch.Tensor]:
    """w1, w3 [n, d, h] and w2 [n, h, d] for the routed (or shared) experts.

    Each expert's matrices come from their own generator so that a subset of
    experts can be regenerated without drawing the rest.
    """
    dt = torch_dtype(wl.dtype)
    if shared:
        n, h, tag = wl.n_shared, wl.h_shared, "shared"
    else:
        n, h, tag = wl.E, wl.h, "expert"
    d = wl.d
    w1 = torch.empty((n, d, h), dtype=dt)
    w3 = torch.empty((n, d, h), dtype=dt)
    w2 = torch.empty((n, h, d), dtype=dt)
    for e in range(n):
        w1[e] = normal((d, h), 1.0 / math.sqrt(d), generator(wl.seed, f"{tag}{e}.w1"), dt)
        w3[e] = normal((d, h), 1.0 / math.sqrt(d), generator(wl.seed, f"{tag}{e}.w3"), dt)
        w2[e] = normal((h, d), 1.0 / math.sqrt(h), generator(wl.seed, f"{tag}{e}.w2"), dt)
    return {"w1": w1, "w3": w3, "w2": w2}


def layer_inputs(wl: Workload, T: Optional[int] = None, weights: bool = True) -> Dict:
    """Every input of one layer call, on the host."""
    Wr = router_weights(wl)
    b = router_bias(wl)
    x, redrawn = tokens(wl, T, Wr, b)
    out = {"x": x, "Wr": Wr, "bias": b, "redrawn": redrawn}
    if weights:
        out.update(expert_weights(wl))
        if wl.n_shared:
            s = expert_weights(wl, shared=True)
            out.update({"w1s": s["w1"], "w3s": s["w3"], "w2s": s["w2"]})
    return out


def grad_out(wl: Workload, T: Optional[int] = None) -> torch.Tensor:
    """G = dL/dout [T, d] for the backward pass, in the workload dtype."""
    T = wl.T if T is None else T
    return normal((T, wl.d), 1.0, generator(wl.seed, "grad_out"), torch_dtype(wl.dtype))

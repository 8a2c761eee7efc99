"""The five synthetic MoE-layer workloads and their sizes.

Shapes follow the layer the pages describe: an FFN that widens a ~4k embedding
to a ~14k hidden size and back ("Mixtral 8x7B and MoE explained", section
"Easy explanation" ¶2), 8 experts with 2 active per token (same page, ¶3), and a
DeepSeek-V2-style layer with 2 shared experts plus many routed experts, top-6
("MoE routing fully explained", section "Easy explanation" ¶4).  The capacity
factors 1.25 and 1.5 are the range that page gives (¶5).

This module holds sizes only; no arithmetic of the method lives here.
"""

from dataclasses import dataclass
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                      # tokens in the batch
    d: int                      # model (embedding) width
    h: int                      # routed-expert hidden width
    E: int                      # routed experts
    k: int                      # experts kept per token
    n_shared: int = 0           # shared experts applied to every token
    h_shared: int = 0           # hidden width of each shared expert
    cf: Optional[Tuple[int, int]] = None   # capacity factor num/den; None = no limit
    dtype: str = "bf16"         # "bf16" or "f32" for activations and expert weights
    zipf_s: Optional[float] = None         # router bias b_e = -s*ln(e+1) when set
    overflow: str = "drop"                 # "drop" or "reroute" (to a spare expert)
    seed: int = 0

    @property
    def has_bias(self) -> bool:
        return self.zipf_s is not None

    def describe(self) -> str:
        cf = "inf" if self.cf is None else f"{self.cf[0]}/{self.cf[1]}"
        s = (f"T={self.T} d={self.d} h={self.h} E={self.E} k={self.k} cf={cf} "
             f"{self.dtype}")
        if self.n_shared:
            s += f" shared={self.n_shared}x{self.h_shared}"
        if self.zipf_s is not None:
            s += f" zipf={self.zipf_s}"
        if self.overflow != "drop":
            s += f" overflow={self.overflow}"
        return s

    def scaled(self, **kw) -> "Workload":
        fields = dict(self.__dict__)
        fields.update(kw)
        return Workload(**fields)


WORKLOADS = {
    # tiny layer, fp32 throughout, no capacity limit
    "tiny": Workload("tiny", T=64, d=128, h=256, E=8, k=2, dtype="f32"),
    # Mixtral-shaped decode batch: weight streaming, HBM-bound
    "decode": Workload("decode", T=32, d=4096, h=14336, E=8, k=2),
    # Mixtral-shaped prefill batch, cf 1.25 (C = 640), Zipf(1.0) router bias
    "prefill": Workload("prefill", T=2048, d=4096, h=14336, E=8, k=2, cf=(5, 4),
                        zipf_s=1.0),
    # DeepSeek-V2-style: 2 shared + 160 routed experts, top-6, cf 1.5 (C = 231)
    "deepseek": Workload("deepseek", T=4096, d=5120, h=1536, E=160, k=6, n_shared=2,
                         h_shared=1536, cf=(3, 2)),
    # large skewed prefill with statistics, cf 1.5 (C = 6144), Zipf(1.2) bias
    "large": Workload("large", T=16384, d=4096, h=14336, E=8, k=2, cf=(3, 2),
                      zipf_s=1.2),
}

ORDER = ["tiny", "decode", "prefill", "deepseek", "large"]

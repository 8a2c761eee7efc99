"""Data-parallel plumbing of the layer: one process per GPU, each running the
whole layer on its own batch (weights replicated), with the routing
statistics made global by summing their additive parts across ranks.

The statistics of the load-balancing loss are ratios of sums (counts, summed
router probabilities, summed token entropies), so the global values follow
from the element-wise sum of each rank's `sums` vector [T, entropy sum,
P sums (E), routed (E), kept (E)] -- the one exchange of the data-parallel
path, a (2 + 3E)-double all-reduce per step.  With a finite capacity factor
each rank applies the capacity rule to its own batch.
"""

from typing import List, Optional

import torch

from . import binding as B


def token_stream(rank: int) -> str:
    """Name of the seeded token stream of a rank (rank 0 draws the base batch)."""
    return "x" if rank == 0 else f"x.rank{rank}"


def sums_len(E: int) -> int:
    return 2 + 3 * E


def allreduce_sums(sums: torch.Tensor, group=None) -> torch.Tensor:
    """Element-wise sum of every rank's statistics sums, in place."""
    import torch.distributed as dist
    dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return sums


def broadcast_weights(tensors: List[Optional[torch.Tensor]], src: int = 0, group=None):
    """Replicates the packed expert weights from `src` to every rank."""
    import torch.distributed as dist
    for t in tensors:
        if t is not None:
            dist.broadcast(t, src=src, group=group)


def global_stats(cfg, routed, kept, ws, sums, stats, group=None, stream=None):
    """This rank's sums, summed over ranks, then the statistics (on the GPU)."""
    B.moe_stats_sums(cfg, routed, kept, ws, sums, stream)
    allreduce_sums(sums, group)
    B.moe_stats_finalize(cfg, sums, stats, stream)

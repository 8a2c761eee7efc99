"""Expert parallelism: the layer with its routed experts partitioned over G ranks.

The pages' own multi-GPU story [Mixtral 8x7B and MoE explained, "Easy
explanation" ¶4: the experts can be spread over GPUs; MoE routing fully
explained, "Easy explanation" ¶3: tokens travel to the GPU that holds their
expert, and the busiest expert sets the step time].  Rank r holds the experts
r*E/G .. (r+1)*E/G - 1 and its own batch of tokens; the router weights are
replicated.

Reading taken: G ranks compute exactly the single-GPU layer on the
concatenation of their batches (rank 0's tokens first).  The capacity is
C = ceil(T_all k cf / E) over the whole concatenation, and an expert's queue
fills in that arrival order: rank r may keep, for expert e, at most
cap[r][e] = C - (assignments to e on lower ranks).  One step:

  1. every rank routes its tokens (moe_route) and reads its per-expert counts
     (moe_route_counts); the counts are all-gathered (G x E int32);
  2. every rank computes the same plan from the counts (`make_plan`) and
     dispatches under its caps (moe_dispatch_capped): its x_perm holds one
     padded segment per expert, the segments of each destination contiguous;
  3. all-to-all of the segment rows: rank r receives, from every source, the
     rows of its own experts;
  4. the owner runs the expert FFN on the (source, expert) groups it received
     (moe_expert_ffn_grouped, fp32 rows out);
  5. all-to-all back (the reverse splits): the output rows land where their
     input rows were in the source's x_perm;
  6. moe_combine_rows forms the outputs with the gates; the statistics are
     summed across ranks as in data parallelism.

The exchanges are torch.distributed collectives (NCCL between GPUs, gloo on
the host in the tests) or, for one process standing in for G ranks on one
GPU, plain copies (`forward_emulated`).  Only the routed experts are
partitioned; the overflow policy is drop.

The peer-memory form folds steps 3 and 5 into the kernels next to them:
moe_dispatch_peers stores every kept row straight into its owner's receive
buffer (NVLink stores from the SMs that gather it), and moe_combine_peers
loads every output row straight from its owner's buffer; no staging copy and
no collective carries the rows.  Rank s's rows start at row
`peer_row_starts(plan, s)[q]` of rank q's buffers, after the rows of the lower
ranks -- the layout the all-to-all produces.  Between the phases the ranks
pass a stream-ordered barrier (the owners read only after every source has
stored; the buffers are reused only after every source has combined):
`forward_dist_peers` takes the buffers from torch's symmetric memory, and
`forward_emulated_peers` runs the ranks' kernels one after another on one GPU.

In the peer-memory form the plan can stay on the device (`device_plan=True`,
the default of `forward_dist_peers`): the counts are gathered into a device
tensor, moe_ep_plan derives every rank's caps, row offsets and received
groups from them on the GPU, and the kernels take those offsets from device
memory, so a step never waits for the host.  The collective form keeps the
host plan: NCCL's all-to-all takes its split sizes on the host.

`StepTimer` measures the share of a step spent in the inter-GPU dispatch
[MoE routing fully explained, "Main insights" ¶3: the dispatch time share is
one of the routing metrics to watch]: CUDA events around the exchange phases
(with their barriers), against the whole step.
"""

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

from . import binding as B


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def capacity(T_all: int, k: int, E: int, cf) -> int:
    """C = ceil(T_all k cf / E) in integers; no limit (cf None) -> T_all."""
    if cf is None:
        return T_all
    num, den = cf
    return ceil_div(T_all * k * num, E * den)


@dataclass
class Plan:
    """The host-side plan of one step, identical on every rank."""
    G: int
    E: int
    E_loc: int
    C: int
    pad: int
    counts: np.ndarray            # [G][E] routed assignments, before the capacity
    cap: np.ndarray = field(init=False)    # [G][E] per-rank capacity of each expert
    kept: np.ndarray = field(init=False)   # [G][E] rows each rank keeps for each expert
    seg: np.ndarray = field(init=False)    # [G][E] padded segment rows in the sender's x_perm
    send: np.ndarray = field(init=False)   # [G][G] rows rank r sends to rank q

    def __post_init__(self):
        c = self.counts.astype(np.int64)
        base = np.cumsum(c, axis=0) - c          # assignments to e on lower ranks
        self.cap = np.clip(self.C - base, 0, None)
        self.kept = np.minimum(c, self.cap)
        self.seg = ceil_div_arr(self.kept, self.pad) * self.pad
        self.send = self.seg.reshape(self.G, self.G, self.E_loc).sum(axis=2)

    def owner(self, e: int) -> int:
        return e // self.E_loc

    def recv_rows(self, rank: int) -> np.ndarray:
        """Rows rank `rank` receives from each source."""
        return self.send[:, rank]

    def groups(self, rank: int):
        """(rows, first row, weight index) of every (source, local expert)
        group in rank `rank`'s receive buffer, sources in order, then experts."""
        rows, off, wi = [], [], []
        at = 0
        for src in range(self.G):
            for el in range(self.E_loc):
                e = rank * self.E_loc + el
                rows.append(int(self.kept[src, e]))
                off.append(at)
                wi.append(el)
                at += int(self.seg[src, e])
        return np.array(rows, np.int32), np.array(off, np.int32), np.array(wi, np.int32)


def ceil_div_arr(a: np.ndarray, b: int) -> np.ndarray:
    return -(-a // b)


def make_plan(counts: np.ndarray, T_all: int, k: int, E: int, cf, pad: int) -> Plan:
    G = counts.shape[0]
    if E % G:
        raise ValueError("E must be a multiple of the number of ranks")
    return Plan(G=G, E=E, E_loc=E // G, C=capacity(T_all, k, E, cf), pad=pad,
                counts=np.asarray(counts, np.int64))


# ---------------------------------------------------------------- exchanges

def send_splits(plan: Plan, rank: int) -> List[int]:
    return [int(v) for v in plan.send[rank]]


def recv_splits(plan: Plan, rank: int) -> List[int]:
    return [int(v) for v in plan.recv_rows(rank)]


def exchange_rows(send: torch.Tensor, plan: Plan, rank: int, group=None) -> torch.Tensor:
    """Step 3: rank `rank` sends its x_perm segments to their experts' owners
    and receives its experts' rows from every source (source order)."""
    import torch.distributed as dist
    rs = recv_splits(plan, rank)
    recv = torch.empty((sum(rs),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(recv, send[:sum(send_splits(plan, rank))].contiguous(), rs,
                           send_splits(plan, rank), group=group)
    return recv


def exchange_back(y: torch.Tensor, plan: Plan, rank: int, group=None) -> torch.Tensor:
    """Step 5: the owner returns the output rows; they land where the input
    rows were in each source's x_perm."""
    import torch.distributed as dist
    ss = send_splits(plan, rank)
    back = torch.empty((sum(ss),) + tuple(y.shape[1:]), dtype=y.dtype, device=y.device)
    dist.all_to_all_single(back, y.contiguous(), ss, recv_splits(plan, rank), group=group)
    return back


def peer_row_starts(plan: Plan, rank: int) -> np.ndarray:
    """[G] first row of rank `rank`'s rows in each rank's receive (and
    output) buffer: the rows every lower rank sends there come first."""
    return plan.send[:rank].sum(axis=0).astype(np.int64)


def device_plan(r: "Rank", counts_all: torch.Tensor, C: int) -> dict:
    """The plan of rank r on the device (moe_ep_plan) from the gathered
    counts [G * E] (device int32); nothing is read back to the host."""
    G, E = r.world, r.wl.E
    dev = counts_all.device
    i32 = dict(dtype=torch.int32, device=dev)
    p = {"cap": torch.empty(E, **i32), "row_start": torch.empty(G, **i32),
         "group_rows": torch.empty(E, **i32), "group_off": torch.empty(E, **i32),
         "group_weight": torch.empty(E, **i32), "recv_rows": torch.empty(1, **i32)}
    B.moe_ep_plan(r.cfg, G, r.rank, counts_all, C, p["cap"], p["row_start"], p["group_rows"],
                  p["group_off"], p["group_weight"], p["recv_rows"])
    return p


class StepTimer:
    """CUDA events around the phases of one expert-parallel step; `share()`
    is the fraction of the step spent dispatching rows to their experts'
    owners and bringing the outputs back (the exchanges and their barriers)."""

    def __init__(self):
        self.ev = {}

    def mark(self, name: str):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.ev[name] = e

    def ms(self, a: str, b: str) -> float:
        return self.ev[a].elapsed_time(self.ev[b])

    def share(self) -> dict:
        torch.cuda.synchronize()
        step = self.ms("start", "end")
        xch = self.ms("dispatch0", "dispatch1") + self.ms("combine0", "combine1")
        return {"step_ms": step, "exchange_ms": xch, "dispatch_share": xch / step if step else 0.0}


def _mark(timer: Optional["StepTimer"], name: str):
    if timer is not None:
        timer.mark(name)


def all_gather_counts(counts: torch.Tensor, world: int, group=None) -> np.ndarray:
    """Step 1's exchange: every rank's per-expert counts, [G][E]."""
    import torch.distributed as dist
    parts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts).cpu().numpy().astype(np.int64)


# ---------------------------------------------------------------- one rank

class Rank:
    """One rank's layer state: its batch, the replicated router, its experts'
    packed weights, and the buffers of one step."""

    def __init__(self, wl, rank: int, world: int, x, Wr, bias, W13_loc, W2p_loc):
        if wl.E % world:
            raise ValueError("E must be a multiple of the number of ranks")
        if wl.n_shared or wl.overflow != "drop" or wl.dtype != "bf16":
            raise ValueError("expert parallelism: bf16, routed experts, drop policy")
        self.wl, self.rank, self.world = wl, rank, world
        T = x.shape[0]
        dev = x.device
        # locally no capacity limit: the global one arrives as per-expert caps
        self.cfg = B.make_config(T, wl.d, wl.h, wl.E, wl.k, dtype=wl.dtype,
                                 has_bias=wl.has_bias)
        self.x, self.Wr, self.bias = x, Wr, bias
        self.W13, self.W2p = W13_loc, W2p_loc
        self.pad = B.moe_segment_pad(self.cfg)
        self.symm = None  # peer-memory form: (recv, y, their symmetric-memory handles)
        rows = max(B.moe_perm_rows(self.cfg), 1)
        i32 = dict(dtype=torch.int32, device=dev)
        self.b = {
            "topk_idx": torch.empty((T, wl.k), **i32),
            "topk_gate": torch.empty((T, wl.k), dtype=torch.float32, device=dev),
            "counts": torch.empty(wl.E, **i32),
            "routed": torch.empty(wl.E, **i32),
            "kept": torch.empty(wl.E, **i32),
            "offsets": torch.empty(wl.E + 1, **i32),
            "perm_token": torch.empty(rows, **i32),
            "slot_of": torch.empty((T, wl.k), **i32),
            "x_perm": torch.empty((rows, wl.d), dtype=x.dtype, device=dev),
            "out": torch.empty((T, wl.d), dtype=x.dtype, device=dev),
            "sums": torch.zeros(2 + 3 * wl.E, dtype=torch.float64, device=dev),
            "ws": torch.empty(max(B.moe_workspace_size(self.cfg), 256), dtype=torch.uint8,
                              device=dev),
        }

    def route(self) -> torch.Tensor:
        b = self.b
        B.moe_route(self.cfg, self.x, self.Wr, self.bias if self.wl.has_bias else None,
                    b["topk_idx"], b["topk_gate"], b["ws"])
        B.moe_route_counts(self.cfg, b["ws"], b["counts"])
        return b["counts"]

    def dispatch(self, plan: Plan) -> torch.Tensor:
        b = self.b
        cap = torch.tensor(plan.cap[self.rank].clip(max=2 ** 31 - 1), dtype=torch.int32,
                           device=self.x.device)
        B.moe_dispatch_capped(self.cfg, b["topk_idx"], self.x, cap, b["routed"], b["kept"],
                              b["offsets"], b["perm_token"], b["slot_of"], b["x_perm"], b["ws"])
        return b["x_perm"][:int(plan.seg[self.rank].sum())]

    def ffn(self, plan: Plan, recv: torch.Tensor, y: Optional[torch.Tensor] = None,
            bound: Optional[int] = None) -> torch.Tensor:
        """Step 4 on the host plan's groups; `bound` (default: the largest group)
        is the bound on a group's rows that picks the GEMM layout."""
        rows, off, wi = plan.groups(self.rank)
        dev = self.x.device
        if y is None:
            y = torch.empty((recv.shape[0], self.wl.d), dtype=torch.float32, device=dev)
        if recv.shape[0] == 0:
            return y
        mx = bound if bound is not None else (int(rows.max()) if rows.size else 0)
        ws = torch.empty(B.moe_grouped_workspace_size(self.cfg, recv.shape[0], mx),
                         dtype=torch.uint8, device=dev)
        B.moe_expert_ffn_grouped(self.cfg, recv, recv.shape[0], torch.from_numpy(rows).to(dev),
                                 torch.from_numpy(off).to(dev), torch.from_numpy(wi).to(dev), mx,
                                 self.W13, self.W2p, y, ws)
        self.ffn_ws = ws
        return y

    def dispatch_peers_dev(self, dplan: dict, recv_bases: List[int]) -> None:
        """Step 2 with step 3 folded in, the plan on the device: this rank's
        rows start at row dplan["row_start"][q] of rank q's receive buffer."""
        b = self.b
        B.moe_dispatch_peers(self.cfg, b["topk_idx"], self.x, dplan["cap"],
                             [int(p) for p in recv_bases], b["routed"], b["kept"], b["offsets"],
                             b["perm_token"], b["slot_of"], b["ws"],
                             dst_row_start=dplan["row_start"])

    def ffn_dev(self, dplan: dict, recv: torch.Tensor, y: torch.Tensor, bound: int) -> None:
        """Step 4 with the received groups described on the device; `bound`
        (host) bounds every group's rows."""
        if recv.shape[0] == 0:
            return
        ws = getattr(self, "ffn_ws_dev", None)
        need = B.moe_grouped_workspace_size(self.cfg, recv.shape[0], bound)
        if ws is None or ws.numel() < need:
            ws = torch.empty(need, dtype=torch.uint8, device=recv.device)
            self.ffn_ws_dev = ws
        B.moe_expert_ffn_grouped(self.cfg, recv, recv.shape[0], dplan["group_rows"],
                                 dplan["group_off"], dplan["group_weight"], bound, self.W13,
                                 self.W2p, y, ws)

    def combine_peers_dev(self, dplan: dict, y_bases: List[int]) -> torch.Tensor:
        b = self.b
        B.moe_combine_peers(self.cfg, [int(p) for p in y_bases], b["topk_idx"], b["offsets"],
                            b["slot_of"], b["topk_gate"], None, b["out"],
                            y_row_start=dplan["row_start"])
        return b["out"]

    def dispatch_peers(self, plan: Plan, recv_bases: List[int]) -> None:
        """Step 2 with step 3 folded in: recv_bases[q] = device address of
        rank q's receive buffer (bf16 [rows][d])."""
        b = self.b
        cap = torch.tensor(plan.cap[self.rank].clip(max=2 ** 31 - 1), dtype=torch.int32,
                           device=self.x.device)
        row_bytes = self.wl.d * self.x.element_size()
        starts = peer_row_starts(plan, self.rank)
        dst = [int(recv_bases[q]) + int(starts[q]) * row_bytes for q in range(self.world)]
        B.moe_dispatch_peers(self.cfg, b["topk_idx"], self.x, cap, dst, b["routed"], b["kept"],
                             b["offsets"], b["perm_token"], b["slot_of"], b["ws"])

    def combine_peers(self, plan: Plan, y_bases: List[int]) -> torch.Tensor:
        """Steps 5 and 6: y_bases[q] = device address of rank q's fp32 output
        rows [rows][d]."""
        b = self.b
        starts = peer_row_starts(plan, self.rank)
        src = [int(y_bases[q]) + int(starts[q]) * self.wl.d * 4 for q in range(self.world)]
        B.moe_combine_peers(self.cfg, src, b["topk_idx"], b["offsets"], b["slot_of"],
                            b["topk_gate"], None, b["out"])
        return b["out"]

    def combine(self, y_back: torch.Tensor) -> torch.Tensor:
        b = self.b
        B.moe_combine_rows(self.cfg, y_back, b["slot_of"], b["topk_gate"], None, b["out"])
        return b["out"]

    def stats_sums(self) -> torch.Tensor:
        b = self.b
        B.moe_stats_sums(self.cfg, b["routed"], b["kept"], b["ws"], b["sums"])
        return b["sums"]


# ---------------------------------------------------------------- drivers

def forward_dist(r: Rank, T_all: int, group=None, timer: Optional[StepTimer] = None):
    """One step on this rank, the exchanges as torch.distributed collectives.
    Returns (out, stats tensor, plan)."""
    _mark(timer, "start")
    counts = all_gather_counts(r.route(), r.world, group)
    plan = make_plan(counts, T_all, r.wl.k, r.wl.E, r.wl.cf, r.pad)
    send = r.dispatch(plan)
    _mark(timer, "dispatch0")
    recv = exchange_rows(send, plan, r.rank, group)
    _mark(timer, "dispatch1")
    y = r.ffn(plan, recv)
    _mark(timer, "combine0")
    back = exchange_back(y, plan, r.rank, group)
    _mark(timer, "combine1")
    out = r.combine(back)
    import torch.distributed as dist
    sums = r.stats_sums()
    dist.all_reduce(sums, group=group)
    stats = torch.zeros(5, dtype=torch.float64, device=sums.device)
    B.moe_stats_finalize(r.cfg, sums, stats)
    _mark(timer, "end")
    return out, stats, plan


def forward_emulated(ranks: List[Rank], T_all: int):
    """G ranks in one process on one device: the same phases, rank by rank,
    with the exchanges done as copies (no kernel waits on another).  Returns
    ([out per rank], stats tensor, plan)."""
    G = len(ranks)
    counts = np.stack([r.route().cpu().numpy() for r in ranks]).astype(np.int64)
    wl = ranks[0].wl
    plan = make_plan(counts, T_all, wl.k, wl.E, wl.cf, ranks[0].pad)
    sends = [r.dispatch(plan) for r in ranks]
    starts = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(plan.send, axis=1)], axis=1)
    recvs = [torch.cat([sends[s][starts[s, q]:starts[s, q + 1]] for s in range(G)])
             for q in range(G)]
    ys = [ranks[q].ffn(plan, recvs[q]) for q in range(G)]
    rstarts = [np.concatenate([[0], np.cumsum(plan.recv_rows(q))]) for q in range(G)]
    backs = [torch.cat([ys[q][rstarts[q][s]:rstarts[q][s + 1]] for q in range(G)])
             for s in range(G)]
    outs = [ranks[s].combine(backs[s]) for s in range(G)]
    sums = sum(r.stats_sums().clone() for r in ranks)
    stats = torch.zeros(5, dtype=torch.float64, device=sums.device)
    B.moe_stats_finalize(ranks[0].cfg, sums, stats)
    return outs, stats, plan


def forward_emulated_peers(ranks: List[Rank], T_all: int, bound: Optional[int] = None):
    """The peer-memory form with G ranks in one process on one device: every
    rank's receive and output buffers live on that device, and the ranks'
    kernels run one after another in stream order (which stands in for the
    barriers).  `bound`: as Rank.ffn.  Returns ([out per rank], stats tensor,
    plan)."""
    G = len(ranks)
    counts = np.stack([r.route().cpu().numpy() for r in ranks]).astype(np.int64)
    wl = ranks[0].wl
    plan = make_plan(counts, T_all, wl.k, wl.E, wl.cf, ranks[0].pad)
    dev = ranks[0].x.device
    recv = [torch.empty((max(int(plan.recv_rows(q).sum()), 1), wl.d), dtype=ranks[0].x.dtype,
                        device=dev) for q in range(G)]
    for r in ranks:
        r.dispatch_peers(plan, [t.data_ptr() for t in recv])
    ys = [ranks[q].ffn(plan, recv[q][:int(plan.recv_rows(q).sum())], bound=bound)
          for q in range(G)]
    ys = [y if y.shape[0] else torch.empty((1, wl.d), dtype=torch.float32, device=dev)
          for y in ys]
    outs = [r.combine_peers(plan, [y.data_ptr() for y in ys]) for r in ranks]
    sums = sum(r.stats_sums().clone() for r in ranks)
    stats = torch.zeros(5, dtype=torch.float64, device=sums.device)
    B.moe_stats_finalize(ranks[0].cfg, sums, stats)
    return outs, stats, plan


def forward_emulated_peers_device(ranks: List[Rank], T_all: int, max_rows: int,
                                  timer: Optional[StepTimer] = None):
    """The peer-memory form with the plan on the device, G ranks emulated in
    one process on one GPU (stream order stands in for the barriers).  No
    count or plan value is read back to the host.  Returns ([out per rank],
    stats tensor)."""
    G = len(ranks)
    wl = ranks[0].wl
    dev = ranks[0].x.device
    _mark(timer, "start")
    counts_all = torch.cat([r.route() for r in ranks])          # [G * E] on the device
    C = capacity(T_all, wl.k, wl.E, wl.cf)
    plans = [device_plan(r, counts_all, C) for r in ranks]
    recv = [torch.empty((max_rows, wl.d), dtype=ranks[0].x.dtype, device=dev) for _ in range(G)]
    ys = [torch.empty((max_rows, wl.d), dtype=torch.float32, device=dev) for _ in range(G)]
    _mark(timer, "dispatch0")
    for r, p in zip(ranks, plans):
        r.dispatch_peers_dev(p, [t.data_ptr() for t in recv])
    _mark(timer, "dispatch1")
    bound = min(C, T_all)
    for q in range(G):
        ranks[q].ffn_dev(plans[q], recv[q], ys[q], bound)
    _mark(timer, "combine0")
    outs = [r.combine_peers_dev(p, [y.data_ptr() for y in ys]) for r, p in zip(ranks, plans)]
    _mark(timer, "combine1")
    sums = sum(r.stats_sums().clone() for r in ranks)
    stats = torch.zeros(5, dtype=torch.float64, device=sums.device)
    B.moe_stats_finalize(ranks[0].cfg, sums, stats)
    _mark(timer, "end")
    return outs, stats, plans


def forward_dist_peers(r: Rank, T_all: int, group=None, max_rows: Optional[int] = None,
                       device_plan_on: bool = True, timer: Optional[StepTimer] = None):
    """One step on this rank (one process per GPU) in the peer-memory form.
    The receive and output buffers are symmetric memory (every rank maps
    every other rank's), sized for `max_rows` received rows (default: every
    token of every rank routed here, T_all * k); the barriers are symmetric
    memory's stream-ordered barrier.  With device_plan_on the plan is computed
    on the GPU (moe_ep_plan) and the step reads nothing back to the host; the
    buffers must then hold the largest possible receive (the default size).
    Returns (out, stats tensor, plan: the host Plan, or the device plan's
    tensors)."""
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem
    wl = r.wl
    _mark(timer, "start")
    rows = max_rows if max_rows is not None else T_all * wl.k + wl.E * r.pad
    if device_plan_on:
        if rows < T_all * wl.k + wl.E * r.pad:
            raise ValueError("with the plan on the device the buffers hold the largest receive")
        counts_all = torch.empty(r.world * wl.E, dtype=torch.int32, device=r.x.device)
        dist.all_gather_into_tensor(counts_all, r.route().contiguous(), group=group)
        C = capacity(T_all, wl.k, wl.E, wl.cf)
        plan = device_plan(r, counts_all, C)
    else:
        counts = all_gather_counts(r.route(), r.world, group)
        plan = make_plan(counts, T_all, wl.k, wl.E, wl.cf, r.pad)
        # the same test on every rank (the plan is the same), so that all of them
        # stop together rather than leave the others at a barrier
        if int(plan.send.sum(axis=0).max()) > rows:
            raise ValueError("the receive buffers are smaller than this step's rows")
    if r.symm is None:
        grp = group if group is not None else dist.group.WORLD
        recv = symm_mem.empty(rows, wl.d, dtype=r.x.dtype, device=r.x.device)
        yb = symm_mem.empty(rows, wl.d, dtype=torch.float32, device=r.x.device)
        r.symm = (recv, yb, symm_mem.rendezvous(recv, grp), symm_mem.rendezvous(yb, grp))
    recv, yb, h_recv, h_y = r.symm
    if recv.shape[0] < rows:
        raise ValueError("max_rows is larger than the buffers allocated at the first step")
    _mark(timer, "dispatch0")
    if device_plan_on:
        r.dispatch_peers_dev(plan, list(h_recv.buffer_ptrs))
    else:
        r.dispatch_peers(plan, list(h_recv.buffer_ptrs))
    h_recv.barrier(channel=0)            # every source has stored its rows here
    _mark(timer, "dispatch1")
    if device_plan_on:
        r.ffn_dev(plan, recv[:rows], yb[:rows], min(C, T_all))
    else:
        n = int(plan.recv_rows(r.rank).sum())
        if n:
            r.ffn(plan, recv[:n], yb[:n])
    h_y.barrier(channel=0)               # every owner's outputs are in place
    _mark(timer, "combine0")
    if device_plan_on:
        out = r.combine_peers_dev(plan, list(h_y.buffer_ptrs))
    else:
        out = r.combine_peers(plan, list(h_y.buffer_ptrs))
    h_y.barrier(channel=1)               # every source has read: buffers free for the next step
    _mark(timer, "combine1")
    sums = r.stats_sums()
    dist.all_reduce(sums, group=group)
    stats = torch.zeros(5, dtype=torch.float64, device=sums.device)
    B.moe_stats_finalize(r.cfg, sums, stats)
    _mark(timer, "end")
    return out, stats, plan

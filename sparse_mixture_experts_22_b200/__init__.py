"""B200-native sparse top-k mixture-of-experts layer.

The layer runs in libmoe_b200.so (hand-written CUDA for sm_100a behind the C
ABI in include/moe.h); `binding` marshals torch tensors into those calls.
`workloads` and `inputs` describe and draw the synthetic batches; `dp` and
`ep` hold the data-parallel and expert-parallel plumbing.
"""

from .workloads import ORDER, WORKLOADS, Workload  # noqa: F401
from . import binding  # noqa: F401  (the .so loads on the first call)
from .binding import (  # noqa: F401
    MoEConfig, MoEError, alloc_grads, alloc_layer, backward, config_of, forward, make_config,
    moe_aux_stats, moe_backward, moe_backward_workspace_size, moe_combine_rows,
    moe_dispatch_capped, moe_expert_ffn_grouped, moe_grouped_workspace_size, moe_launch_count,
    moe_route_counts, moe_segment_pad, pack_weights_backward, moe_dispatch_peers,
    moe_combine_peers, moe_ep_plan, moe_set_pdl, moe_set_pair_tiles, moe_set_shared_overlap, moe_hidden_split, MOE_BF16, MOE_F32,
    moe_set_shared_sms,
    moe_capacity, moe_combine, moe_dispatch, moe_expert_ffn, moe_ffn_splits, moe_forward,
    moe_pack_weights, moe_perm_rows, moe_read_device_status, moe_route, moe_set_wait_limit_ns,
    moe_stats_finalize, moe_stats_sums, moe_trace_begin, moe_trace_end, moe_workspace_size,
    pack_weights, stats_dict,
)

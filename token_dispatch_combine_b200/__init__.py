"""MoE expert-parallel token round trip on one B200 (sm_100a).

route -> dispatch -> grouped SwiGLU expert FFN -> combine, as hand-written
CUDA kernels behind the C ABI of include/moe_b200.h.  This package is the
ctypes binding of that library (``_native``) plus torch-facing wrappers with
the same names (``api``).  Importing it builds/loads the library and raises
if that is impossible: there is no other implementation to fall back to.
"""
from . import _native
from .api import (DispatchOut, EplbPlan, MoEBalancedRoundTrip, MoEHostPipeline, MoERoundTrip, moe_combine,
                  moe_combine_rank_partials, moe_dispatch, moe_dispatch_counted, moe_reduce_rank_partials,
                  moe_route_count, moe_route_count_workspace_bytes, moe_ffn_down_combine, moe_combine_finalize,
                  moe_dispatch_workspace_bytes, moe_eplb_plan, moe_eplb_remap, moe_eplb_replicate,
                  moe_expert_ffn, moe_expert_ffn_gather, moe_ffn_down, moe_ffn_gate_up, moe_ffn_gate_up_gather,
                  moe_ffn_tiling_for, moe_get_error, moe_get_ffn_tiling, moe_route, moe_router_topk,
                  moe_set_ffn_tiling, new_dispatch_workspace)
from .ep import (EpPeer, EpPlan, MoEEPRank, ep_round_trip_one_gpu, ep_round_trip_ranks, ep_share_buffers,
                 moe_enable_peer_access, moe_ep_exchange_offsets, moe_ep_pack, moe_ep_plan, moe_ep_plan_host,
                 moe_ep_plan_workspace_bytes, moe_ep_recv_index)
from ._native import FFN_DOWN, FFN_GATE_UP, FFN_TILING_AUTO, FFN_TILING_PAIR, FFN_TILING_SINGLE, MoeError

_native.lib()  # build (if needed) and load now: fail loudly at import

__all__ = [
    "DispatchOut", "MoEHostPipeline", "MoERoundTrip", "MoeError", "moe_combine", "moe_dispatch", "moe_dispatch_workspace_bytes",
    "moe_expert_ffn", "moe_expert_ffn_gather", "moe_ffn_down", "moe_ffn_gate_up", "moe_ffn_gate_up_gather",
    "moe_get_error", "moe_route", "new_dispatch_workspace", "moe_set_ffn_tiling", "moe_get_ffn_tiling",
    "moe_ffn_tiling_for", "FFN_TILING_AUTO", "FFN_TILING_SINGLE", "FFN_TILING_PAIR", "FFN_GATE_UP", "FFN_DOWN",
    "moe_router_topk", "EplbPlan", "MoEBalancedRoundTrip", "moe_eplb_plan", "moe_eplb_remap", "moe_eplb_replicate",
    "moe_combine_rank_partials", "moe_reduce_rank_partials", "EpPeer", "EpPlan", "MoEEPRank", "ep_round_trip_one_gpu",
    "ep_round_trip_ranks", "ep_share_buffers", "moe_enable_peer_access",
    "moe_ep_exchange_offsets", "moe_ep_pack", "moe_ep_plan", "moe_ep_plan_host", "moe_ep_plan_workspace_bytes",
    "moe_ep_recv_index", "moe_route_count", "moe_dispatch_counted", "moe_ffn_down_combine", "moe_combine_finalize",
    "moe_route_count_workspace_bytes",
]

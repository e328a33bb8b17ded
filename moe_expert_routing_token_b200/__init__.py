"""B200-native (sm_100a) Mixture-of-Experts token-to-expert routing.

The compute lives in ``libmoe_routing.so`` (hand-written CUDA kernels behind
the C ABI in ``include/moe_routing.h``); this package is its thin binding.
Build the library with ``python -m moe_expert_routing_token_b200.build``.
"""
from .routing import (  # noqa: F401
    MOE_DTYPE_BF16,
    MOE_DTYPE_F32,
    MOE_WEIGHT_E_BY_K,
    MOE_WEIGHT_K_BY_E,
    RoutingError,
    biased_grouped_topk,
    expert_permutation,
    expert_permutation_workspace_size,
    fill_shared_expert_slot,
    fill_shared_expert_slot_philox,
    fused_router_top1,
    fused_router_topk,
    fused_router_workspace_size,
    grouped_topk,
    lib,
    sort_topk_by_id,
    topk_softmax,
    watchdog_trips,
)

__all__ = [
    "topk_softmax", "grouped_topk", "biased_grouped_topk", "fused_router_topk",
    "fused_router_workspace_size", "lib", "RoutingError", "watchdog_trips", "expert_permutation",
    "expert_permutation_workspace_size", "fill_shared_expert_slot", "fill_shared_expert_slot_philox", "sort_topk_by_id", "fused_router_top1",
]

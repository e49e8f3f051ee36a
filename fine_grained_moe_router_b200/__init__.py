"""B200-native forward pass of one fine-grained Mixture-of-Experts FFN layer.

The compute lives in ``libmoe.so`` (hand-written sm_100a CUDA kernels behind
the C ABI of ``include/moe.h``); this package is its Python binding plus a
small convenience wrapper. Importing it fails if the library is not built.
"""
from ._binding import (  # noqa: F401
    EXPORTED, LIB_PATH, MOE_BF16, MOE_F32, MoEError, MoELayerDesc, MoELayerWeights, MoERouting,
    MoEStats, alloc_workspace, dtype_code, make_desc, make_routing, make_weights,
    moe_check_status, moe_kernel_launch_count, moe_combine, moe_dispatch, moe_dispatch_noalloc, moe_expert_gemms, moe_gather_rows, moe_ep_local_order, moe_expert_stats, moe_bias_update, moe_grouped_ffn,
    moe_layer_forward, moe_layer_forward_noisy, moe_layer_forward_profiled, moe_topk_from_logits_noisy, FORWARD_STAGES, moe_router_topk, moe_topk_from_logits, moe_workspace_size, status_string,
)
from .layer import MoELayer  # noqa: F401

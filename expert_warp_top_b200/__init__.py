"""expert_warp_top_b200: the hot path of an Occult-style mixture-of-experts
layer (top-k routing, BRIM-guided dispatch, grouped SwiGLU experts on tcgen05,
per-rank pre-reduce and combine) as hand-written CUDA for B200 (sm_100a),
with its training backward (input- and weight-gradient GEMMs on tcgen05,
routing backward) through the same BRIMs.

The CUDA library is loaded on first use; without it every call raises.
"""
from ._binding import (  # noqa: F401
    EXPORTS, MOE_BF16, MOE_F32, MOE_FFN_IDENTITY, MOE_FFN_SWIGLU, MOE_OK, MOE_ERR_CUDA,
    MOE_ERR_DEVICE_CHECK, MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MoeError,
    dtype_code, lib_path, load, moe_abi_version, moe_brim_build, moe_brim_build_noalloc, moe_brim_workspace_size,
    moe_coact_histogram, moe_combine_scatter, moe_count_dispatched_rows, moe_dispatch_gather,
    moe_expert_ffn, moe_expert_ffn_workspace_size, moe_get_device_status,
    moe_prepare_shared_weights, moe_prepare_weights, moe_route_topk, moe_set_debug,
    moe_layer_workspace_size, moe_layer_forward, moe_layer_forward_host, moe_place_greedy,
    moe_route_brim, moe_route_brim_workspace_size, moe_prune_topk,
    moe_expert_ffn_train, moe_expert_ffn_backward, moe_expert_ffn_backward_workspace_size,
    moe_route_backward, moe_layer_train_workspace_size, moe_layer_forward_train,
    moe_layer_backward, moe_interlayer_histogram, moe_rank_affinity, moe_predict_home,
    moe_count_local, moe_token_shuffle_workspace_size, moe_token_shuffle,
)
from .layer import MoELayer, unpack_gate_up  # noqa: F401

"""B200-native (sm_100a) token-choice MoE layer: router, dispatch, grouped
SwiGLU experts, combine and backward, behind the C ABI of include/moe.h.

Importing the package does not load the CUDA library; the first call into
the API does, and fails loudly if libmoe.so has not been built
(`python -m mixture_experts_routing_fp32_b200.build`).
"""
from .api import (MoEError, MoeConfig, MoeSizes, config_from, make_config,
                  moe_aux_loss, moe_backward, moe_check_status, moe_combine,
                  moe_dispatch, moe_expert_ffn, moe_get_sizes, moe_launch_count,
                  moe_router, moe_set_side_streams, moe_aux_loss_seq, moe_bias_update,
                  moe_route_expert_choice, moe_expert_ffn_gather,
                  moe_expert_ffn_combine, moe_aux_stats, moe_aux_loss_global,
                  moe_set_backward_streams)
from .layer import MoELayer

__all__ = ["MoEError", "MoeConfig", "MoeSizes", "config_from", "make_config",
           "moe_aux_loss", "moe_backward", "moe_check_status", "moe_combine",
           "moe_dispatch", "moe_expert_ffn", "moe_get_sizes", "moe_launch_count",
           "moe_router", "moe_set_side_streams", "moe_aux_loss_seq", "moe_bias_update",
           "moe_route_expert_choice", "moe_expert_ffn_gather",
           "moe_expert_ffn_combine", "moe_aux_stats", "moe_aux_loss_global",
           "moe_set_backward_streams", "MoELayer"]

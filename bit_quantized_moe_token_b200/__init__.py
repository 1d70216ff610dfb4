"""W4A8-FP8 routed mixture-of-experts layer for B200 (sm_100a).

The work happens in ``libmoe_w4a8.so`` (hand-written CUDA, C ABI in
``include/moe_w4a8.h``); this package only marshals torch tensors into it.
"""
from ._binding import (MOE_OK, Layer, MoeError, fp8_quant_tokens, layer_struct, lib,
                       moe_last_device_status, moe_route_topk, moe_route_workspace_bytes,
                       moe_router_logits,
                       moe_status_string, moe_w4a8_forward, moe_w4a8_forward_profiled,
                       moe_w4a8_workspace_bytes, STAGES, N_STAGE_EVENTS,
                       moe_w4a8_workspace_layout, w4a8_pack_weights,
                       moe_selftest_bounded_wait, Layer8, layer8_struct, w8a8_quant_weights,
                       moe_w8a8_workspace_bytes, moe_w8a8_workspace_layout, moe_w8a8_forward,
                       moe_w8a8_forward_profiled, moe_router_topk, moe_router_topk_workspace_bytes,
                       moe_w4a8_forward_router, moe_w8a8_forward_router, Layer4, layer4_struct,
                       nvfp4_quant_weights, moe_nvfp4_workspace_bytes, moe_nvfp4_workspace_layout,
                       moe_nvfp4_forward, moe_nvfp4_forward_profiled, moe_nvfp4_forward_router,
                       LayerH, moe_hybrid_workspace_bytes, moe_hybrid_workspace_layout,
                       moe_hybrid_forward, moe_hybrid_forward_profiled, ep_record_bytes,
                       moe_ep_dispatch_workspace_bytes, moe_ep_dispatch, moe_ep_experts_workspace_bytes,
                       moe_ep_experts_forward, moe_ep_combine)
from .layer import (alloc_workspace, forward, hybrid_from, make_layer, make_layer_nvfp4, make_layer_w8a8,
                    pack_expert_weights, quant_expert_weights_nvfp4, quant_expert_weights_w8a8)

__all__ = ["MOE_OK", "Layer", "MoeError", "fp8_quant_tokens", "layer_struct", "lib",
           "moe_last_device_status", "moe_route_topk", "moe_route_workspace_bytes",
           "moe_router_logits",
           "moe_status_string", "moe_w4a8_forward", "moe_w4a8_forward_profiled", "STAGES",
           "N_STAGE_EVENTS", "moe_w4a8_workspace_bytes",
           "moe_w4a8_workspace_layout", "w4a8_pack_weights", "alloc_workspace", "forward",
           "make_layer", "pack_expert_weights", "moe_selftest_bounded_wait",
           "Layer8", "layer8_struct", "w8a8_quant_weights", "moe_w8a8_workspace_bytes",
           "moe_w8a8_workspace_layout", "moe_w8a8_forward", "moe_w8a8_forward_profiled",
           "make_layer_w8a8", "quant_expert_weights_w8a8", "moe_router_topk",
           "moe_router_topk_workspace_bytes", "moe_w4a8_forward_router", "moe_w8a8_forward_router",
           "Layer4", "layer4_struct", "nvfp4_quant_weights", "moe_nvfp4_workspace_bytes",
           "moe_nvfp4_workspace_layout", "moe_nvfp4_forward", "moe_nvfp4_forward_profiled",
           "make_layer_nvfp4", "quant_expert_weights_nvfp4", "moe_nvfp4_forward_router",
           "LayerH", "moe_hybrid_workspace_bytes", "moe_hybrid_workspace_layout", "moe_hybrid_forward",
           "moe_hybrid_forward_profiled", "hybrid_from", "ep_record_bytes",
           "moe_ep_dispatch_workspace_bytes", "moe_ep_dispatch", "moe_ep_experts_workspace_bytes",
           "moe_ep_experts_forward", "moe_ep_combine"]

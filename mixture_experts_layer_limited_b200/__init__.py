"""DeepSeek-V3 / V2-Lite MoE layer forward on NVIDIA B200 (sm_100a).

The compute lives in libmoe.so (C ABI, include/moe.h), built by
`mixture_experts_layer_limited_b200.build`. `native` binds its entry points
one to one; `layer.MoELayer` chains them into the layer forward;
`pipeline.HostPipeline` runs forwards over host-resident batches with the
copies overlapped.
"""
from . import native
from .native import (moe_route, moe_gate_logits, moe_permute, moe_permute_workspace_size, moe_grouped_swiglu,
                     moe_gate_up_swiglu, moe_gate_up_swiglu_gather, moe_down_proj,
                     moe_gate_up_swiglu_with_shared, moe_down_proj_with_shared, moe_down_proj_combine,
                     moe_swiglu_ffn_sync_size, moe_swiglu_ffn_with_shared, moe_combine, moe_bias_update, moe_aux_loss, moe_aux_loss_workspace_size,
                     moe_quantize_blocks, moe_quantize_rows, moe_read_device_status, load_library, MoEError)
from .layer import MoELayer, LayerSpec
from .pipeline import HostPipeline

__all__ = ["native", "moe_route", "moe_gate_logits", "moe_permute", "moe_permute_workspace_size",
           "moe_grouped_swiglu", "moe_gate_up_swiglu", "moe_gate_up_swiglu_gather", "moe_down_proj",
           "moe_gate_up_swiglu_with_shared", "moe_down_proj_with_shared", "moe_down_proj_combine",
           "moe_swiglu_ffn_sync_size", "moe_swiglu_ffn_with_shared", "moe_combine", "moe_bias_update",
           "moe_aux_loss", "moe_aux_loss_workspace_size", "moe_quantize_blocks", "moe_quantize_rows",
           "moe_read_device_status", "load_library", "MoEError", "MoELayer", "LayerSpec", "HostPipeline"]

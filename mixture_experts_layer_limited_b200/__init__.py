"""DeepSeek-V3 / V2-Lite MoE layer forward on NVIDIA B200 (sm_100a).

The compute lives in libmoe.so (C ABI, include/moe.h), built by
`mixture_experts_layer_limited_b200.build`. `native` binds its entry points
one to one; `layer.MoELayer` chains them into the layer forward.
"""
from . import native
from .native import (moe_route, moe_permute, moe_permute_workspace_size, moe_grouped_swiglu,
                     moe_gate_up_swiglu, moe_gate_up_swiglu_gather, moe_down_proj,
                     moe_combine, moe_bias_update, moe_quantize_blocks, moe_quantize_rows,
                     moe_read_device_status, load_library, MoEError)
from .layer import MoELayer, LayerSpec

__all__ = ["native", "moe_route", "moe_permute", "moe_permute_workspace_size",
           "moe_grouped_swiglu", "moe_gate_up_swiglu", "moe_gate_up_swiglu_gather", "moe_down_proj", "moe_combine", "moe_bias_update", "moe_quantize_blocks",
           "moe_quantize_rows", "moe_read_device_status", "load_library", "MoEError",
           "MoELayer", "LayerSpec"]

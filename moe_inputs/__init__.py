"""Seeded synthetic inputs for the MoE layer forward.

This module is shared by the CPU oracle and the CUDA path. It holds the five
layer shapes and seeded random draws, and nothing of the method's own
arithmetic (no routing, no quantisation, no FFN): every value it returns is a
plain random draw, cast once to the storage dtype.

Shapes follow the pages:
  * DeepSeek-V2-Lite MoE layer: "MoE 混合专家模型推理参数与前向传播详解"
    (zhiyuanblog.org/blog/moe-inference) §1.3 MoE config and §2 parameter table.
  * DeepSeek-V3 MoE layer: the gsyq.cn DeepSeek-V3 MoE/MLA teardown, §3
    (moe_router.json: 256 routed + 1 shared, top-8, n_group 8, topk_group 4,
    norm_topk_prob true, routed_scaling_factor 2.5, sigmoid scoring).
"""
from .configs import MoEConfig, CONFIGS, get_config, tiny_grouped_config
from .generate import make_inputs, make_logits, MoEInputs

__all__ = ["MoEConfig", "CONFIGS", "get_config", "tiny_grouped_config",
           "make_inputs", "make_logits", "MoEInputs"]

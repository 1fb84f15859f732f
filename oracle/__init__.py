"""Plain CPU oracle of the DeepSeek-V3 / V2-Lite MoE layer forward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only the tests, the smoke check in the repository's entry module and the
benchmark's CPU-baseline / reference arm may call it. It shares no code with
the CUDA library; the two meet only through the seeded inputs of `moe_inputs`.

Every floating-point value is carried in float64, except the router's
selection decisions, which are taken on float32 scores (the precision of the
GPU kernel, see `route_from_logits`).

Parity status per function (what pins each one is listed in the tests):
  e4m3_values / quantize_e4m3 / round_to_e4m3 /
  fp8_quantize_* / fp8_qdq_*                    pinned (format facts, torch cast,
                                                the two roundings agree)
  gate_logits                                   pinned (identity gate)
  route_from_logits                             pinned (brute force, invariants)
  permute                                       pinned (worked example)
  swiglu_hidden / swiglu_ffn                    pinned (closed forms SiLU(+-1),
                                                SiLU(ln 3) = 3/4 ln 3; gate/up order)
  combine                                       pinned (hand example, equals the
                                                layer's own sum over slots)
  moe_forward                                   pinned (dense brute force,
                                                combine identities)
  bias_update / load_cv                         pinned (closed forms)
  seq_aux_loss                                  pinned (closed forms: balanced,
                                                collapsed, disjoint, per-sequence)
"""
from .moe_oracle import (
    e4m3_values, quantize_e4m3, dequantize_e4m3, round_to_e4m3, fp8_quantize_blocks,
    fp8_quantize_rows, fp8_qdq_blocks, fp8_qdq_rows, gate_logits, selection_scores, route_from_logits,
    RouteResult, permute, swiglu_hidden, swiglu_ffn, moe_forward, combine, bias_update, load_cv,
    seq_aux_loss,
)

__all__ = [
    "e4m3_values", "quantize_e4m3", "dequantize_e4m3", "round_to_e4m3",
    "fp8_quantize_blocks", "fp8_quantize_rows", "fp8_qdq_blocks", "fp8_qdq_rows", "gate_logits", "selection_scores",
    "route_from_logits", "RouteResult", "permute", "swiglu_hidden", "swiglu_ffn",
    "moe_forward", "combine", "bias_update", "load_cv", "seq_aux_loss",
]

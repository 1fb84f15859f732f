"""Seeded draws of every input tensor of the MoE layer.

Recipe (one torch.Generator per call, on the device the tensors live on,
drawn in this fixed order):
  x     ~ N(0, 1)                        [T, H]      (skewed layer: + 0.5*xbar)
  gate  ~ N(0, 0.02^2)                   [E, H]      (skewed layer: rows e < skew
                                                      get + 0.5*xbar)
  bias  ~ U(-0.05, 0.05)                 [E] fp32    (sigmoid layers only)
  w13   ~ N(0, 0.02^2)                   [E, 2I, H]  rows [0, I) gate, [I, 2I) up
  w2    ~ N(0, 0.02^2)                   [E, H, I]
  sw13  ~ N(0, 0.02^2)                   [2 I_s, H]  merged shared expert
  sw2   ~ N(0, 0.02^2)                   [H, I_s]
Draws are fp32 and are cast once (round to nearest even) to bf16 storage.
xbar is a seeded unit vector drawn before everything else (skewed layer only).
Weights are stored out-features-major (K-major), the stacked layout of the
"MoE 混合专家模型推理参数与前向传播详解" page, §2.2 (w13 (E, 2I, H), w2 (E, H, I)).
"""
from dataclasses import dataclass
from typing import Optional

import torch

from .configs import MoEConfig


@dataclass
class MoEInputs:
    cfg: MoEConfig
    x: torch.Tensor
    gate: torch.Tensor
    bias: Optional[torch.Tensor]
    w13: Optional[torch.Tensor]
    w2: Optional[torch.Tensor]
    sw13: Optional[torch.Tensor]
    sw2: Optional[torch.Tensor]
    xbar: Optional[torch.Tensor] = None


def _normal(gen, shape, std, device, chunk_dim0=None):
    """fp32 N(0, std^2) draw cast to bf16, drawn chunk by chunk along dim 0."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if chunk_dim0 is None:
        chunk_dim0 = shape[0]
    for s in range(0, shape[0], chunk_dim0):
        e = min(shape[0], s + chunk_dim0)
        tmp = torch.randn((e - s,) + tuple(shape[1:]), generator=gen,
                          dtype=torch.float32, device=device)
        if std != 1.0:
            tmp.mul_(std)
        out[s:e].copy_(tmp)
    return out


def make_inputs(cfg: MoEConfig, device="cpu", seed: Optional[int] = None,
                experts: bool = True, shared: bool = True) -> MoEInputs:
    """Draw every input of `cfg` on `device` from `seed` (default cfg.seed)."""
    seed = cfg.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, H, E, I, I_s = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_s

    xbar = None
    if cfg.skew_experts:
        v = torch.randn(H, generator=gen, dtype=torch.float32, device=device)
        xbar = v / torch.linalg.vector_norm(v)

    x32 = torch.randn((T, H), generator=gen, dtype=torch.float32, device=device)
    if xbar is not None:
        x32.add_(0.5 * xbar)
    x = x32.to(torch.bfloat16)
    del x32

    g32 = torch.randn((E, H), generator=gen, dtype=torch.float32, device=device)
    g32.mul_(0.02)
    if xbar is not None:
        g32[: cfg.skew_experts].add_(0.5 * xbar)
    gate = g32.to(torch.bfloat16)
    del g32

    bias = None
    if cfg.has_bias:
        bias = (torch.rand(E, generator=gen, dtype=torch.float32, device=device)
                * 0.1 - 0.05)

    w13 = w2 = sw13 = sw2 = None
    if experts:
        per = max(1, (1 << 27) // (2 * I * H))  # keep fp32 temporaries small
        w13 = _normal(gen, (E, 2 * I, H), 0.02, device, chunk_dim0=per)
        w2 = _normal(gen, (E, H, I), 0.02, device, chunk_dim0=per)
    if shared and I_s > 0:
        sw13 = _normal(gen, (2 * I_s, H), 0.02, device)
        sw2 = _normal(gen, (H, I_s), 0.02, device)
    return MoEInputs(cfg, x, gate, bias, w13, w2, sw13, sw2, xbar)


def make_logits(cfg: MoEConfig, device="cpu", seed: Optional[int] = None,
                T: Optional[int] = None) -> torch.Tensor:
    """fp32 router logits [T, E] with the spread of x @ gate^T at this shape.

    Used to feed identical logits to both the oracle and the CUDA router.
    Values are N(0, H * 0.02^2); the draw is rounded to fp32 only.
    """
    seed = (cfg.seed + 7777) if seed is None else seed
    T = cfg.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    std = (cfg.H ** 0.5) * 0.02
    return torch.randn((T, cfg.E), generator=gen, dtype=torch.float32,
                       device=device) * std

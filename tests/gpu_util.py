"""Shared helpers of the GPU parity tests (not a test module)."""
import numpy as np
import torch

import oracle
from mixture_experts_layer_limited_b200 import native as N

BF16_TOL = 2e-2     # max|y - y_ref| / max|y_ref| for BF16 layers
FP8_TOL = 6e-2      # same for the E4M3 layer
NEAR_TIE = 1e-5     # routing decisions closer than this are excluded and counted


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def rel_err(y, ref) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(y - ref).max() / np.abs(ref).max())


def scoring_code(cfg) -> int:
    return N.MOE_SIGMOID if cfg.scoring == "sigmoid" else N.MOE_SOFTMAX


def oracle_route(L32: np.ndarray, cfg, bias: np.ndarray = None):
    return oracle.route_from_logits(L32, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                    cfg.norm_topk_prob, cfg.scale, bias)


def gpu_route(cfg, T, x=None, gate=None, bias=None, logits=None, write_logits=True):
    """Runs moe_route; returns (ids, w, counts, logits) device tensors."""
    dev = torch.device("cuda")
    ids = torch.empty(T, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(T, cfg.k, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    if logits is None and write_logits:
        logits = torch.empty(T, cfg.E, dtype=torch.float32, device=dev)
    N.moe_route(T, cfg.H, cfg.E, cfg.k, cfg.n_group, cfg.topk_group, scoring_code(cfg),
                cfg.norm_topk_prob, cfg.scale, x, gate, bias, logits, ids, w, counts)
    return ids, w, counts, logits


def near_tie_mask(route) -> np.ndarray:
    return (route.kth_gap < NEAR_TIE) | (route.group_gap < NEAR_TIE)


def uniform_bias(E, seed, device="cuda"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.rand(E, generator=g, dtype=torch.float32, device=device) * 0.1 - 0.05


def routing_mismatch(ids_gpu: np.ndarray, route) -> np.ndarray:
    """Tokens whose chosen expert SET differs (slot order may flip between
    two chosen experts whose scores are within float noise; y is the same)."""
    return np.any(np.sort(ids_gpu, axis=1) != np.sort(route.ids, axis=1), axis=1)


def describe_mismatch(ids_gpu, route, tokens):
    lines = []
    for t in tokens[:5]:
        lines.append(f"token {t}: gpu {ids_gpu[t].tolist()} oracle {route.ids[t].tolist()} "
                     f"kth_gap {route.kth_gap[t]:.3e} group_gap {route.group_gap[t]:.3e}")
    return "\n".join(lines)

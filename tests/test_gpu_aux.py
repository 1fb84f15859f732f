"""Sequence-level auxiliary balance loss ("MoE 混合专家模型推理参数与前向传播详解"
§6.2) of libmoe against the CPU oracle (needs a B200).

Both sides evaluate and sum the scores in fp64; they differ only in the order
of the sums and in the last bits of exp, far below the single fp32 rounding of
the result, so the value must agree to a few fp32 ulps (rel 1e-6). A dropped
normalisation, a wrong sequence grouping or a load/importance index mix-up is
O(1e-2) or more."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import get_config, tiny_grouped_config, make_logits
from mixture_experts_layer_limited_b200 import native as N
from mixture_experts_layer_limited_b200.layer import LayerSpec, MoELayer
from gpu_util import np32, oracle_route, scoring_code, uniform_bias

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL = 1e-6


def _cfg(name):
    return tiny_grouped_config() if name == "tiny_grouped" else get_config(name)


def _gpu_aux(cfg, T, seq_len, L, ids, alpha=0.001):
    ws = torch.empty(N.moe_aux_loss_workspace_size(T, cfg.E, seq_len), dtype=torch.uint8, device=DEV)
    out = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_aux_loss(T, cfg.E, cfg.k, seq_len, scoring_code(cfg), L, ids, alpha, out, ws, status)
    assert N.moe_read_device_status(status) == 0
    return float(out.item())


@pytest.mark.parametrize("name,T,seq_len", [
    ("tiny", None, None), ("tiny", None, 16), ("tiny_grouped", None, 8),
    ("v2lite", None, None), ("v2lite", None, 1024), ("v2lite", 129, None),
    ("v3", None, None), ("v3", None, 4096), ("v3", 1000, 200), ("v3", 1000, 1), ("v3", 1, None),
])
def test_aux_loss_matches_oracle(name, T, seq_len):
    cfg = _cfg(name)
    T = T or cfg.T
    seq_len = seq_len or T
    L = make_logits(cfg, device=DEV, T=T)
    bias = uniform_bias(cfg.E, cfg.seed + 5) if cfg.scoring == "sigmoid" else None
    r = oracle_route(np32(L), cfg, np32(bias) if bias is not None else None)
    ids = torch.from_numpy(r.ids.astype(np.int32)).to(DEV)
    got = _gpu_aux(cfg, T, seq_len, L, ids)
    ref = oracle.seq_aux_loss(np32(L), r.ids, cfg.E, cfg.k, cfg.scoring, seq_len, 0.001)
    print(f"{name} T={T} seq_len={seq_len}: aux {got:.9e} oracle {ref:.9e}")
    assert got == pytest.approx(ref, rel=REL)


@pytest.mark.parametrize("scoring", ["softmax", "sigmoid"])
def test_aux_loss_closed_forms_on_gpu(scoring):
    cfg = dataclasses.replace(get_config("tiny"), scoring=scoring)
    T, E, k = 256, cfg.E, cfg.k
    zeros = torch.zeros(T, E, dtype=torch.float32, device=DEV)
    rr = ((torch.arange(T)[:, None] * k + torch.arange(k)[None, :]) % E).to(torch.int32).to(DEV)
    assert _gpu_aux(cfg, T, T, zeros, rr, alpha=1.0) == pytest.approx(1.0, rel=REL)
    assert _gpu_aux(cfg, T, 64, zeros, rr, alpha=1.0) == pytest.approx(1.0, rel=REL)
    if scoring == "softmax":
        L = torch.full((T, E), -1e4, dtype=torch.float32, device=DEV)
        L[:, :k] = 0.0
        first_k = torch.arange(k, dtype=torch.int32, device=DEV).repeat(T, 1)
        assert _gpu_aux(cfg, T, T, L, first_k, alpha=1.0) == pytest.approx(E / k, rel=REL)


def test_aux_loss_flags_bad_expert_ids():
    cfg = get_config("tiny")
    T = 64
    L = make_logits(cfg, device=DEV, T=T)
    ids = torch.zeros(T, cfg.k, dtype=torch.int32, device=DEV)
    ids[3, 1] = cfg.E
    ws = torch.empty(N.moe_aux_loss_workspace_size(T, cfg.E, T), dtype=torch.uint8, device=DEV)
    out = torch.empty(1, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_aux_loss(T, cfg.E, cfg.k, T, N.MOE_SOFTMAX, L, ids, 1.0, out, ws, status)
    assert N.moe_read_device_status(status) & N.MOE_DEVSTAT_BAD_EXPERT_ID


@pytest.mark.parametrize("name", ["v2lite", "v3"])
def test_layer_aux_loss_after_routing(name):
    cfg = get_config(name)
    T = 2048
    spec = LayerSpec.from_config(cfg)
    g = torch.Generator(device=DEV)
    g.manual_seed(11)
    gate = (torch.randn(cfg.E, cfg.H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    tiny = torch.zeros(1, 1, 1, dtype=torch.bfloat16, device=DEV)     # experts unused here
    bias = uniform_bias(cfg.E, cfg.seed + 5) if cfg.scoring == "sigmoid" else None
    layer = MoELayer(spec, gate, tiny, tiny, None, None, bias, T_max=T, tiled_weights=False)
    L = make_logits(cfg, device=DEV, T=T)
    x = torch.zeros(T, cfg.H, dtype=torch.bfloat16, device=DEV)
    layer.logits[:T].copy_(L)                    # the logits the layer keeps for the aux loss
    layer.route(x, logits_in=layer.logits[:T])
    r = oracle_route(np32(L), cfg, np32(bias) if bias is not None else None)
    assert np.array_equal(layer.ids[:T].cpu().numpy(), r.ids)
    for seq_len in (T, 512):
        got = float(layer.aux_loss(T, seq_len).item())
        ref = oracle.seq_aux_loss(np32(L), r.ids, cfg.E, cfg.k, cfg.scoring, seq_len, 0.001)
        assert got == pytest.approx(ref, rel=REL)

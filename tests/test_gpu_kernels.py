"""Per-kernel parity of libmoe against the CPU oracle (needs a B200).

Bit-exact: E4M3 codes and scales, routing ids / counts given identical fp32
logits, the permutation, the bias trajectory. Floating point: within the
tolerance each test states."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle import moe_oracle as O
from moe_inputs import get_config, tiny_grouped_config, make_inputs, make_logits
from mixture_experts_layer_limited_b200 import native as N

from gpu_util import (np64, np32, rel_err, oracle_route, gpu_route, near_tie_mask, uniform_bias,
                      routing_mismatch, describe_mismatch, BF16_TOL, FP8_TOL)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


# ------------------------------------------------------------------ E4M3
def test_quantize_blocks_bytes_match_oracle():
    g = _gen(1)
    w = (torch.randn(3, 256, 384, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w[1, :128, :128] = 0                     # all-zero block -> scale 1
    w[2, 5, 7] = 3.0                         # outlier block
    w[2, 200, 300] = -1e-30                  # tiny negative -> signed zero code
    q = torch.empty(3, 256, 384, dtype=torch.uint8, device=DEV)
    s = torch.empty(3, 2, 3, dtype=torch.float32, device=DEV)
    N.moe_quantize_blocks(3, 256, 384, w, q, s)
    torch.cuda.synchronize()
    for b in range(3):
        qo, so = oracle.fp8_quantize_blocks(np32(w[b]))
        assert np.array_equal(q[b].cpu().numpy(), qo)
        assert np.array_equal(s[b].cpu().numpy(), so)


def test_quantize_rows_bytes_match_oracle():
    g = _gen(2)
    a = (torch.randn(257, 512, generator=g, device=DEV) * 3).to(torch.bfloat16)
    a[7, 128:256] = 0
    q = torch.empty(257, 512, dtype=torch.uint8, device=DEV)
    s = torch.empty(257, 4, dtype=torch.float32, device=DEV)
    N.moe_quantize_rows(257, 512, a, q, s)
    qo, so = oracle.fp8_quantize_rows(np32(a))
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)


# ---------------------------------------------------------------- router
ROUTE_CASES = [("tiny", None), ("tiny_grouped", None), ("v2lite", None), ("v3", None),
               ("v3", 1000), ("v3_ties", 777), ("v2lite", 1)]


def _cfg(name):
    if name == "tiny_grouped":
        return tiny_grouped_config()
    if name == "v3_ties":
        return get_config("v3")
    return get_config(name)


@pytest.mark.parametrize("name,T", ROUTE_CASES)
def test_route_from_logits_bit_exact(name, T):
    cfg = _cfg(name)
    T = T or cfg.T
    L = make_logits(cfg, device=DEV, T=T)
    if name == "v3_ties":
        L = torch.round(L * 4) / 4           # many exact ties in scores and group scores
    bias = uniform_bias(cfg.E, cfg.seed + 5) if cfg.scoring == "sigmoid" else None
    if name == "v3_ties":
        bias = torch.round(bias * 50) / 50
    ids, w, counts, _ = gpu_route(cfg, T, bias=bias, logits=L)
    torch.cuda.synchronize()
    r = oracle_route(np32(L), cfg, np32(bias) if bias is not None else None)
    assert np.array_equal(ids.cpu().numpy(), r.ids)
    assert np.array_equal(counts.cpu().numpy(), r.counts)
    np.testing.assert_allclose(w.cpu().numpy(), r.weights, rtol=5e-6, atol=1e-7)


def _near_tie_logits(T, E, G, gaps, rng):
    """Sigmoid-scored logits (no bias) where token t's 8th and 9th best
    experts, or its 4th and 5th best groups, are a chosen distance apart.
    Groups of E/G experts; every token has two strong experts in each of
    four groups (0, 2, 4, 6), then the tie is placed either between two
    experts of group 0 (the k-th / (k+1)-th boundary) or between groups 1
    and 3 (the kept / dropped group boundary)."""
    gsz = E // G
    L = np.full((T, E), -6.0, dtype=np.float32) + rng.uniform(0, 0.01, (T, E)).astype(np.float32)
    sig = lambda v: 1.0 / (1.0 + np.exp(-np.float64(v)))
    for t in range(T):
        gap = gaps[t % len(gaps)]
        for gi, g in enumerate((0, 2, 4, 6)):
            L[t, g * gsz + 3] = 4.0 - gi * 0.25
            L[t, g * gsz + 5] = 3.9 - gi * 0.25
        if (t // len(gaps)) % 2 == 0:
            # experts: seven clear winners in groups 0, 2, 4, 6 (two each but
            # group 6's second is weak), then the 8th / 9th pair in group 0
            L[t, 6 * gsz + 5] = -1.0
            a = np.float32(1.0)
            L[t, 0 * gsz + 7] = a
            # find b with sigmoid(a) - sigmoid(b) ~ gap in fp32 (the scores the oracle compares)
            target = np.float32(sig(a)) - np.float32(gap)
            b = np.float32(np.log(target / (1 - target)))
            L[t, 0 * gsz + 9] = b
        else:
            # groups: groups 1 and 3 compete for the 4th place, their top-2
            # sums a chosen distance apart; groups 2, 4, 6 strong, 0 weak
            L[t, 0 * gsz + 3] = -2.0
            L[t, 0 * gsz + 5] = -2.0
            L[t, 1 * gsz + 1] = 0.5
            L[t, 1 * gsz + 2] = 0.5
            s1 = np.float32(np.float32(sig(0.5)) + np.float32(sig(0.5)))
            target = np.float32(s1 - np.float32(gap)) - np.float32(sig(0.5))
            L[t, 3 * gsz + 1] = 0.5
            L[t, 3 * gsz + 2] = np.float32(np.log(target / (1 - target)))
    return L


def test_route_sigmoid_decisions_at_tiny_score_gaps_bit_exact():
    """Tokens whose k-th / (k+1)-th selection scores, or whose last kept and
    first dropped group scores, differ by 0 to 1e-4 (fp32 distances of a few
    ulp and up): routed on identical fp32 logits, ids, counts and weights
    must be the oracle's, bit for bit where the decision is taken."""
    cfg = dataclasses.replace(get_config("v3"), n_group=8, topk_group=4, k=8)
    rng = np.random.default_rng(77)
    gaps = [0.0, 1e-7, 5e-7, 1e-6, 2e-6, 3e-6, 4e-6, 5e-6, 7e-6, 8e-6, 9e-6, 1.2e-5, 3e-5, 1e-4]
    T = 28 * 20
    L = _near_tie_logits(T, cfg.E, cfg.n_group, gaps, rng)
    Ld = torch.from_numpy(L).to(DEV)
    for bias in (None, uniform_bias(cfg.E, 91) * 0.0):
        ids, w, counts, _ = gpu_route(cfg, T, bias=bias, logits=Ld)
        torch.cuda.synchronize()
        r = oracle_route(L, cfg, np32(bias) if bias is not None else None)
        assert np.array_equal(ids.cpu().numpy(), r.ids)
        assert np.array_equal(counts.cpu().numpy(), r.counts)
        np.testing.assert_allclose(w.cpu().numpy(), r.weights, rtol=5e-6, atol=1e-7)


@pytest.mark.parametrize("topk_group", [1, 2, 4, 8])
def test_route_topk_group_sweep_bit_exact_with_load_cv(topk_group):
    """The group-limit sweep at the V3 shape (8 groups): ids and counts
    bit-exact for every topk_group, and the load CV of moe_bias_update (gamma
    0: the bias stays) equal to the oracle's from the same integer counts."""
    cfg = dataclasses.replace(get_config("v3"), topk_group=topk_group)
    L = make_logits(cfg, device=DEV)
    bias = uniform_bias(cfg.E, cfg.seed + 5)
    ids, w, counts, _ = gpu_route(cfg, cfg.T, bias=bias, logits=L)
    cv = torch.empty(1, dtype=torch.float32, device=DEV)
    b = bias.clone()
    N.moe_bias_update(cfg.E, cfg.T, cfg.k, counts, b, 0.0, cv)
    torch.cuda.synchronize()
    r = oracle_route(np32(L), cfg, np32(bias))
    assert np.array_equal(ids.cpu().numpy(), r.ids)
    assert np.array_equal(counts.cpu().numpy(), r.counts)
    assert torch.equal(b, bias)
    ref_cv = oracle.load_cv(r.counts)
    print(f"topk_group={topk_group}: load CV {cv.item():.5f} (oracle {ref_cv:.5f})")
    assert cv.item() == pytest.approx(ref_cv, rel=1e-6)
    groups_used = (r.ids // (cfg.E // cfg.n_group))
    assert max(len(set(row)) for row in groups_used.tolist()) <= topk_group


# T picks the gate GEMM's cluster size (CTAs sharing one 128-token tile's
# hidden size): 8 up to 18 tiles (tiny, where some CTAs get no K block; 1000;
# 1; 129), 4 up to 37 (v2lite 4096; 3000 with a 56-token tail), 2 beyond (v3).
@pytest.mark.parametrize("name,T", [("tiny", None), ("tiny_grouped", None), ("v2lite", None),
                                    ("v3", None), ("v3", 1000), ("v3", 1), ("v2lite", 129),
                                    ("v3", 3000)])
def test_route_gate_gemm(name, T):
    cfg = _cfg(name)
    T = T or cfg.T
    inp = make_inputs(dataclasses.replace(cfg, T=T), device=DEV, experts=False, shared=False)
    bias = inp.bias
    ids, w, counts, L = gpu_route(cfg, T, x=inp.x, gate=inp.gate, bias=bias)
    torch.cuda.synchronize()
    L64 = oracle.gate_logits(np64(inp.x), np64(inp.gate))
    # fp32 accumulation of H bf16 products on the tensor cores: ~sqrt(H) * 2^-24 of
    # the partial sums; a layout or index mistake is O(1)
    assert rel_err(np64(L), L64) < 3e-5
    r = oracle_route(L64.astype(np.float32), cfg, np32(bias) if bias is not None else None)
    flagged = near_tie_mask(r)
    ids_g = ids.cpu().numpy()
    mism = routing_mismatch(ids_g, r)
    bad = np.nonzero(mism & ~flagged)[0]
    assert len(bad) == 0, f"{len(bad)} unflagged tokens differ\n" + describe_mismatch(ids_g, r, bad)
    order_flips = int(np.sum(np.any(ids_g != r.ids, axis=1) & ~mism))
    ok = ~flagged & np.all(ids_g == r.ids, axis=1)
    np.testing.assert_allclose(w.cpu().numpy()[ok], r.weights[ok], rtol=2e-5, atol=1e-6)
    print(f"{name} T={T}: slot-order flips among chosen experts {order_flips}")
    assert int(counts.sum()) == T * cfg.k
    print(f"{name} T={T}: near-tie tokens excluded {int(flagged.sum())}")


# Shapes outside the eight-threads-per-token kernel's range (k > 8, n_group
# not dividing 8, E / 8 not a power of two from 2 to 32) are routed by the
# general one-warp-per-token kernel: ids, counts and weights against the
# oracle as for the default kernel.
WARP_ROUTE_CASES = [
    ("v3 k=9", "v3", dict(k=9), 2048),
    ("v3 16 groups keep 8", "v3", dict(n_group=16, topk_group=8), 2048),
    ("E=48 softmax top-6", "v2lite", dict(E=48), 1500),
    ("tiny k=12", "tiny", dict(k=12), None),
    ("tiny_grouped k=9 ties", "tiny_grouped", dict(k=9, topk_group=3), 500),
]


@pytest.mark.parametrize("label,name,over,T", WARP_ROUTE_CASES, ids=[c[0] for c in WARP_ROUTE_CASES])
def test_route_warp_per_token_shapes_bit_exact(label, name, over, T):
    cfg = dataclasses.replace(_cfg(name), **over)
    T = T or cfg.T
    L = make_logits(cfg, device=DEV, T=T)
    bias = uniform_bias(cfg.E, cfg.seed + 5) if cfg.scoring == "sigmoid" else None
    if "ties" in label:
        L = torch.round(L * 4) / 4
        bias = torch.round(bias * 50) / 50
    ids, w, counts, _ = gpu_route(cfg, T, bias=bias, logits=L)
    torch.cuda.synchronize()
    r = oracle_route(np32(L), cfg, np32(bias) if bias is not None else None)
    assert np.array_equal(ids.cpu().numpy(), r.ids)
    assert np.array_equal(counts.cpu().numpy(), r.counts)
    np.testing.assert_allclose(w.cpu().numpy(), r.weights, rtol=5e-6, atol=1e-7)


@pytest.mark.parametrize("k", [8, 9], ids=["eight-threads-kernel", "warp-kernel"])
def test_route_token_with_nan_scores_is_flagged_not_routed(k):
    """Without a group limit, a token whose logits are all NaN has no winner
    in any round: its slots get id -1 and weight 0, the status word is
    flagged, nothing is counted for it, and the other tokens route as usual.
    (With a group limit the experts of the dropped groups score -inf, which
    still compares, so such a token is routed there with NaN weights.)
    k = 8 runs the eight-threads-per-token kernel, k = 9 the warp kernel."""
    cfg = dataclasses.replace(get_config("v3"), n_group=1, topk_group=1, k=k)
    T = 64
    L = make_logits(cfg, device=DEV, T=T)
    L[5] = float("nan")
    bias = uniform_bias(cfg.E, cfg.seed + 5)
    ids = torch.empty(T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, cfg.k, dtype=torch.float32, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_route(T, cfg.H, cfg.E, cfg.k, cfg.n_group, cfg.topk_group, N.MOE_SIGMOID, cfg.norm_topk_prob,
                cfg.scale, None, None, bias, L, ids, w, counts, status)
    torch.cuda.synchronize()
    assert N.moe_read_device_status(status) & N.MOE_DEVSTAT_BAD_EXPERT_ID
    assert torch.all(ids[5] == -1) and torch.all(w[5] == 0)
    keep = np.array([t for t in range(T) if t != 5])
    r = oracle_route(np32(L[torch.as_tensor(keep, device=DEV)]), cfg, np32(bias))
    assert np.array_equal(ids.cpu().numpy()[keep], r.ids)
    assert int(counts.sum()) == (T - 1) * cfg.k


@pytest.mark.parametrize("name,T", [("tiny", None), ("v3", None), ("v3", 1000), ("v3", 3000)])
def test_gate_logits_then_route_equals_route(name, T):
    """moe_gate_logits followed by moe_route on those logits (x = NULL) is
    moe_route in two calls: logits, ids, weights and counts bit for bit."""
    cfg = _cfg(name)
    T = T or cfg.T
    inp = make_inputs(dataclasses.replace(cfg, T=T), device=DEV, experts=False, shared=False)
    ids0, w0, c0, L0 = gpu_route(cfg, T, x=inp.x, gate=inp.gate, bias=inp.bias)
    L1 = torch.full_like(L0, float("nan"))
    N.moe_gate_logits(T, cfg.H, cfg.E, inp.x, inp.gate, L1)
    ids1, w1, c1, _ = gpu_route(cfg, T, bias=inp.bias, logits=L1)
    torch.cuda.synchronize()
    assert torch.equal(L0, L1)
    assert torch.equal(ids0, ids1) and torch.equal(w0, w1) and torch.equal(c0, c1)


# --------------------------------------------------------------- permute
def _ids_from_oracle(T, k, E, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    L = rng.standard_normal((T, E)).astype(np.float32)
    if skew:
        L[:, :4] += skew
    r = oracle.route_from_logits(L, k, 1, 1, "softmax", False, 1.0)
    return r.ids, r.weights.astype(np.float32)


@pytest.mark.parametrize("T,k,E,H,skew", [(64, 4, 16, 256, 0.0), (8192, 8, 256, 7168, 0.0),
                                          (1000, 6, 64, 2048, 0.0), (2000, 8, 256, 512, 3.0),
                                          (1, 1, 16, 256, 0.0), (3, 16, 16, 128, 0.0),
                                          (50, 2, 16, 28672, 0.0)])
def test_permute_bit_exact(T, k, E, H, skew):
    ids_np, w_np = _ids_from_oracle(T, k, E, seed=T + E, skew=skew)
    _check_permute(ids_np, w_np, E, H)


@pytest.mark.parametrize("T,k,E", [(200, 16, 16), (1000, 4, 4), (129, 8, 256), (64, 16, 1024)])
def test_permute_repeated_ids_keep_slot_order(T, k, E):
    """ids drawn with replacement, so a token may name one expert in several
    of its slots, and k = 16 puts a block's slots over several passes of the
    histogram kernel: rows still follow the stable order, token then slot."""
    rng = np.random.default_rng(T * k + E)
    ids_np = rng.integers(0, E, size=(T, k)).astype(np.int32)
    ids_np[0, :] = ids_np[0, 0]                        # one token with a single expert in every slot
    w_np = rng.random((T, k)).astype(np.float32)
    _check_permute(ids_np, w_np, E, 128)


def _check_permute(ids_np, w_np, E, H):
    T, k = ids_np.shape
    offsets_o, src_o, s2r_o = oracle.permute(ids_np, E)
    ids = torch.from_numpy(ids_np).to(DEV)
    tw = torch.from_numpy(w_np).to(DEV)
    x = torch.randn(T, H, generator=_gen(3), device=DEV).to(torch.bfloat16)
    R = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(R, dtype=torch.int32, device=DEV)
    s2r = torch.empty(R, dtype=torch.int32, device=DEV)
    roww = torch.empty(R, dtype=torch.float32, device=DEV)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(N.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_permute(T, k, E, H, ids, tw, x, N.MOE_BF16, None, xp, None, offsets, src, s2r, roww, ws, status)
    assert N.moe_read_device_status(status) == 0
    assert np.array_equal(offsets.cpu().numpy(), offsets_o)
    assert np.array_equal(src.cpu().numpy(), src_o)
    assert np.array_equal(s2r.cpu().numpy(), s2r_o)
    assert np.array_equal(roww.cpu().numpy(), w_np.reshape(-1)[np.argsort(s2r_o)])
    assert torch.equal(xp, x[torch.from_numpy(src_o).to(DEV)])


def test_permute_e4m3_rows_and_scales():
    T, k, E, H = 300, 8, 64, 512
    ids_np, w_np = _ids_from_oracle(T, k, E, seed=9)
    _, src_o, _ = oracle.permute(ids_np, E)
    xq = torch.randint(0, 255, (T, H), generator=_gen(4), device=DEV, dtype=torch.uint8)
    xs = torch.rand(T, H // 128, generator=_gen(5), device=DEV)
    R = T * k
    out = [torch.empty(E + 1, dtype=torch.int32, device=DEV)] + \
          [torch.empty(R, dtype=torch.int32, device=DEV) for _ in range(2)]
    roww = torch.empty(R, dtype=torch.float32, device=DEV)
    xp = torch.empty(R, H, dtype=torch.uint8, device=DEV)
    xps = torch.empty(R, H // 128, dtype=torch.float32, device=DEV)
    ws = torch.empty(N.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    N.moe_permute(T, k, E, H, torch.from_numpy(ids_np).to(DEV), torch.from_numpy(w_np).to(DEV),
                  xq, N.MOE_E4M3, xs, xp, xps, out[0], out[1], out[2], roww, ws)
    idx = torch.from_numpy(src_o).to(DEV)
    assert torch.equal(xp, xq[idx])
    assert torch.equal(xps, xs[idx])


@pytest.mark.parametrize("T,k,E,H", [(256, 8, 256, 7168), (300, 6, 64, 640), (1, 1, 16, 128)])
def test_permute_quantises_bf16_rows_to_e4m3(T, k, E, H):
    """perm_dtype E4M3 with bf16 x: every row of x_perm holds its token's
    1x128-tile E4M3 codes and scales, byte for byte the oracle's
    fp8_quantize_rows of x, and x_q / x_q_scale the token's own (H = 640:
    five tiles, so a warp step covers a partial group of four)."""
    ids_np, w_np = _ids_from_oracle(T, k, E, seed=T + H)
    off_o, src_o, s2r_o = oracle.permute(ids_np, E)
    g = _gen(T + 7)
    x = (torch.randn(T, H, generator=g, device=DEV) * 3).to(torch.bfloat16)
    x[0, 128:256] = 0                                  # an all-zero tile: scale 1, zero codes
    if T > 1:
        x[1, :128] = -x[1, :128].abs()                 # a tile of negative values only
    R = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(R, dtype=torch.int32, device=DEV)
    s2r = torch.empty(R, dtype=torch.int32, device=DEV)
    roww = torch.empty(R, dtype=torch.float32, device=DEV)
    xp = torch.empty(R, H, dtype=torch.uint8, device=DEV)
    xps = torch.empty(R, H // 128, dtype=torch.float32, device=DEV)
    xq = torch.empty(T, H, dtype=torch.uint8, device=DEV)
    xqs = torch.empty(T, H // 128, dtype=torch.float32, device=DEV)
    ws = torch.empty(N.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_permute(T, k, E, H, torch.from_numpy(ids_np).to(DEV), torch.from_numpy(w_np).to(DEV), x, N.MOE_BF16,
                  None, xp, xps, offsets, src, s2r, roww, ws, status, perm_dtype=N.MOE_E4M3, x_q=xq,
                  x_q_scale=xqs)
    assert N.moe_read_device_status(status) == 0
    qo, so = oracle.fp8_quantize_rows(np32(x))
    assert np.array_equal(xq.cpu().numpy(), qo)
    assert np.array_equal(xqs.cpu().numpy(), so)
    assert np.array_equal(xp.cpu().numpy(), qo[src_o])
    assert np.array_equal(xps.cpu().numpy(), so[src_o])
    assert np.array_equal(offsets.cpu().numpy(), off_o)
    assert np.array_equal(s2r.cpu().numpy(), s2r_o)
    assert np.array_equal(roww.cpu().numpy(), w_np.reshape(-1)[np.argsort(s2r_o)])


def test_permute_flags_out_of_range_ids_without_writing_outside():
    T, k, E, H = 128, 4, 16, 256
    ids_np, w_np = _ids_from_oracle(T, k, E, seed=10)
    ids_np = ids_np.copy()
    ids_np[5, 2] = 99                         # out of range: counted nowhere, flagged
    ids_np[77, 0] = -3
    R = T * k
    guard = torch.full((R + 64, H), 7, dtype=torch.bfloat16, device=DEV)
    xp = guard[:R]
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(R, dtype=torch.int32, device=DEV)
    s2r = torch.empty(R, dtype=torch.int32, device=DEV)
    ws = torch.empty(N.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    x = torch.randn(T, H, generator=_gen(6), device=DEV).to(torch.bfloat16)
    N.moe_permute(T, k, E, H, torch.from_numpy(ids_np).to(DEV), None, x, N.MOE_BF16, None, xp, None,
                  offsets, src, s2r, None, ws, status)
    assert N.moe_read_device_status(status) & N.MOE_DEVSTAT_BAD_EXPERT_ID
    s2r_np = s2r.cpu().numpy()
    assert s2r_np[5 * k + 2] == -1 and s2r_np[77 * k + 0] == -1
    assert torch.all(guard[R:] == 7)         # nothing written past the output


# ---------------------------------------------------- grouped SwiGLU GEMM
def _segments(sizes):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return off


def _ref_grouped(a, w13, w2, off, row_w):
    a64, w13_64, w2_64 = np64(a), np64(w13), np64(w2)
    rw = np32(row_w).astype(np.float64) if row_w is not None else None
    out = np.zeros((a.shape[0], w2.shape[1]))
    hs = np.zeros((a.shape[0], w2.shape[2]))
    for g in range(len(off) - 1):
        s, e = off[g], off[g + 1]
        if e == s:
            continue
        hs[s:e] = oracle.swiglu_hidden(a64[s:e], w13_64[g])
        o = oracle.swiglu_ffn(a64[s:e], w13_64[g], w2_64[g])
        out[s:e] = o * (rw[s:e, None] if rw is not None else 1.0)
    return out, hs


@pytest.mark.parametrize("H,I,sizes", [
    (512, 256, [0, 1, 15, 16, 17, 100, 255, 256, 257, 600, 0, 33]),
    (256, 128, [64]),
    (7168, 2048, [300, 77]),
    (2048, 1408, [384, 0, 5, 513]),
    (512, 256, [1200, 2, 8]),
    # segments of more than 8 token blocks of 256: the tile order's last,
    # partial chunk of token blocks (5000 rows = 20 blocks = 8 + 8 + 4)
    (512, 256, [2300, 5000, 3]),
    (7168, 2048, [2100, 0, 17]),
    # segments just past a multiple of 256 rows: balanced token blocks of
    # 136-144 rows (two for 257-288 rows, three for 513-545)
    (512, 256, [257, 270, 272, 273, 288, 289, 544, 545, 530, 0, 256]),
    (7168, 2048, [270, 282, 256, 520, 288]),
])
def test_grouped_swiglu_bf16(H, I, sizes):
    G = len(sizes)
    off = _segments(sizes)
    rows = int(off[-1])
    g = _gen(H + I)
    a = torch.randn(rows, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(rows, generator=g, device=DEV) + 0.5
    h = torch.empty(rows, I, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, H, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_grouped_swiglu(rows, H, w13, w2, N.MOE_BF16, G, I, a, torch.from_numpy(off).to(DEV), row_w,
                         h, out, dev_status=status)
    assert N.moe_read_device_status(status) == 0
    ref, href = _ref_grouped(a, w13, w2, off, row_w)
    eh, eo = rel_err(np64(h), href), rel_err(np64(out), ref)
    print(f"H={H} I={I} sizes={sizes}: h err {eh:.2e}, out err {eo:.2e}")
    assert eh < 1e-2 and eo < BF16_TOL


@pytest.mark.parametrize("H,I,I_s,sizes,T", [
    (512, 256, 384, [0, 17, 300, 5, 256, 0, 129], 300),
    (7168, 2048, 2048, [300, 77, 512, 1], 1000),
    (512, 256, 384, [280, 1, 0, 530, 288], 270),     # routed and shared rows just past a full block
    (2048, 1408, 2816, [384, 0, 5, 513], 129),
])
def test_routed_and_shared_in_one_launch(H, I, I_s, sizes, T):
    """moe_*_with_shared: the routed segments and a shared FFN of T rows (its
    own I_s, weight 1) in one launch per GEMM. Every output tile is computed as
    in the separate launches, so the results must be bit-identical to them,
    and within the bf16 tolerance of the oracle."""
    G = len(sizes)
    off = _segments(sizes)
    R = int(off[-1])
    g = _gen(H + I + I_s + T)
    xp = torch.randn(R, H, generator=g, device=DEV).to(torch.bfloat16)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw13 = (torch.randn(1, 2 * I_s, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw2 = (torch.randn(1, H, I_s, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(R, generator=g, device=DEV) + 0.5
    offd = torch.from_numpy(off).to(DEV)
    e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=DEV)
    h, sh_h, o, sh_o = e(R, I), e(T, I_s), e(R, H), e(T, H)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_gate_up_swiglu_with_shared(R, H, w13, N.MOE_BF16, G, I, xp, offd, h, T, sw13, I_s, x, sh_h,
                                     dev_status=status)
    N.moe_down_proj_with_shared(R, H, w2, N.MOE_BF16, G, I, h, offd, row_w, o, T, sw2, I_s, sh_h, sh_o,
                                dev_status=status)
    h2, sh_h2, o2, sh_o2 = e(R, I), e(T, I_s), e(R, H), e(T, H)
    N.moe_gate_up_swiglu(R, H, w13, N.MOE_BF16, G, I, xp, offd, h2)
    N.moe_gate_up_swiglu(T, H, sw13, N.MOE_BF16, 1, I_s, x, None, sh_h2)
    N.moe_down_proj(R, H, w2, N.MOE_BF16, G, I, h2, offd, row_w, o2)
    N.moe_down_proj(T, H, sw2, N.MOE_BF16, 1, I_s, sh_h2, None, None, sh_o2)
    assert N.moe_read_device_status(status) == 0
    for got, sep, name in ((h, h2, "h"), (sh_h, sh_h2, "shared h"), (o, o2, "out"), (sh_o, sh_o2, "shared out")):
        assert torch.equal(got, sep), f"{name} differs from the separate launches"
    ref, href = _ref_grouped(xp, w13, w2, off, row_w)
    sref, shref = _ref_grouped(x, sw13, sw2, np.array([0, T], np.int32), None)
    errs = [rel_err(np64(h), href), rel_err(np64(o), ref), rel_err(np64(sh_h), shref), rel_err(np64(sh_o), sref)]
    print(f"H={H} I={I} I_s={I_s}: errors {[f'{v:.2e}' for v in errs]}")
    assert errs[0] < 1e-2 and errs[2] < 1e-2 and errs[1] < BF16_TOL and errs[3] < BF16_TOL


@pytest.mark.parametrize("H,I,I_s,sizes,T", [
    (512, 256, 384, [0, 17, 300, 5, 256, 0, 129], 300),
    (7168, 2048, 2048, [2100, 0, 17, 260, 513], 1000),
    (2048, 1408, 2816, [384, 0, 5, 513], 129),
])
def test_swiglu_ffn_one_launch_equals_two_launches(H, I, I_s, sizes, T):
    """moe_swiglu_ffn_with_shared runs both GEMMs, routed and shared, in one
    launch whose down tiles wait on per-token-block counters of the gate/up
    tiles: h, out, shared h and shared out must be bit-identical to
    moe_gate_up_swiglu_with_shared followed by moe_down_proj_with_shared
    (segments over 8 token blocks, empty segments, I_s != I), and out within
    the bf16 tolerance of the oracle. Run twice on the same scratch: the
    counters are zeroed by each call."""
    G = len(sizes)
    off = _segments(sizes)
    R = int(off[-1])
    g = _gen(H + I + I_s + T + 1)
    xp = torch.randn(R, H, generator=g, device=DEV).to(torch.bfloat16)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw13 = (torch.randn(1, 2 * I_s, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw2 = (torch.randn(1, H, I_s, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(R, generator=g, device=DEV) + 0.5
    offd = torch.from_numpy(off).to(DEV)
    e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=DEV)
    h, sh_h, o, sh_o = e(R, I), e(T, I_s), e(R, H), e(T, H)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_gate_up_swiglu_with_shared(R, H, w13, N.MOE_BF16, G, I, xp, offd, h, T, sw13, I_s, x, sh_h,
                                     dev_status=status)
    N.moe_down_proj_with_shared(R, H, w2, N.MOE_BF16, G, I, h, offd, row_w, o, T, sw2, I_s, sh_h, sh_o,
                                dev_status=status)
    sync = torch.empty(N.moe_swiglu_ffn_sync_size(R, G, T), dtype=torch.uint8, device=DEV)
    for _ in range(2):
        h2, sh_h2, o2, sh_o2 = e(R, I), e(T, I_s), e(R, H), e(T, H)
        N.moe_swiglu_ffn_with_shared(R, H, w13, w2, G, I, xp, offd, row_w, h2, o2, T, sw13, sw2, I_s, x,
                                     sh_h2, sh_o2, sync, dev_status=status)
        assert N.moe_read_device_status(status) == 0
        for got, ref, name in ((h2, h, "h"), (sh_h2, sh_h, "shared h"), (o2, o, "out"), (sh_o2, sh_o, "shared out")):
            assert torch.equal(got, ref), f"{name} differs from the two launches"
    ref, _ = _ref_grouped(xp, w13, w2, off, row_w)
    assert rel_err(np64(o2), ref) < BF16_TOL


@pytest.mark.parametrize("H,I,I_s,sizes,T", [
    (512, 256, 384, [0, 17, 300, 5, 256, 0, 129], 300),
    (7168, 2048, 2048, [2100, 0, 17, 260, 513], 1000),
])
def test_tiled_weights_match_row_major(H, I, I_s, sizes, T):
    """moe_tile_ffn_weights lays each weight tile the GEMMs load in one step
    out contiguously (checked against a reshape of the row-major tensor), and
    the grouped GEMMs read the tiled copies to the same h and outputs, bit for
    bit, as the row-major weights: two launches, the one-launch FFN and the
    gathering gate/up GEMM."""
    G = len(sizes)
    off = _segments(sizes)
    R = int(off[-1])
    g = _gen(H + I + 3 * T)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    src = torch.randint(0, T, (R,), generator=g, device=DEV, dtype=torch.int32)
    xp = x[src.long()].contiguous()
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw13 = (torch.randn(1, 2 * I_s, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    sw2 = (torch.randn(1, H, I_s, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(R, generator=g, device=DEV) + 0.5
    offd = torch.from_numpy(off).to(DEV)
    # w2: [g, b, kb, 256 rows, 64]; w13: [g, f, kb, (gate | up), 128 rows, 64]
    tiles2 = lambda w: w.reshape(w.shape[0], w.shape[1] // 256, 256, w.shape[2] // 64, 64).permute(0, 1, 3, 2, 4)
    tiles13 = lambda w: w.reshape(w.shape[0], 2, w.shape[1] // 256, 128, w.shape[2] // 64, 64).permute(0, 2, 4, 1, 3, 5)
    t13, t2, ts13, ts2 = (torch.empty_like(w) for w in (w13, w2, sw13, sw2))
    N.moe_tile_ffn_weights(H, w13, w2, G, I, t13, t2)
    N.moe_tile_ffn_weights(H, sw13, sw2, 1, I_s, ts13, ts2)
    assert torch.equal(t13.reshape(-1), tiles13(w13).reshape(-1))
    assert torch.equal(t2.reshape(-1), tiles2(w2).reshape(-1))
    assert torch.equal(ts13.reshape(-1), tiles13(sw13).reshape(-1))
    assert torch.equal(ts2.reshape(-1), tiles2(sw2).reshape(-1))
    e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    outs = []
    for a13, a2, s13, s2, tl in ((w13, w2, sw13, sw2, False), (t13, t2, ts13, ts2, True)):
        h, sh_h, o, sh_o = e(R, I), e(T, I_s), e(R, H), e(T, H)
        N.moe_gate_up_swiglu_with_shared(R, H, a13, N.MOE_BF16, G, I, xp, offd, h, T, s13, I_s, x, sh_h,
                                         dev_status=status, tiled=tl)
        N.moe_down_proj_with_shared(R, H, a2, N.MOE_BF16, G, I, h, offd, row_w, o, T, s2, I_s, sh_h, sh_o,
                                    dev_status=status, tiled=tl)
        outs.append((h, sh_h, o, sh_o))
    sync = torch.empty(N.moe_swiglu_ffn_sync_size(R, G, T), dtype=torch.uint8, device=DEV)
    h, sh_h, o, sh_o = e(R, I), e(T, I_s), e(R, H), e(T, H)
    N.moe_swiglu_ffn_with_shared(R, H, t13, t2, G, I, xp, offd, row_w, h, o, T, ts13, ts2, I_s, x, sh_h, sh_o,
                                 sync, dev_status=status, tiled=True)
    outs.append((h, sh_h, o, sh_o))
    h_gat = e(R, I)
    N.moe_gate_up_swiglu_gather(R, H, t13, G, I, x, T, src, offd, h_gat, dev_status=status, tiled=True)
    torch.cuda.synchronize()
    assert N.moe_read_device_status(status) == 0
    assert torch.equal(h_gat, outs[0][0])
    for got in outs[1:]:
        for a, b in zip(got, outs[0]):
            assert torch.equal(a, b)


def test_swiglu_ffn_rejects_e4m3_and_short_scratch():
    """The one-launch FFN is bf16 only, and its scratch must hold a counter
    per token block (checked on the host, nothing launched)."""
    R, H, I, T, G = 64, 256, 128, 16, 4
    z = lambda *shape, dt=torch.bfloat16: torch.zeros(*shape, dtype=dt, device=DEV)
    offd = torch.tensor([0, 16, 32, 48, 64], dtype=torch.int32, device=DEV)
    args = [R, H, z(G, 2 * I, H), z(G, H, I), G, I, z(R, H), offd, None, z(R, I), z(R, H), T,
            z(1, 2 * I, H), z(1, H, I), I, z(T, H), z(T, I), z(T, H)]
    n = N.moe_swiglu_ffn_sync_size(R, G, T)
    with pytest.raises(N.MoEError):
        N.moe_swiglu_ffn_with_shared(*args, torch.empty(n - 4, dtype=torch.uint8, device=DEV))
    lib = N.load_library()
    w = N.FFNWeights(args[2].data_ptr(), args[3].data_ptr(), None, None, N.MOE_E4M3, G, I)
    sw = N.FFNWeights(args[12].data_ptr(), args[13].data_ptr(), None, None, N.MOE_E4M3, 1, I)
    sync = torch.empty(n, dtype=torch.uint8, device=DEV)
    st = lib.moe_swiglu_ffn_with_shared(R, H, ctypes.byref(w), args[6].data_ptr(), offd.data_ptr(), None,
                                        args[9].data_ptr(), args[10].data_ptr(), T, ctypes.byref(sw),
                                        args[15].data_ptr(), args[16].data_ptr(), args[17].data_ptr(),
                                        sync.data_ptr(), n, None, None)
    assert st != 0


def test_grouped_swiglu_bf16_single_group_no_offsets():
    rows, H, I = 300, 512, 384
    g = _gen(77)
    a = torch.randn(rows, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(1, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(1, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    h = torch.empty(rows, I, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, H, dtype=torch.bfloat16, device=DEV)
    N.moe_grouped_swiglu(rows, H, w13, w2, N.MOE_BF16, 1, I, a, None, None, h, out)
    ref, _ = _ref_grouped(a, w13, w2, np.array([0, rows]), None)
    assert rel_err(np64(out), ref) < BF16_TOL


@pytest.mark.parametrize("H,I,sizes", [
    (512, 256, [0, 1, 8, 31, 32, 33, 70, 16]),
    (7168, 2048, [9, 3, 40]),
])
def test_grouped_swiglu_e4m3(H, I, sizes):
    G = len(sizes)
    off = _segments(sizes)
    rows = int(off[-1])
    g = _gen(H + I + 1)
    a = torch.randn(rows, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(rows, generator=g, device=DEV) + 0.5
    q13 = torch.empty(G, 2 * I, H, dtype=torch.uint8, device=DEV)
    s13 = torch.empty(G, 2 * I // 128, H // 128, dtype=torch.float32, device=DEV)
    q2 = torch.empty(G, H, I, dtype=torch.uint8, device=DEV)
    s2 = torch.empty(G, H // 128, I // 128, dtype=torch.float32, device=DEV)
    N.moe_quantize_blocks(G, 2 * I, H, w13, q13, s13)
    N.moe_quantize_blocks(G, H, I, w2, q2, s2)
    aq = torch.empty(rows, H, dtype=torch.uint8, device=DEV)
    as_ = torch.empty(rows, H // 128, dtype=torch.float32, device=DEV)
    N.moe_quantize_rows(rows, H, a, aq, as_)
    h = torch.empty(rows, I, dtype=torch.uint8, device=DEV)
    hs = torch.empty(rows, I // 128, dtype=torch.float32, device=DEV)
    out = torch.empty(rows, H, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_grouped_swiglu(rows, H, q13, q2, N.MOE_E4M3, G, I, aq, torch.from_numpy(off).to(DEV), row_w,
                         h, out, w13_scale=s13, w2_scale=s2, a_scale=as_, h_scale_ws=hs, dev_status=status)
    assert N.moe_read_device_status(status) == 0
    a32, rw = np32(a), np32(row_w).astype(np.float64)
    ref = np.zeros((rows, H))
    for gi in range(G):
        s, e = off[gi], off[gi + 1]
        if e > s:
            ref[s:e] = O._swiglu_fp8(oracle.fp8_qdq_rows(a32[s:e]), np32(w13[gi]), np32(w2[gi])) * rw[s:e, None]
    err = rel_err(np64(out), ref)
    print(f"E4M3 H={H} I={I}: out err {err:.2e}")
    assert err < FP8_TOL


# --------------------------------------------------------------- combine
@pytest.mark.parametrize("weighted,shared", [(True, True), (False, True), (True, False)])
def test_combine(weighted, shared):
    T, k, H = 300, 6, 512
    g = _gen(8)
    eo = torch.randn(T * k, H, generator=g, device=DEV).to(torch.bfloat16)
    perm = torch.randperm(T * k, generator=g, device=DEV).to(torch.int32)
    tw = torch.rand(T, k, generator=g, device=DEV) if weighted else None
    sh = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16) if shared else None
    y = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    N.moe_combine(T, k, H, eo, perm, tw, sh, y)
    ref = oracle.combine(np64(eo), perm.cpu().numpy(), k, np32(tw) if weighted else None,
                         np64(sh) if shared else None)
    # fp32 sum, one bf16 rounding: within half an ulp of bf16 (2^-8 relative)
    assert np.all(np.abs(np64(y) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


def test_combine_full_size_sampled_tokens():
    """The V3 shape (T = 8192, k = 8, H = 7168: 1.2 GB moved in one launch):
    every token combined on the GPU; the first, the last and 62 random tokens
    compared on every feature with the oracle's combine of those tokens."""
    T, k, H = 8192, 8, 7168
    g = _gen(9)
    eo = torch.randn(T * k, H, generator=g, device=DEV).to(torch.bfloat16)
    perm = torch.randperm(T * k, generator=g, device=DEV).to(torch.int32)
    tw = torch.rand(T, k, generator=g, device=DEV)
    sh = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    y = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    N.moe_combine(T, k, H, eo, perm, tw, sh, y)
    rng = np.random.default_rng(3)
    S = np.unique(np.concatenate([[0, T - 1], rng.choice(np.arange(1, T - 1), 62, replace=False)]))
    rows = perm.cpu().numpy().reshape(T, k)[S].reshape(-1)          # the sampled tokens' rows, slot order
    St = torch.from_numpy(S).to(DEV)
    ref = oracle.combine(np64(eo[torch.from_numpy(rows).to(DEV)]), np.arange(len(rows)), k,
                         np32(tw[St]), np64(sh[St]))
    got = np64(y[St])
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


# ----------------------------------------------------------- bias update
def test_bias_update_bit_exact_ten_steps():
    E, T, k, gamma = 256, 8192, 8, 0.001
    rng = np.random.default_rng(12)
    bias_np = (rng.random(E) * 0.1 - 0.05).astype(np.float32)
    bias = torch.from_numpy(bias_np).to(DEV)
    cv = torch.empty(1, dtype=torch.float32, device=DEV)
    for step in range(10):
        c = rng.multinomial(T * k, np.ones(E) / E).astype(np.int32)
        if step == 3:
            c[:] = T * k // E                  # exactly balanced: nothing moves
        counts = torch.from_numpy(c).to(DEV)
        N.moe_bias_update(E, T, k, counts, bias, gamma, cv)
        bias_np = oracle.bias_update(c, bias_np, gamma, T, k)
        assert np.array_equal(bias.cpu().numpy(), bias_np)
        assert abs(float(cv.item()) - oracle.load_cv(c)) <= 1e-6 * max(1.0, oracle.load_cv(c))


# ------------------------------------------- permutation fused into GEMM 1
def test_gate_up_gather_matches_permuted_copy_and_oracle():
    T, k, E, H, I = 1500, 6, 16, 512, 256
    ids_np, w_np = _ids_from_oracle(T, k, E, seed=21)
    off_np, src_np, _ = oracle.permute(ids_np, E)
    R = T * k
    g = _gen(22)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(E, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    src = torch.from_numpy(src_np.astype(np.int32)).to(DEV)
    off = torch.from_numpy(off_np.astype(np.int32)).to(DEV)
    xp = x[src.long()].contiguous()
    h_ref = torch.empty(R, I, dtype=torch.bfloat16, device=DEV)
    h_gat = torch.empty(R, I, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_gate_up_swiglu(R, H, w13, N.MOE_BF16, E, I, xp, off, h_ref)
    N.moe_gate_up_swiglu_gather(R, H, w13, E, I, x, T, src, off, h_gat, dev_status=status)
    assert N.moe_read_device_status(status) == 0
    assert torch.equal(h_gat, h_ref)             # same tiles, same data: bit-identical
    x64, w64 = np64(x), np64(w13)
    href = np.zeros((R, I))
    for e in range(E):
        s, t = off_np[e], off_np[e + 1]
        href[s:t] = oracle.swiglu_hidden(x64[src_np[s:t]], w64[e])
    assert rel_err(np64(h_gat), href) < 1e-2


def test_gate_up_gather_flags_bad_rows():
    T, k, E, H, I = 200, 4, 16, 256, 128
    ids_np, _ = _ids_from_oracle(T, k, E, seed=23)
    off_np, src_np, _ = oracle.permute(ids_np, E)
    src_np = src_np.astype(np.int32).copy()
    src_np[7] = T + 5                             # outside x: flagged, never read
    g = _gen(24)
    x = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(E, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    h = torch.empty(T * k, I, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    N.moe_gate_up_swiglu_gather(T * k, H, w13, E, I, x, T, torch.from_numpy(src_np).to(DEV),
                                torch.from_numpy(off_np.astype(np.int32)).to(DEV), h, dev_status=status)
    assert N.moe_read_device_status(status) & N.MOE_DEVSTAT_BAD_EXPERT_ID


# -------------------------------------------------- bounded waits time out
def test_wait_limit_runs_out_then_the_same_call_is_correct():
    """With a wait limit of a few nanoseconds every wait of the grouped GEMM
    that does not succeed at once gives up: the kernel sets MOE_DEVSTAT_TIMEOUT
    in its status word (moe_read_device_status maps it to
    MOE_ERR_DEVICE_TIMEOUT), drains its in-flight copies and MMAs, frees its
    tensor memory and returns, without a trap. The context stays usable: the
    same call with the default limit on the same stream matches the oracle."""
    H, I, sizes = 512, 256, [300, 17, 0, 129]
    G = len(sizes)
    off = _segments(sizes)
    rows = int(off[-1])
    g = _gen(4242)
    a = torch.randn(rows, H, generator=g, device=DEV).to(torch.bfloat16)
    w13 = (torch.randn(G, 2 * I, H, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(G, H, I, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    row_w = torch.rand(rows, generator=g, device=DEV) + 0.5
    offd = torch.from_numpy(off).to(DEV)
    h = torch.empty(rows, I, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(rows, H, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert N.moe_wait_limit_ns() == 2_000_000_000
    N.moe_set_wait_limit_ns(5)
    try:
        assert N.moe_wait_limit_ns() == 5
        N.moe_grouped_swiglu(rows, H, w13, w2, N.MOE_BF16, G, I, a, offd, row_w, h, out, dev_status=status)
        raw = N.moe_read_device_status(status)
    finally:
        N.moe_set_wait_limit_ns(0)
    assert N.moe_wait_limit_ns() == 2_000_000_000
    assert raw == N.MOE_DEVSTAT_TIMEOUT, raw
    code = ctypes.c_int32(0)
    assert N.load_library().moe_read_device_status(
        ctypes.c_void_p(status.data_ptr()), ctypes.byref(code),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == N.MOE_ERR_DEVICE_TIMEOUT
    status.zero_()
    N.moe_grouped_swiglu(rows, H, w13, w2, N.MOE_BF16, G, I, a, offd, row_w, h, out, dev_status=status)
    assert N.moe_read_device_status(status) == 0
    ref, href = _ref_grouped(a, w13, w2, off, row_w)
    assert rel_err(np64(h), href) < 1e-2 and rel_err(np64(out), ref) < BF16_TOL

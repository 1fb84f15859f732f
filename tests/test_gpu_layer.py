"""End-to-end parity of the MoE layer forward (needs a B200).

Routing is compared id for id on every token whose k-th / (k+1)-th selection
scores (or g-th / (g+1)-th group scores) are at least 1e-5 apart in the
oracle; closer tokens are excluded and counted. Outputs are compared as
max|y - y_oracle| / max|y_oracle| over the compared tokens."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import get_config, tiny_grouped_config, make_inputs
from mixture_experts_layer_limited_b200 import MoELayer, LayerSpec
from mixture_experts_layer_limited_b200 import native as N

from gpu_util import (np64, np32, rel_err, oracle_route, near_tie_mask, routing_mismatch,
                      describe_mismatch, BF16_TOL, FP8_TOL)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(cfg, inp, T_max=None):
    return MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                    inp.bias, T_max or cfg.T)


def _check_permutation_properties(layer, T, k, E):
    """Properties of the permutation that hold at any size."""
    ids = layer.ids[:T].cpu().numpy()
    off = layer.offsets.cpu().numpy()
    src = layer.src_token[:T * k].cpu().numpy()
    s2r = layer.slot_to_row[:T * k].cpu().numpy()
    counts = layer.counts.cpu().numpy()
    assert off[0] == 0 and off[-1] == T * k and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.diff(off), counts)
    assert np.array_equal(np.bincount(ids.ravel(), minlength=E), counts)
    assert np.array_equal(np.sort(s2r), np.arange(T * k))
    assert np.array_equal(src[s2r], np.repeat(np.arange(T), k))
    seg_of_row = np.repeat(np.arange(E), np.diff(off))
    assert np.array_equal(seg_of_row[s2r], ids.ravel())
    for e in range(E):                        # ascending tokens inside each segment
        assert np.all(np.diff(src[off[e]:off[e + 1]]) > 0)


def _oracle_tokens(cfg, inp, toks, feats=None, fp8=False, threads=1):
    """Oracle routing + output for the given tokens (and features); the
    experts are evaluated on `threads` host threads."""
    x64 = np64(inp.x[toks])
    L = oracle.gate_logits(x64, np64(inp.gate)).astype(np.float32)
    bias = np32(inp.bias) if inp.bias is not None else None
    r = oracle_route(L, cfg, bias)
    def ew(e):
        return np32(inp.w13[e]), np32(inp.w2[e])

    shared = (np32(inp.sw13), np32(inp.sw2)) if inp.sw13 is not None else None
    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            y = oracle.moe_forward(x64, r, ew, shared, fp8=fp8, out_features=feats, map_fn=ex.map)
    else:
        y = oracle.moe_forward(x64, r, ew, shared, fp8=fp8, out_features=feats)
    return r, y


def _host_threads():
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    return max(1, min(16, n))


TOKEN_BLOCK = 256      # token rows per grouped-GEMM tile (bf16)
CHUNK_BLOCKS = 8       # token blocks per rasterisation chunk


def coverage_tokens(layer, T, k, E, n_min=256, seed=0):
    """Tokens whose full output rows are compared with the oracle: tokens 0
    and T-1; one token of every expert segment that received rows (so every
    expert's weights are exercised); the tokens of the first and last rows of
    the longest segment; for every segment longer than 8 token blocks, the
    tokens of the first and last rows of its last token block (the grouped
    GEMM's last, partial chunk of token blocks); then random tokens up to
    n_min. Chosen from the GPU's permutation, which the caller has already
    checked for its invariants."""
    off = layer.offsets.cpu().numpy().astype(np.int64)
    src = layer.src_token[:T * k].cpu().numpy().astype(np.int64)
    counts = np.diff(off)
    rng = np.random.default_rng(seed)
    toks = {0, T - 1}
    for e in range(E):
        if counts[e] > 0:
            toks.add(int(src[off[e] + rng.integers(counts[e])]))
    e_long = int(np.argmax(counts))
    toks |= {int(src[off[e_long]]), int(src[off[e_long + 1] - 1])}
    tail = 0
    for e in np.nonzero(counts > CHUNK_BLOCKS * TOKEN_BLOCK)[0]:
        n = int(counts[e])
        ntb = -(-n // TOKEN_BLOCK)
        bn = -(-(-(-n // ntb)) // 16) * 16
        toks |= {int(src[off[e] + (ntb - 1) * bn]), int(src[off[e + 1] - 1])}
        tail += 1
    extra = [t for t in rng.permutation(T) if t not in toks]
    toks |= set(int(t) for t in extra[:max(0, n_min - len(toks))])
    return np.array(sorted(toks)), tail


def _compare_full_rows(cfg, inp, layer, y, toks, tol, fp8=False):
    """Every feature of the given tokens' outputs against the oracle; routing
    ids on the same tokens; near ties excluded and counted."""
    r, yref = _oracle_tokens(cfg, inp, toks, fp8=fp8, threads=_host_threads())
    flagged = near_tie_mask(r)
    ids_g = layer.ids[torch.as_tensor(toks, device=DEV)].cpu().numpy()
    mism = routing_mismatch(ids_g, r)
    assert not np.any(mism & ~flagged), describe_mismatch(ids_g, r, np.nonzero(mism & ~flagged)[0])
    ok = ~flagged & ~mism
    yg = np64(y[torch.as_tensor(toks, device=DEV)])
    err = rel_err(yg[ok], yref[ok])
    assert np.all(np.isfinite(yg))
    return err, int(flagged.sum()), int(ok.sum())


@pytest.mark.parametrize("name", ["tiny", "tiny_grouped", "v2lite"])
def test_layer_full_oracle(name):
    cfg = tiny_grouped_config() if name == "tiny_grouped" else get_config(name)
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, cfg.T, cfg.k, cfg.E)
    r, yref = _oracle_tokens(cfg, inp, np.arange(cfg.T))
    flagged = near_tie_mask(r)
    ids_g = layer.ids[:cfg.T].cpu().numpy()
    mism = routing_mismatch(ids_g, r)
    assert not np.any(mism & ~flagged), describe_mismatch(ids_g, r, np.nonzero(mism & ~flagged)[0])
    ok = ~flagged & ~mism
    err = rel_err(np64(y)[ok], yref[ok])
    print(f"{name}: err {err:.2e}, near-tie tokens excluded {int(flagged.sum())}")
    assert err < BF16_TOL


def test_layer_v3_full_size_every_expert_all_features():
    """The V3 layer at its full size (T = 8192): >= 256 tokens covering every
    expert segment, tokens 0 and T-1 and the ends of the longest segment,
    compared with the oracle on all 7168 features."""
    cfg = get_config("v3")
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, cfg.T, cfg.k, cfg.E)
    toks, _ = coverage_tokens(layer, cfg.T, cfg.k, cfg.E, seed=31)
    err, excl, n = _compare_full_rows(cfg, inp, layer, y, toks, BF16_TOL)
    print(f"v3 T=8192: {n} tokens x {cfg.H} features compared, err {err:.2e}, near ties excluded {excl}")
    assert len(toks) >= 256 and err < BF16_TOL


def test_layer_v3_fp8_decode_all_tokens_all_features():
    cfg = get_config("v3_fp8_decode")
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, cfg.T, cfg.k, cfg.E)
    # the activation codes the permutation carried are the oracle's bytes
    qo, so = oracle.fp8_quantize_rows(np32(inp.x))
    assert np.array_equal(layer.xq[:cfg.T].cpu().numpy(), qo)
    assert np.array_equal(layer.xs[:cfg.T].cpu().numpy(), so)
    toks = np.arange(cfg.T)
    err, excl, n = _compare_full_rows(cfg, inp, layer, y, toks, FP8_TOL, fp8=True)
    print(f"v3 fp8 decode: {n} tokens x {cfg.H} features compared, err {err:.2e}, near ties excluded {excl}")
    assert err < FP8_TOL


def test_layer_v3_skewed_bias_loop():
    cfg = get_config("v3_skewed")
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    T, E, k = cfg.T, cfg.E, cfg.k
    # (a) ten bias steps on identical fp32 logits: routing, counts and the
    #     bias trajectory must be bit-exact
    L32 = oracle.gate_logits(np64(inp.x), np64(inp.gate)).astype(np.float32)
    L_dev = torch.from_numpy(L32).to(DEV)
    bias_o = np32(inp.bias).copy()
    cvs = []
    hot = []
    for step in range(cfg.bias_steps + 1):
        layer.route(None, logits_in=L_dev)
        r = oracle.route_from_logits(L32, k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                     cfg.norm_topk_prob, cfg.scale, bias_o)
        ids_g = layer.ids[:T].cpu().numpy()
        assert np.array_equal(ids_g, r.ids), f"step {step}"
        assert np.array_equal(layer.counts.cpu().numpy(), r.counts)
        cvs.append(oracle.load_cv(r.counts))
        hot.append(float(r.counts[:cfg.skew_experts].sum()) / (T * k))
        if step == cfg.bias_steps:
            break
        layer.bias_step(T, cfg.gamma)
        torch.cuda.synchronize()
        bias_o = oracle.bias_update(r.counts, bias_o, cfg.gamma, T, k)
        assert np.array_equal(layer.bias.cpu().numpy(), bias_o), f"step {step}"
        assert abs(float(layer.load_cv.item()) - cvs[-1]) < 1e-6
    print("load CV per step:", " ".join(f"{c:.4f}" for c in cvs))
    print("share of experts 0-15 per step:", " ".join(f"{h:.3f}" for h in hot))
    # the load CV drops step over step (never rises) and ends below its start
    assert all(b <= a for a, b in zip(cvs, cvs[1:])), cvs
    assert cvs[cfg.bias_steps] < cvs[0]
    # (b) a full forward from x at this size with the final bias: >= 256 tokens
    #     covering every expert segment (and the last token blocks of the hot
    #     experts' long segments) against the oracle on all features
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, T, k, E)
    inp.bias = layer.bias.clone()             # the bias the forward used
    toks, tail = coverage_tokens(layer, T, k, E, seed=33)
    err, excl, n = _compare_full_rows(cfg, inp, layer, y, toks, BF16_TOL)
    print(f"v3 skewed: {n} tokens x {cfg.H} features compared ({tail} segments longer than 8 token "
          f"blocks), err {err:.2e}, near ties excluded {excl}")
    assert tail > 0 and err < BF16_TOL


def test_layer_gather_variant_matches_default():
    """The permutation fused into GEMM 1 gives the same layer output."""
    cfg = get_config("v2lite", T=1024)
    inp = make_inputs(cfg, device=DEV)
    y0 = _layer(cfg, inp).forward(inp.x).clone()
    lay = MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                   inp.bias, cfg.T, gather=True)
    y1 = lay.forward(inp.x)
    torch.cuda.synchronize()
    assert lay.device_status() == 0
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("name", ["v2lite", "v3"])
def test_layer_shared_expert_in_routed_launches_matches_separate(name):
    """The shared expert run inside the routed experts' launches (the default)
    gives the same layer output as its own launches, bit for bit."""
    cfg = get_config(name, T=1024)
    inp = make_inputs(cfg, device=DEV)
    fused = _layer(cfg, inp)
    assert fused.fuse_shared
    y0 = fused.forward(inp.x).clone()
    apart = MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                     inp.bias, cfg.T, fuse_shared=False)
    y1 = apart.forward(inp.x)
    torch.cuda.synchronize()
    assert fused.device_status() == 0 and apart.device_status() == 0
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("name", ["v2lite", "v3", "v3_skewed"])
def test_layer_one_launch_ffn_matches_two_launches(name):
    """Both expert GEMMs in one launch (tiles from a counter, down tiles waiting
    on their token block's gate/up tiles) give the layer output of the two
    launches bit for bit, at the full sizes of three layers."""
    cfg = get_config(name)
    inp = make_inputs(cfg, device=DEV)
    mk = lambda fuse: MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                               inp.bias, cfg.T, fuse_ffn=fuse)
    one = mk(True)
    assert any(n == "ffn" for n, _ in one.stages(inp.x))
    y1 = one.forward(inp.x).clone()
    torch.cuda.synchronize()
    assert one.device_status() == 0
    del one
    two = mk(False)
    y2 = two.forward(inp.x)
    torch.cuda.synchronize()
    assert two.device_status() == 0
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("name,fuse", [("tiny", None), ("v2lite", None), ("v3", None), ("v3_skewed", True)])
def test_layer_tiled_weights_match_row_major(name, fuse):
    """The layer holding its bf16 weights tiled (the default) gives the output
    of the same layer reading the caller's row-major weights, bit for bit, at
    the full sizes (both GEMM forms: two launches, and one launch for the
    skewed layer)."""
    cfg = get_config(name)
    inp = make_inputs(cfg, device=DEV)
    mk = lambda tiled: MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                                inp.bias, cfg.T, fuse_ffn=fuse, tiled_weights=tiled)
    lt = mk(True)
    assert lt.tiled
    y1 = lt.forward(inp.x).clone()
    torch.cuda.synchronize()
    assert lt.device_status() == 0
    del lt
    lr = mk(False)
    assert not lr.tiled and lr.w13.data_ptr() == inp.w13.data_ptr()
    y2 = lr.forward(inp.x)
    torch.cuda.synchronize()
    assert lr.device_status() == 0
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("name", ["v2lite", "v3"])
def test_host_pipeline_matches_one_forward_at_a_time(name):
    """HostPipeline overlaps each batch's copies with its neighbours' compute;
    every output must equal the plain forward of that batch, bit for bit,
    also with a bias step between forwards."""
    from mixture_experts_layer_limited_b200 import HostPipeline
    cfg = get_config(name, T=1024)
    inp = make_inputs(cfg, device=DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(77)
    xs = [torch.randn(cfg.T, cfg.H, generator=g, device=DEV).to(torch.bfloat16) for _ in range(5)]
    with_bias = inp.bias is not None

    ref_layer = _layer(cfg, inp)
    refs = []
    for x in xs:
        refs.append(ref_layer.forward(x).clone())
        if with_bias:
            ref_layer.bias_step(cfg.T, cfg.gamma, load_cv=False)

    layer = _layer(cfg, inp)
    pipe = HostPipeline(layer, cfg.T)
    x_host = [x.cpu().pin_memory() for x in xs]
    y_host = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in xs]
    step = (lambda i: layer.bias_step(cfg.T, cfg.gamma, load_cv=False)) if with_bias else None
    pipe.run(x_host, y_host, step)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    for i, (y, r) in enumerate(zip(y_host, refs)):
        assert torch.equal(y, r.cpu()), f"batch {i} differs"
    if with_bias:
        assert torch.equal(layer.bias, ref_layer.bias)


def _run_from_logits(layer, x, L):
    """The forward with routing taken from the given fp32 logits."""
    T = x.shape[0]
    layer.route(x, logits_in=L)
    for name, run in layer.stages(x)[1:]:
        run()
    return layer.y[:T]


@pytest.mark.parametrize("name", ["v2lite", "v3"])
def test_layer_collapsed_routing(name):
    """Degenerate load: every token picks the same k experts (the other
    experts get no rows at all; the k segments hold T rows each, several
    token blocks). Through the permutation, both grouped GEMMs and combine."""
    cfg = get_config(name, T=512 if name == "v2lite" else 256)
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    L = torch.full((cfg.T, cfg.E), -8.0, dtype=torch.float32, device=DEV)
    hot = torch.arange(cfg.k, device=DEV)                 # inside the first group
    L[:, hot] = 8.0 + torch.arange(cfg.k, device=DEV, dtype=torch.float32) * 0.25
    y = _run_from_logits(layer, inp.x, L)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    counts = layer.counts.cpu().numpy()
    assert sorted(np.nonzero(counts)[0].tolist()) == sorted(hot.cpu().tolist())
    assert np.all(counts[hot.cpu().numpy()] == cfg.T)
    _check_permutation_properties(layer, cfg.T, cfg.k, cfg.E)
    bias = np32(inp.bias) if inp.bias is not None else None
    r = oracle_route(np32(L), cfg, bias)
    assert np.array_equal(layer.ids[:cfg.T].cpu().numpy(), r.ids)
    rng = np.random.default_rng(5)
    feats = np.sort(rng.choice(cfg.H, 256, replace=False))
    ew = lambda e: (np32(inp.w13[e]), np32(inp.w2[e]))
    shared = (np32(inp.sw13), np32(inp.sw2)) if inp.sw13 is not None else None
    yref = oracle.moe_forward(np64(inp.x), r, ew, shared, out_features=feats)
    err = rel_err(np64(y[:, torch.as_tensor(feats, device=DEV)]), yref)
    print(f"{name} collapsed routing: err {err:.2e}")
    assert err < BF16_TOL


@pytest.mark.parametrize("name", ["tiny", "v3"])
def test_layer_single_token(name):
    """T = 1: every routed segment has one row or none."""
    cfg = get_config(name, T=1)
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, 1, cfg.k, cfg.E)
    r, yref = _oracle_tokens(cfg, inp, np.arange(1))
    assert not (near_tie_mask(r)[0]) and np.array_equal(np.sort(layer.ids[:1].cpu().numpy()), np.sort(r.ids))
    err = rel_err(np64(y), yref)
    print(f"{name} T=1: err {err:.2e}")
    assert err < BF16_TOL


@pytest.mark.parametrize("name", ["tiny", "v3"])
def test_layer_cuda_graph_replay_matches_eager(name):
    """The forward (+ bias step) captured as one CUDA graph gives the eager
    results, bit for bit, over several replays with new inputs."""
    cfg = get_config(name, T=64 if name == "tiny" else 1024)
    inp = make_inputs(cfg, device=DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    xs = [torch.randn(cfg.T, cfg.H, generator=g, device=DEV).to(torch.bfloat16) for _ in range(3)]
    gamma = cfg.gamma if inp.bias is not None else None
    eager = _layer(cfg, inp)
    refs = []
    for x in xs:
        refs.append(eager.forward(x).clone())
        if gamma is not None:
            eager.bias_step(cfg.T, gamma, load_cv=False)
    layer = _layer(cfg, inp)
    x_in = torch.empty_like(xs[0])
    x_in.copy_(xs[0])
    replay = layer.capture(x_in, gamma)
    # capture ran the forward once outside the graph (no bias step): start over
    if gamma is not None:
        layer.bias.copy_(inp.bias)
    for x, r in zip(xs, refs):
        x_in.copy_(x)
        replay()
        torch.cuda.synchronize()
        assert torch.equal(layer.y[:cfg.T], r)
    assert layer.device_status() == 0
    if gamma is not None:
        assert torch.equal(layer.bias, eager.bias)


def test_layer_v3_largest_batch():
    """T = 65536 tokens (524288 routed rows, 7.5 GB of permuted activations):
    the permutation's invariants on every row, and >= 256 tokens covering
    every expert segment and the last token blocks of every segment longer
    than 8 token blocks against the oracle on all features."""
    cfg = get_config("v3", T=65536)
    inp = make_inputs(cfg, device=DEV)
    layer = _layer(cfg, inp)
    y = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _check_permutation_properties(layer, cfg.T, cfg.k, cfg.E)
    toks, tail = coverage_tokens(layer, cfg.T, cfg.k, cfg.E, seed=65536)
    err, excl, n = _compare_full_rows(cfg, inp, layer, y, toks, BF16_TOL)
    print(f"v3 T=65536: {n} tokens x {cfg.H} features compared ({tail} segments longer than 8 token "
          f"blocks), err {err:.2e}, near ties excluded {excl}")
    assert tail > 0 and err < BF16_TOL


@pytest.mark.parametrize("name", ["tiny", "v2lite", "v3"])
def test_layer_combine_fused_into_down_gemm(name):
    """The combine inside the down GEMM (fp32 atomic adds at each row's token)
    against the oracle, and close to the default path, which rounds each
    expert's output to bf16 before the combine."""
    cfg = get_config(name) if name != "v3" else get_config("v3", T=2048)
    inp = make_inputs(cfg, device=DEV)
    y_ref_path = _layer(cfg, inp).forward(inp.x).clone()
    lay = MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                   inp.bias, cfg.T, fuse_combine=True)
    assert [n for n, _ in lay.stages(inp.x)][-1] == "down_combine"
    y = lay.forward(inp.x)
    torch.cuda.synchronize()
    assert lay.device_status() == 0
    diff = rel_err(np64(y), np64(y_ref_path))
    rng = np.random.default_rng(8)
    toks = np.arange(cfg.T) if cfg.T <= 4096 and name != "v3" else np.sort(rng.choice(cfg.T, 8, replace=False))
    feats = None if name != "v3" else np.sort(rng.choice(cfg.H, 256, replace=False))
    r, yref = _oracle_tokens(cfg, inp, toks, feats)
    flagged = near_tie_mask(r)
    ok = ~flagged & ~routing_mismatch(lay.ids[toks].cpu().numpy(), r)
    yg = np64(y[toks]) if feats is None else np64(y[toks][:, torch.as_tensor(feats, device=DEV)])
    err = rel_err(yg[ok], yref[ok])
    print(f"{name} fused combine: err {err:.2e}, vs default path {diff:.2e}")
    assert err < BF16_TOL and diff < 1e-2

"""Pins of the CPU oracle to facts outside itself (CPU only, no GPU).

Each test ties one oracle function to what the pages or the mathematics fix:
a worked example printed on a page, a closed form, a format fact, a library
routine that computes the same thing another way, or brute force on tiny
inputs. Each is chosen so a plausible slip in the oracle (a dropped term, a
wrong sign or index, a swapped operand, a biased weight) fails it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import moe_oracle as O
from moe_inputs import get_config, tiny_grouped_config, make_inputs, make_logits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- permutation
def test_permute_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "permute_worked_example.json")))
    ids = np.array(g["topk_ids"])
    E = 12
    offsets, src_token, slot_to_row = oracle.permute(ids, E)
    for e_str, toks in g["segments"].items():
        e = int(e_str)
        assert list(src_token[offsets[e]:offsets[e + 1]]) == toks
    nonempty = sorted({0} | {int(offsets[e + 1]) for e in range(E) if offsets[e + 1] > offsets[e]})
    assert nonempty == g["nonempty_offsets"]
    assert offsets[-1] == ids.size
    # inverse map: row of slot (t, j) holds token t and lies in expert ids[t, j]'s segment
    for t in range(ids.shape[0]):
        for j in range(ids.shape[1]):
            r = slot_to_row[t * ids.shape[1] + j]
            assert src_token[r] == t
            e = ids[t, j]
            assert offsets[e] <= r < offsets[e + 1]


def test_permute_is_bijection_random():
    rng = np.random.default_rng(3)
    T, k, E = 300, 6, 64
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    offsets, src_token, slot_to_row = oracle.permute(ids, E)
    assert sorted(slot_to_row.tolist()) == list(range(T * k))
    assert np.all(np.diff(offsets) >= 0) and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), np.bincount(ids.ravel(), minlength=E))
    for e in range(E):
        seg = src_token[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)          # ascending token order
        assert np.all((ids[seg] == e).any(axis=1))


# ---------------------------------------------------------------------- E4M3
def test_e4m3_format_facts():
    v = oracle.e4m3_values()
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x38] == 1.0
    assert v[0x08] == 2.0 ** -6            # smallest normal
    assert v[0x01] == 2.0 ** -9            # smallest subnormal
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    finite = v[~np.isnan(v)]
    assert len(np.unique(finite)) == 253   # +0 and -0 compare equal


def test_e4m3_rounding_ties_and_saturation():
    q = oracle.quantize_e4m3(np.array(
        [1.0625, 1.1875, 1.9375, 500.0, -470.0, 449.0, 2.0 ** -10, 3 * 2.0 ** -11,
         -1e-4, 0.0], np.float32))
    # 1.0625 ties 1.0/1.125 -> 1.0 (even); 1.1875 ties 1.125/1.25 -> 1.25 (even);
    # 1.9375 ties 1.875/2.0 -> 2.0; beyond 448 saturates; 2^-10 ties 0/2^-9 -> 0;
    # 1.5*2^-10 -> 2^-9; tiny negatives keep the sign bit.
    assert list(q) == [0x38, 0x3A, 0x40, 0x7E, 0xFE, 0x7E, 0x00, 0x01, 0x80, 0x00]


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * rng.choice([1e-3, 0.1, 1, 30, 200], 200000)).astype(np.float32)
    x = np.clip(x, -448, 448)
    ours = oracle.dequantize_e4m3(oracle.quantize_e4m3(x))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_two_e4m3_roundings_agree():
    # table search over the 256 codes vs arithmetic rounding to 3 mantissa bits
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(300000) * rng.choice([1e-4, 1e-3, 0.02, 1, 50, 300, 600], 300000)).astype(np.float32)
    grid = oracle.e4m3_values()[:127]
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)   # exact ties
    x = np.concatenate([x, mids, -mids, np.float32([0.0, -0.0, 448.0, 464.0, 465.0, 1e6])])
    a = oracle.dequantize_e4m3(oracle.quantize_e4m3(x))
    b = oracle.round_to_e4m3(x)
    assert np.array_equal(a, b)
    w = (rng.standard_normal((256, 256)) * 0.02).astype(np.float32)
    q, s = oracle.fp8_quantize_blocks(w)
    assert np.array_equal(O.fp8_dequant_blocks(q, s), oracle.fp8_qdq_blocks(w))
    qr, sr = oracle.fp8_quantize_rows(w)
    assert np.array_equal(O.fp8_dequant_rows(qr, sr), oracle.fp8_qdq_rows(w))


def test_fp8_block_quant_roundtrip_bound_and_exact_grid():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((256, 384)) * 0.02).astype(np.float32)
    q, s = oracle.fp8_quantize_blocks(w)
    assert s.shape == (2, 3)
    amax = np.abs(w.reshape(2, 128, 3, 128)).max(axis=(1, 3))
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    dq = O.fp8_dequant_blocks(q, s)
    normal = np.abs(w) >= np.repeat(np.repeat(s, 128, 0), 128, 1) * 2.0 ** -6
    err = np.abs(dq - w)[normal] / np.abs(w)[normal]
    assert err.max() <= 2.0 ** -4 + 1e-12
    # values already on the E4M3 grid x a power of two come back exactly
    grid = oracle.e4m3_values()[:127]
    g = rng.choice(grid, size=(128, 128)) * 2.0 ** -10
    g[5, 7] = 448.0 * 2.0 ** -10                 # pins the block amax
    g = np.where(rng.random(g.shape) < 0.5, -g, g).astype(np.float32)
    q2, s2 = oracle.fp8_quantize_blocks(g)
    assert s2[0, 0] == np.float32(2.0 ** -10)
    assert np.array_equal(O.fp8_dequant_blocks(q2, s2), g.astype(np.float64))
    # an all-zero block takes scale 1 and code 0
    q3, s3 = oracle.fp8_quantize_rows(np.zeros((2, 128), np.float32))
    assert np.all(s3 == 1.0) and np.all(q3 == 0)


# ------------------------------------------------------------------ router
def _brute_route(L32, k, G, g, scoring, norm, scale, bias32):
    """Independent formulation: per token, Python-sorted tuple keys."""
    T, E = L32.shape
    gsz = E // G
    ids_all, w_all = [], []
    for t in range(T):
        Lt = [float(v) for v in L32[t]]
        if scoring == "sigmoid":
            unb = [1.0 / (1.0 + math.exp(-v)) for v in Lt]
            sel = [np.float32(np.float32(u) + (np.float32(bias32[e]) if bias32 is not None else np.float32(0)))
                   for e, u in enumerate(unb)]
        else:
            m = max(Lt)
            ex = [math.exp(v - m) for v in Lt]
            s = sum(ex)
            unb = [v / s for v in ex]
            sel = [np.float32(v) for v in Lt] if (G == 1 and bias32 is None) else [np.float32(u) for u in unb]
        if G > 1:
            gsc = []
            for gi in range(G):
                mem = sorted(sel[gi * gsz:(gi + 1) * gsz], reverse=True)
                gsc.append(np.float32(mem[0] + mem[1]))
            # enumerate every subset of g groups; keep the lexicographically best
            # (scores sorted descending, then lowest indices) -- equals "top g".
            best = None
            for sub in itertools.combinations(range(G), g):
                key = (sorted([float(gsc[i]) for i in sub], reverse=True),
                       [-i for i in sub])
                if best is None or key > best[0]:
                    best = (key, sub)
            kept = set(best[1])
            cand = [e for e in range(E) if e // gsz in kept]
        else:
            cand = list(range(E))
        chosen = sorted(cand, key=lambda e: (-float(sel[e]), e))[:k]
        w = [unb[e] for e in chosen]
        if norm:
            tot = sum(w)
            w = [v / tot for v in w]
        ids_all.append(chosen)
        w_all.append([v * scale for v in w])
    return np.array(ids_all), np.array(w_all)


@pytest.mark.parametrize("case", ["softmax_g1", "sigmoid_grouped", "softmax_grouped", "coarse_ties"])
def test_route_matches_brute_force(case):
    rng = np.random.default_rng(7)
    T, E = 120, 16
    if case == "softmax_g1":
        kw = dict(k=4, n_group=1, topk_group=1, scoring="softmax", norm_topk_prob=False, scale=1.0)
        bias = None
    elif case == "softmax_grouped":
        kw = dict(k=3, n_group=4, topk_group=2, scoring="softmax", norm_topk_prob=True, scale=1.0)
        bias = None
    else:
        kw = dict(k=4, n_group=4, topk_group=2, scoring="sigmoid", norm_topk_prob=True, scale=2.5)
        bias = (rng.random(E) * 0.1 - 0.05).astype(np.float32)
    L = (rng.standard_normal((T, E)) * 1.7).astype(np.float32)
    if case == "coarse_ties":
        L = np.round(L * 2) / 2                    # many exact ties
        L = L.astype(np.float32)
        bias = np.round(bias * 20) / 20
        bias = bias.astype(np.float32)
    r = oracle.route_from_logits(L, bias32=bias, **kw)
    ids_b, w_b = _brute_route(L, kw["k"], kw["n_group"], kw["topk_group"], kw["scoring"],
                              kw["norm_topk_prob"], kw["scale"], bias)
    assert np.array_equal(r.ids, ids_b)
    np.testing.assert_allclose(r.weights, w_b, rtol=1e-12, atol=0)


def test_route_invariants_v3_shape():
    cfg = get_config("v3", T=512)
    L = make_logits(cfg).numpy()
    inp_bias = (np.random.default_rng(5).random(cfg.E) * 0.1 - 0.05).astype(np.float32)
    r = oracle.route_from_logits(L, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                 cfg.norm_topk_prob, cfg.scale, inp_bias)
    gsz = cfg.E // cfg.n_group
    for t in range(cfg.T):
        assert len(set(r.ids[t])) == cfg.k
        assert len(set(r.ids[t] // gsz)) <= cfg.topk_group
        assert set(r.ids[t] // gsz) <= set(r.kept_groups[t])
    np.testing.assert_allclose(r.weights.sum(axis=1), cfg.scale, rtol=1e-12)
    # weights are the UNBIASED sigmoid, renormalised: ratios equal sigmoid ratios
    sig = 1.0 / (1.0 + np.exp(-L.astype(np.float64)))
    ratio = r.weights[:, 1:] / r.weights[:, :1]
    sr = np.take_along_axis(sig, r.ids[:, 1:].astype(np.int64), 1) / np.take_along_axis(sig, r.ids[:, :1].astype(np.int64), 1)
    np.testing.assert_allclose(ratio, sr, rtol=1e-12)
    assert r.counts.sum() == cfg.T * cfg.k


def test_route_softmax_greedy_is_textbook_topk():
    cfg = get_config("v2lite", T=256)
    L = make_logits(cfg).numpy()
    r = oracle.route_from_logits(L, cfg.k, 1, 1, "softmax", False, 1.0)
    # textbook greedy top-k: lexsort on (index, -logit)
    for t in range(cfg.T):
        order = np.lexsort((np.arange(cfg.E), -L[t].astype(np.float64)))[:cfg.k]
        assert list(r.ids[t]) == list(order)
    # no renormalisation: weights are the softmax probabilities, which sum to 1 over E
    p = torch.softmax(torch.from_numpy(L.astype(np.float64)), dim=1).numpy()
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(r.weights, np.take_along_axis(p, r.ids.astype(np.int64), 1), rtol=1e-12)
    assert np.all(r.weights.sum(1) < 1.0)


def test_group_score_is_top2_sum_and_masked_experts_excluded():
    # 4 groups of 4 experts, keep 2 groups, pick 2 experts. Sigmoid with bias.
    # Group 0 has the single best expert but a weak runner-up; group 1 has two
    # good experts; group 2 all mediocre but high total; group 3 low.
    L = np.array([[4.0, -6.0, -6.0, -6.0,
                   2.0, 2.0, -6.0, -6.0,
                   0.5, 0.5, 0.5, 0.5,
                   -3.0, -3.0, -3.0, -3.0]], np.float32)
    bias = np.zeros(16, np.float32)
    r = oracle.route_from_logits(L, 2, 4, 2, "sigmoid", True, 1.0, bias)
    sig = 1 / (1 + np.exp(-L[0].astype(np.float64)))
    gsc = [sorted(sig[i * 4:(i + 1) * 4])[-1] + sorted(sig[i * 4:(i + 1) * 4])[-2] for i in range(4)]
    # top-2 sums: g1 (1.762) > g2 (1.245) > g0 (0.985) > g3 : keep groups 1, 2
    assert sorted(r.kept_groups[0].tolist()) == [1, 2]
    assert gsc[1] > gsc[2] > gsc[0]
    assert list(r.ids[0]) == [4, 5]
    # With a large negative bias every biased score is < 0; experts of dropped
    # groups must still never be chosen (a 0.0 fill would select them).
    bias2 = np.full(16, -0.9, np.float32)
    r2 = oracle.route_from_logits(L, 6, 4, 2, "sigmoid", True, 1.0, bias2)
    assert set(r2.ids[0] // 4) <= {1, 2}


# -------------------------------------------------------------- gate + FFN
def test_gate_logits_identity_gate():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 32))
    G = np.zeros((8, 32))
    G[np.arange(8), np.arange(8) * 3] = 1.0
    np.testing.assert_array_equal(oracle.gate_logits(x, G), x[:, np.arange(8) * 3])


def test_swiglu_closed_form():
    # x = 1, w1 = a*Id (gate rows first), w3 = b*Id (up rows), w2 = c*Id:
    # out = c * SiLU(a) * b ; SiLU(1) = 1/(1+e^-1) = 0.7310585786300049
    n = 8
    Id = np.eye(n)
    a, b, c = 1.0, 2.0, 3.0
    w13 = np.concatenate([a * Id, b * Id])
    out = oracle.swiglu_ffn(np.ones((1, n)), w13, c * Id)
    np.testing.assert_allclose(out, 3.0 * 2.0 * 0.7310585786300049, rtol=1e-15)
    # negative pre-activation: SiLU(-1) = -0.2689414213699951
    out2 = oracle.swiglu_ffn(-np.ones((1, n)), w13, c * Id)
    np.testing.assert_allclose(out2, 3.0 * (-2.0) * (-0.2689414213699951), rtol=1e-15)


def test_swiglu_hidden_closed_form_and_gate_up_order():
    # x = (ln 3, 2): w1 picks x0 (gate), w3 picks x1 (up):
    # sigmoid(ln 3) = 3/4, so h = SiLU(ln 3) * 2 = (3/4) ln 3 * 2 = 1.5 ln 3
    x = np.array([[np.log(3.0), 2.0]])
    w13 = np.array([[1.0, 0.0], [0.0, 1.0]])          # [w1; w3], I = 1
    np.testing.assert_allclose(oracle.swiglu_hidden(x, w13), [[1.5 * np.log(3.0)]], rtol=1e-15)
    # gate and up swapped: SiLU(2) * ln 3 = 2 / (1 + e^-2) * ln 3, not the same
    swapped = oracle.swiglu_hidden(x, w13[::-1])
    np.testing.assert_allclose(swapped, [[2.0 / (1.0 + np.exp(-2.0)) * np.log(3.0)]], rtol=1e-15)
    assert abs(swapped[0, 0] - 1.5 * np.log(3.0)) > 0.1
    # the expert is h followed by the down projection
    rng = np.random.default_rng(11)
    xr, w13r, w2r = rng.standard_normal((5, 16)), rng.standard_normal((12, 16)), rng.standard_normal((16, 6))
    np.testing.assert_allclose(oracle.swiglu_ffn(xr, w13r, w2r), oracle.swiglu_hidden(xr, w13r) @ w2r.T,
                               rtol=1e-14)


def test_combine_hand_example():
    # 2 tokens, k = 2; expert rows (already permuted): r0=(1,2) r1=(10,20) r2=(100,200) r3=(-1,-1)
    # token 0 -> rows 2, 0 with weights 0.5, 2; token 1 -> rows 3, 1 with weights 1, 0.1
    eo = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0], [-1.0, -1.0]])
    s2r = np.array([2, 0, 3, 1])
    w = np.array([[0.5, 2.0], [1.0, 0.1]])
    sh = np.array([[7.0, 8.0], [0.0, 1.0]])
    y = oracle.combine(eo, s2r, 2, w, sh)
    np.testing.assert_array_equal(y, [[7 + 50 + 2, 8 + 100 + 4], [0 - 1 + 1, 1 - 1 + 2]])
    # weights already in the rows, no shared expert; a dropped slot (-1) adds nothing
    np.testing.assert_array_equal(oracle.combine(eo, np.array([2, 0, -1, 1]), 2),
                                  [[101.0, 202.0], [10.0, 20.0]])


def test_combine_of_permuted_expert_rows_equals_layer_sum():
    """combine over the permutation's rows gives moe_forward's output: the
    per-slot expert outputs laid out in the permuted row order, unpermuted by
    slot_to_row and summed with the routing weights and the shared expert."""
    cfg = tiny_grouped_config()
    inp = make_inputs(cfg)
    x = inp.x.float().numpy()
    w13, w2 = inp.w13.float().numpy(), inp.w2.float().numpy()
    sh = (inp.sw13.float().numpy(), inp.sw2.float().numpy())
    L32 = oracle.gate_logits(x, inp.gate.float().numpy()).astype(np.float32)
    r = oracle.route_from_logits(L32, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                 cfg.norm_topk_prob, cfg.scale, inp.bias.numpy())
    y, _, shared, per_slot = oracle.moe_forward(x, r, lambda e: (w13[e], w2[e]), sh, return_parts=True)
    _, src, s2r = oracle.permute(r.ids, cfg.E)
    rows = per_slot.reshape(cfg.T * cfg.k, -1)[np.argsort(s2r)]       # row p holds slot s with s2r[s] = p
    np.testing.assert_allclose(oracle.combine(rows, s2r, cfg.k, r.weights, shared), y, rtol=1e-12, atol=1e-12)


def _dense_bruteforce(x, route, w13, w2, sw13, sw2, E):
    """Every expert on every token, masked by the routing weights."""
    x = x.astype(np.float64)
    T = x.shape[0]
    I = w13.shape[1] // 2
    gu = np.einsum("th,eih->tei", x, w13.astype(np.float64))
    g, u = gu[..., :I], gu[..., I:]
    h = g / (1 + np.exp(-g)) * u
    out = np.einsum("tei,ehi->teh", h, w2.astype(np.float64))
    W = np.zeros((T, E))
    np.put_along_axis(W, route.ids.astype(np.int64), route.weights, axis=1)
    y = np.einsum("te,teh->th", W, out)
    gu_s = x @ sw13.astype(np.float64).T
    Is = sw13.shape[0] // 2
    hs = gu_s[:, :Is] / (1 + np.exp(-gu_s[:, :Is])) * gu_s[:, Is:]
    return y + hs @ sw2.astype(np.float64).T


@pytest.mark.parametrize("which", ["tiny", "tiny_grouped"])
def test_moe_forward_equals_dense_bruteforce(which):
    cfg = get_config("tiny") if which == "tiny" else tiny_grouped_config()
    inp = make_inputs(cfg)
    x = inp.x.float().numpy()
    G = inp.gate.float().numpy()
    w13 = inp.w13.float().numpy()
    w2 = inp.w2.float().numpy()
    L32 = oracle.gate_logits(x, G).astype(np.float32)
    bias = inp.bias.numpy() if inp.bias is not None else None
    r = oracle.route_from_logits(L32, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                 cfg.norm_topk_prob, cfg.scale, bias)
    y = oracle.moe_forward(x, r, lambda e: (w13[e], w2[e]),
                           (inp.sw13.float().numpy(), inp.sw2.float().numpy()))
    yd = _dense_bruteforce(x, r, w13, w2, inp.sw13.float().numpy(), inp.sw2.float().numpy(), cfg.E)
    np.testing.assert_allclose(y, yd, rtol=1e-10, atol=1e-12)


def test_combine_identical_experts_unit_weights():
    # every expert identical, weights 1 -> y = k * FFN(x) + shared(x)
    rng = np.random.default_rng(4)
    T, H, I, E, k = 10, 16, 8, 6, 3
    x = rng.standard_normal((T, H))
    w13 = rng.standard_normal((2 * I, H)) * 0.3
    w2 = rng.standard_normal((H, I)) * 0.3
    s13 = rng.standard_normal((2 * I, H)) * 0.3
    s2 = rng.standard_normal((H, I)) * 0.3
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    r = O.RouteResult(ids, np.ones((T, k)), None, None, None, None, None)
    y = oracle.moe_forward(x, r, lambda e: (w13, w2), (s13, s2))
    f = oracle.swiglu_ffn(x, w13, w2)
    s = oracle.swiglu_ffn(x, s13, s2)
    np.testing.assert_allclose(y, k * f + s, rtol=1e-12, atol=1e-12)


def _torch_fp8_expert(x, w13, w2):
    """The FP8 expert again, with torch's own E4M3 cast doing the rounding."""
    def q_rows(a):
        a = torch.from_numpy(np.asarray(a, np.float32))
        t = a.reshape(a.shape[0], -1, 128)
        amax = t.abs().amax(dim=2, keepdim=True)
        s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
        return ((t / s).to(torch.float8_e4m3fn).to(torch.float64) * s.double()).reshape(a.shape)

    def q_blocks(w):
        w = torch.from_numpy(np.asarray(w, np.float32))
        N, K = w.shape
        t = w.reshape(N // 128, 128, K // 128, 128)
        amax = t.abs().amax(dim=(1, 3), keepdim=True)
        s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
        return ((t / s).to(torch.float8_e4m3fn).to(torch.float64) * s.double()).reshape(N, K)

    I = w13.shape[0] // 2
    gu = q_rows(x) @ q_blocks(w13).T
    g, u = gu[:, :I], gu[:, I:]
    h = g * torch.sigmoid(g) * u
    return (q_rows(h.float().numpy()) @ q_blocks(w2).T).numpy()


def test_fp8_expert_matches_torch_cast_formulation():
    cfg = tiny_grouped_config()
    inp = make_inputs(cfg)
    x = inp.x.float().numpy()[:40]
    w13 = inp.w13.float().numpy()[3]
    w2 = inp.w2.float().numpy()[3]
    xq, xs = oracle.fp8_quantize_rows(x)
    ours = O._swiglu_fp8(O.fp8_dequant_rows(xq, xs), w13, w2)
    # restricting the output to a few features changes nothing
    feats = [0, 5, 130, 255]
    part = O._swiglu_fp8(O.fp8_dequant_rows(xq, xs), w13, w2, feats)
    np.testing.assert_allclose(part, ours[:, feats], rtol=1e-12, atol=1e-15)
    ref = _torch_fp8_expert(x, w13, w2)
    np.testing.assert_allclose(ours, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    # and quantisation is visible against the unquantised expert
    full = oracle.swiglu_ffn(x, w13, w2)
    rel = np.abs(ours - full).max() / np.abs(full).max()
    assert 1e-4 < rel < 0.15


# ------------------------------------------------------------ bias, load CV
def test_bias_update_literal_and_sign_zero():
    counts = np.array([3, 1, 2, 2])             # T*k = 8, E = 4, mean 2
    b0 = np.array([0.01, -0.02, 0.03, 0.0], np.float32)
    b1 = oracle.bias_update(counts, b0, 0.001, T=2, k=4)
    expect = np.array([0.01 - 0.001, -0.02 + 0.001, 0.03, 0.0], np.float32)
    np.testing.assert_array_equal(b1, np.array([np.float32(0.01) - np.float32(0.001),
                                                np.float32(-0.02) + np.float32(0.001),
                                                np.float32(0.03), np.float32(0.0)], np.float32))
    np.testing.assert_allclose(b1, expect, rtol=1e-6)
    assert b1.dtype == np.float32


def test_bias_update_ten_steps_closed_form():
    rng = np.random.default_rng(9)
    E, T, k, gamma = 256, 1024, 8, 0.001
    counts = rng.integers(0, 70, E)
    counts[0] = T * k // E                      # exactly at the mean: never moves
    b0 = (rng.random(E) * 0.1 - 0.05).astype(np.float32)
    b = b0
    for _ in range(10):
        b = oracle.bias_update(counts, b, gamma, T, k)
    s = np.sign(counts * E - T * k)
    np.testing.assert_allclose(b.astype(np.float64), b0 - 10 * gamma * s, atol=1e-7)
    assert b[0] == b0[0]
    assert np.all(np.abs(b.astype(np.float64) - b0) <= 10 * gamma + 1e-7)


def test_load_cv_literal():
    # counts 1,2,3,4: mean 2.5, sample variance 5/3 -> CV = sqrt(5/3)/2.5
    assert oracle.load_cv(np.array([1, 2, 3, 4])) == pytest.approx(0.5163977794943222, rel=1e-15)
    assert oracle.load_cv(np.full(16, 7)) == 0.0


# ------------------------------------------------- the pages' size accounting
def test_v2lite_parameter_counts():
    # "MoE 混合专家模型推理参数与前向传播详解" §2.2: one expert = 3 x 2048 x 1408 = 8.65M;
    # §2.4: per token 6 routed + 2 shared + router = 69.3M.
    cfg = get_config("v2lite")
    per_expert = 3 * cfg.H * cfg.I
    assert round(per_expert / 1e6, 2) == 8.65
    active = cfg.flops() / cfg.T / 2
    assert round(active / 1e6, 1) == 69.3


# ------------------------------------- sequence-level aux loss (closed forms)
# "MoE 混合专家模型推理参数与前向传播详解" §6.2: aux = E * sum_e load_e * importance_e,
# added to the loss times aux_loss_alpha = 0.001.
def _round_robin_ids(T, k, E):
    return (np.arange(T)[:, None] * k + np.arange(k)[None, :]) % E


@pytest.mark.parametrize("scoring", ["softmax", "sigmoid"])
def test_seq_aux_loss_is_one_when_balanced(scoring):
    T, E, k = 64, 16, 4
    L = np.zeros((T, E), np.float32)                 # every score equal: importance 1/E
    ids = _round_robin_ids(T, k, E)                  # every expert gets T*k/E assignments
    assert oracle.seq_aux_loss(L, ids, E, k, scoring, T, 1.0) == pytest.approx(1.0, rel=1e-14)
    assert oracle.seq_aux_loss(L, ids, E, k, scoring, T, 0.001) == pytest.approx(0.001, rel=1e-14)


def test_seq_aux_loss_collapsed_routing_is_E_over_k():
    T, E, k = 64, 16, 4
    L = np.full((T, E), -1e4, np.float32)
    L[:, :k] = 0.0                                   # softmax mass 1/k on experts 0..k-1, 0 elsewhere
    ids = np.tile(np.arange(k), (T, 1))
    assert oracle.seq_aux_loss(L, ids, E, k, "softmax", T, 1.0) == pytest.approx(E / k, rel=1e-14)
    # the same loads against scores that sit on other experts: no overlap, zero loss
    L2 = np.full((T, E), -1e4, np.float32)
    L2[:, k:2 * k] = 0.0
    assert oracle.seq_aux_loss(L2, ids, E, k, "softmax", T, 1.0) == 0.0


def test_seq_aux_loss_is_per_sequence():
    T, E, k = 64, 16, 4
    L = np.full((T, E), -1e4, np.float32)
    ids = np.zeros((T, k), np.int64)
    L[:32, 0:4] = 0.0
    ids[:32] = np.arange(0, 4)
    L[32:, 4:8] = 0.0
    ids[32:] = np.arange(4, 8)
    # two sequences, each collapsed on its own four experts: E/k each
    assert oracle.seq_aux_loss(L, ids, E, k, "softmax", 32, 1.0) == pytest.approx(4.0, rel=1e-14)
    # one sequence: loads and importances spread over eight experts, 16 * 8 / 64
    assert oracle.seq_aux_loss(L, ids, E, k, "softmax", 64, 1.0) == pytest.approx(2.0, rel=1e-14)


@pytest.mark.parametrize("scoring,row0", [("softmax", [np.log(3.0), 0.0]),
                                          ("sigmoid", [np.log(3.0), -np.log(3.0)])])
def test_seq_aux_loss_two_token_hand_example(scoring, row0):
    # token 0 scores (3/4, 1/4) in both scorings (sigmoid(ln 3) = 3/4 and the two
    # sigmoids sum to 1), token 1 scores (1/2, 1/2): importance (5/8, 3/8)
    L = np.array([row0, [0.0, 0.0]], np.float32)
    both_on_0 = np.array([[0], [0]])
    split = np.array([[0], [1]])
    assert oracle.seq_aux_loss(L, both_on_0, 2, 1, scoring, 2, 1.0) == pytest.approx(1.25, rel=1e-6)
    assert oracle.seq_aux_loss(L, split, 2, 1, scoring, 2, 1.0) == pytest.approx(1.0, rel=1e-6)
    assert oracle.seq_aux_loss(L, np.array([[1], [1]]), 2, 1, scoring, 2, 1.0) == pytest.approx(0.75, rel=1e-6)


def test_moe_forward_thread_pool_map_gives_identical_result():
    """Evaluating the experts side by side changes nothing: their outputs are
    summed in expert order either way."""
    from concurrent.futures import ThreadPoolExecutor
    cfg = tiny_grouped_config()
    inp = make_inputs(cfg)
    x = inp.x.float().numpy()
    w13, w2 = inp.w13.float().numpy(), inp.w2.float().numpy()
    sh = (inp.sw13.float().numpy(), inp.sw2.float().numpy())
    L32 = oracle.gate_logits(x, inp.gate.float().numpy()).astype(np.float32)
    r = oracle.route_from_logits(L32, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                 cfg.norm_topk_prob, cfg.scale, inp.bias.numpy())
    y0 = oracle.moe_forward(x, r, lambda e: (w13[e], w2[e]), sh)
    with ThreadPoolExecutor(4) as ex:
        y1 = oracle.moe_forward(x, r, lambda e: (w13[e], w2[e]), sh, map_fn=ex.map)
    np.testing.assert_array_equal(y0, y1)

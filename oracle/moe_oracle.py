"""CPU oracle: the MoE layer forward written out from the pages, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Pages followed (cited by title and section):
  [V3-teardown]  gsyq.cn "为什么要在本地拆解 DeepSeek-V3 的 MoE 与 MLA",
                 §3 moe_router.json / infer.toml, §4 route() and the load
                 statistic.
  [MoE-walk]     zhiyuanblog.org "MoE 混合专家模型推理参数与前向传播详解",
                 §2.2-2.3 (weights), §3.1-3.4 (routing, permutation, SwiGLU
                 experts, shared experts, combine).
  [V3-digest]    xxqk.cn DeepSeek V3/R1/Janus-Pro digest, §2.2 (aux-loss-free
                 bias and device-limited routing).
  [FP8-infer]    blog.hotdry.top DeepSeek-V3 FP8 inference post, "FP8 混合精度"
                 section (E4M3, 1x128 activation / 128x128 weight tiles).
  [MoE-walk §6.2] the same zhiyuanblog.org page, "辅助损失（训练时）": the
                 sequence-level auxiliary balance loss (seq_aux, alpha 0.001).

Readings taken where the pages are silent or disagree:
  * The selection bias only decides which experts are chosen; the weights
    are the unbiased sigmoid scores.
  * Experts outside the kept groups are excluded (treated as -inf), not set
    to 0.0 as the [V3-teardown] snippet writes.
  * Ties: lower expert index wins, lower group index wins.
  * routed_scaling_factor multiplies the weights whether or not they are
    renormalised.
  * Softmax with a single group and no bias selects on the logits (softmax
    is strictly increasing, so the chosen set is the same and fp32 logits
    carry no rounding of their own).
  * FP8 scale = amax / 448 in fp32 (1.0 when amax = 0); code =
    round-to-nearest-even, saturating, of x / scale computed in fp32.
  * Bias step: b_e <- b_e - gamma * sign(c_e * E - T * k), the sign taken on
    exact integers, the subtraction rounded once in fp32.
  * Sequence-level aux loss: the T tokens form T / seq_len sequences of
    seq_len consecutive tokens. An expert's load is its share of the
    sequence's seq_len * k assignments; its importance is the mean over the
    sequence's tokens of the token's score for it, normalised over all E
    experts (the softmax probability; for sigmoid scoring sigma / sum of
    sigma). Per sequence: E * sum_e load_e * importance_e (1 when both are
    uniform); the value is alpha times the mean over sequences.
"""
from dataclasses import dataclass
from typing import Callable, Optional, Tuple

import numpy as np

E4M3_MAX = 448.0


# --------------------------------------------------------------------------
# FP8 E4M3 ([FP8-infer]; [V3-teardown] §3 infer.toml weight_block_size
# [128, 128], activation_scheme dynamic).
# --------------------------------------------------------------------------
def e4m3_values() -> np.ndarray:
    """Value of each of the 256 E4M3 codes (1 sign, 4 exponent bits with bias
    7, 3 mantissa bits; exponent 0 is subnormal; S.1111.111 is NaN; no inf)."""
    codes = np.arange(256, dtype=np.int64)
    sign = (codes >> 7) & 1
    exp = (codes >> 3) & 0xF
    man = codes & 0x7
    normal = (1.0 + man / 8.0) * np.power(2.0, exp - 7.0)
    subnormal = (man / 8.0) * 2.0 ** -6
    val = np.where(exp == 0, subnormal, normal)
    val = np.where(sign == 1, -val, val)
    val[(exp == 15) & (man == 7)] = np.nan
    return val


_E4M3_POS = e4m3_values()[:127]          # codes 0x00..0x7E, ascending


def quantize_e4m3(y32: np.ndarray) -> np.ndarray:
    """E4M3 code of each float32 value: nearest representable, ties to the
    even code, magnitudes beyond 448 clamped to 448, sign bit kept."""
    y = np.asarray(y32, dtype=np.float32).astype(np.float64)
    a = np.abs(y)
    neg = np.signbit(y)
    hi = np.searchsorted(_E4M3_POS, a, side="left")       # POS[hi-1] < a <= POS[hi]
    hi = np.clip(hi, 1, 126)
    lo = hi - 1
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a >= E4M3_MAX, 126, mag)
    mag = np.where(a == 0.0, 0, mag)
    return (mag | (neg.astype(np.int64) << 7)).astype(np.uint8)


def dequantize_e4m3(codes: np.ndarray) -> np.ndarray:
    return e4m3_values()[np.asarray(codes, dtype=np.int64)]


def round_to_e4m3(y32: np.ndarray) -> np.ndarray:
    """The value `quantize_e4m3` picks, computed arithmetically: keep 3
    mantissa bits (quantum 2^(e-4) for |y| = m * 2^e, m in [0.5, 1), never
    finer than the subnormal step 2^-9), round half to even, clamp to 448."""
    y = np.asarray(y32, dtype=np.float32).astype(np.float64)
    _, e = np.frexp(y)
    quantum = np.ldexp(1.0, np.maximum(e - 4, -9))
    r = np.round(y / quantum) * quantum
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def _scale_of(amax32: np.ndarray) -> np.ndarray:
    amax32 = np.asarray(amax32, dtype=np.float32)
    s = amax32 / np.float32(E4M3_MAX)
    return np.where(amax32 == 0, np.float32(1.0), s).astype(np.float32)


def fp8_quantize_blocks(w: np.ndarray, block: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """Weight quantisation per block x block tile of an [N, K] matrix.
    Returns (codes uint8 [N, K], scales float32 [N/block, K/block])."""
    w32 = np.asarray(w, dtype=np.float32)
    N, K = w32.shape
    assert N % block == 0 and K % block == 0
    tiles = w32.reshape(N // block, block, K // block, block)
    amax = np.abs(tiles).max(axis=(1, 3))
    scale = _scale_of(amax)
    q = quantize_e4m3(tiles / scale[:, None, :, None])
    return q.reshape(N, K), scale


def fp8_quantize_rows(a: np.ndarray, block: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """Activation quantisation per 1 x block tile of an [M, K] matrix.
    Returns (codes uint8 [M, K], scales float32 [M, K/block])."""
    a32 = np.asarray(a, dtype=np.float32)
    M, K = a32.shape
    assert K % block == 0
    tiles = a32.reshape(M, K // block, block)
    amax = np.abs(tiles).max(axis=2)
    scale = _scale_of(amax)
    q = quantize_e4m3(tiles / scale[:, :, None])
    return q.reshape(M, K), scale


def fp8_qdq_blocks(w: np.ndarray, block: int = 128) -> np.ndarray:
    """Dequantised values of `fp8_quantize_blocks(w)` (via `round_to_e4m3`)."""
    w32 = np.asarray(w, dtype=np.float32)
    N, K = w32.shape
    tiles = w32.reshape(N // block, block, K // block, block)
    scale = _scale_of(np.abs(tiles).max(axis=(1, 3)))
    v = round_to_e4m3(tiles / scale[:, None, :, None])
    return (v * scale[:, None, :, None].astype(np.float64)).reshape(N, K)


def fp8_qdq_rows(a: np.ndarray, block: int = 128) -> np.ndarray:
    """Dequantised values of `fp8_quantize_rows(a)` (via `round_to_e4m3`)."""
    a32 = np.asarray(a, dtype=np.float32)
    M, K = a32.shape
    tiles = a32.reshape(M, K // block, block)
    scale = _scale_of(np.abs(tiles).max(axis=2))
    v = round_to_e4m3(tiles / scale[:, :, None])
    return (v * scale[:, :, None].astype(np.float64)).reshape(M, K)


def fp8_dequant_blocks(q: np.ndarray, scale: np.ndarray, block: int = 128) -> np.ndarray:
    v = dequantize_e4m3(q)
    return v * np.repeat(np.repeat(scale.astype(np.float64), block, 0), block, 1)


def fp8_dequant_rows(q: np.ndarray, scale: np.ndarray, block: int = 128) -> np.ndarray:
    v = dequantize_e4m3(q)
    return v * np.repeat(scale.astype(np.float64), block, 1)


# --------------------------------------------------------------------------
# Router ([MoE-walk] §2.1, §3.1; [V3-teardown] §3, §4 route();
# [V3-digest] §2.2).
# --------------------------------------------------------------------------
def gate_logits(x: np.ndarray, gate: np.ndarray) -> np.ndarray:
    """router_logits = hidden_states @ gate.weight^T ([MoE-walk] §2.1)."""
    return np.asarray(x, np.float64) @ np.asarray(gate, np.float64).T


def selection_scores(logits32: np.ndarray, scoring: str, n_group: int,
                     bias32: Optional[np.ndarray] = None):
    """Scores the router selects on, and the unbiased scores the weights use.

    sigmoid: sel = fp32(sigmoid(L)) + b (an fp32 add); weights use sigmoid(L).
    softmax: weights use softmax over all experts; with one group and no
             bias the selection is on the logits themselves, otherwise on
             fp32(softmax) (+ b).
    The sigmoid and softmax are evaluated in float64 and rounded once to
    float32, so the decision does not depend on any one exp implementation.
    """
    L32 = np.asarray(logits32, dtype=np.float32)
    L = L32.astype(np.float64)
    if scoring == "sigmoid":
        sig64 = 1.0 / (1.0 + np.exp(-L))
        sel = sig64.astype(np.float32)
        if bias32 is not None:
            sel = sel + np.asarray(bias32, dtype=np.float32)[None, :]
        return sel.astype(np.float32), sig64
    if scoring == "softmax":
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m)
        p64 = e / e.sum(axis=1, keepdims=True)
        if n_group == 1 and bias32 is None:
            return L32.copy(), p64
        sel = p64.astype(np.float32)
        if bias32 is not None:
            sel = sel + np.asarray(bias32, dtype=np.float32)[None, :]
        return sel.astype(np.float32), p64
    raise ValueError(scoring)


@dataclass
class RouteResult:
    ids: np.ndarray          # [T, k] int32, slot order: score desc, index asc
    weights: np.ndarray      # [T, k] float64
    sel: np.ndarray          # [T, E] float32 selection scores
    kept_groups: np.ndarray  # [T, g] int
    kth_gap: np.ndarray      # [T] gap between k-th and (k+1)-th candidate score
    group_gap: np.ndarray    # [T] gap between g-th and (g+1)-th group score
    counts: np.ndarray       # [E] int64


def route_from_logits(logits32: np.ndarray, k: int, n_group: int, topk_group: int,
                      scoring: str, norm_topk_prob: bool, scale: float,
                      bias32: Optional[np.ndarray] = None) -> RouteResult:
    """Group-limited top-k routing ([V3-teardown] §4 route(); [MoE-walk] §3.1).

    1. selection scores (see `selection_scores`);
    2. if n_group > 1: view the E experts as n_group contiguous groups; a
       group's score is the fp32 sum of its two largest selection scores;
       keep the topk_group best groups;
    3. take the k best selection scores among experts of kept groups;
    4. weights = unbiased scores of those experts; if norm_topk_prob divide by
       their sum; multiply by routed_scaling_factor.
    """
    sel, unbiased = selection_scores(logits32, scoring, n_group, bias32)
    T, E = sel.shape
    gsz = E // n_group
    if n_group > 1:
        grouped = sel.reshape(T, n_group, gsz)
        top = -np.sort(-grouped, axis=2)                     # descending
        if gsz >= 2:
            gscore = (top[:, :, 0] + top[:, :, 1]).astype(np.float32)
        else:
            gscore = top[:, :, 0].astype(np.float32)
        gorder = np.argsort(-gscore, axis=1, kind="stable")
        kept = gorder[:, :topk_group]
        gs_sorted = np.take_along_axis(gscore, gorder, axis=1).astype(np.float64)
        if topk_group < n_group:
            group_gap = gs_sorted[:, topk_group - 1] - gs_sorted[:, topk_group]
        else:
            group_gap = np.full(T, np.inf)
        cand = np.zeros((T, n_group), dtype=bool)
        np.put_along_axis(cand, kept, True, axis=1)
        cand = np.repeat(cand, gsz, axis=1)
    else:
        kept = np.zeros((T, 1), dtype=np.int64)
        group_gap = np.full(T, np.inf)
        cand = np.ones((T, E), dtype=bool)

    masked = np.where(cand, sel.astype(np.float64), -np.inf)
    order = np.argsort(-masked, axis=1, kind="stable")
    ids = order[:, :k]
    # near-tie statistic in the score space the pages select on
    if scoring == "softmax" and bias32 is None:
        gap_space = np.where(cand, unbiased, -np.inf)
    else:
        gap_space = masked
    srt = np.take_along_axis(gap_space, order, axis=1)
    ncand = cand.sum(axis=1)
    kth_gap = np.full(T, np.inf)
    more = ncand > k
    if k < E and more.any():
        kth_gap[more] = srt[more, k - 1] - srt[more, k]

    w = np.take_along_axis(unbiased, ids, axis=1)
    if norm_topk_prob:
        w = w / w.sum(axis=1, keepdims=True)
    w = w * float(scale)
    counts = np.bincount(ids.reshape(-1), minlength=E).astype(np.int64)
    return RouteResult(ids.astype(np.int32), w, sel, kept, kth_gap, group_gap, counts)


# --------------------------------------------------------------------------
# Permutation ([MoE-walk] §3.2 and its worked example).
# --------------------------------------------------------------------------
def permute(ids: np.ndarray, E: int):
    """Expand each token k times and order the copies by expert.

    Segment e holds the tokens routed to expert e in ascending token order
    (the worked example of [MoE-walk] §3.2). Returns
      offsets     [E+1]  expert_first_token_offset (empty experts repeat)
      src_token   [T*k]  row -> token
      slot_to_row [T*k]  t*k + j -> row (inv_permuted_idx)
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")           # expert-major, then t*k+j
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    src_token = order // k
    slot_to_row = np.empty(T * k, dtype=np.int64)
    slot_to_row[order] = np.arange(T * k)
    return offsets, src_token, slot_to_row


# --------------------------------------------------------------------------
# Experts ([MoE-walk] §3.3.1 SwiGLU, §3.3.2 shared experts).
# --------------------------------------------------------------------------
def swiglu_hidden(x: np.ndarray, w13: np.ndarray) -> np.ndarray:
    """The expert's intermediate activation: gate_up = x @ w13^T; gate, up =
    its first / last I columns (w13 stacks w1 over w3); h = SiLU(gate) * up
    with SiLU(v) = v * sigmoid(v)."""
    x = np.asarray(x, np.float64)
    w13 = np.asarray(w13, np.float64)
    I = w13.shape[0] // 2
    gu = x @ w13.T
    g, u = gu[:, :I], gu[:, I:]
    return g * (1.0 / (1.0 + np.exp(-g))) * u


def swiglu_ffn(x: np.ndarray, w13: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """One SwiGLU expert: out = h @ w2^T with h = swiglu_hidden(x, w13)."""
    return swiglu_hidden(x, w13) @ np.asarray(w2, np.float64).T


def _swiglu_fp8(xd, w13, w2, w2_rows=None):
    """The same expert in E4M3: weights per 128x128 block, activations per
    1x128 tile (xd = the dequantised activations), h re-quantised per 1x128.
    `w2_rows` optionally restricts the output to those features (the blocks
    holding them are quantised exactly as in the whole matrix)."""
    h = swiglu_hidden(xd, fp8_qdq_blocks(w13))
    hd = fp8_qdq_rows(h.astype(np.float32))
    if w2_rows is None:
        return hd @ fp8_qdq_blocks(w2).T
    blocks = np.unique(np.asarray(w2_rows) // 128)
    sub = np.concatenate([np.asarray(w2[b * 128:(b + 1) * 128]) for b in blocks])
    dq = fp8_qdq_blocks(sub)
    pos = {b: i for i, b in enumerate(blocks)}
    idx = [pos[r // 128] * 128 + r % 128 for r in w2_rows]
    return hd @ dq[idx].T


def moe_forward(x: np.ndarray, route: RouteResult,
                expert_weights: Callable[[int], Tuple[np.ndarray, np.ndarray]],
                shared: Optional[Tuple[np.ndarray, np.ndarray]], fp8: bool = False,
                return_parts: bool = False, out_features=None, map_fn=map):
    """y_t = shared(x_t) + sum_j w_tj * E_{id_tj}(x_t)  ([MoE-walk] §3.4).

    `x` holds the tokens to evaluate (any subset; the layer is per token), and
    `route` their routing. `expert_weights(e)` returns (w13_e, w2_e) for one
    expert, so the caller can widen one expert at a time. `out_features`
    (optional) limits the output to those hidden features. `map_fn` evaluates
    the experts (default: one after another; a thread pool's map runs them
    side by side); their outputs are summed in expert order either way.
    """
    x = np.asarray(x, np.float64)
    T, H = x.shape
    ids = route.ids
    k = ids.shape[1]
    xd = fp8_qdq_rows(x.astype(np.float32)) if fp8 else None
    Hout = H if out_features is None else len(out_features)
    routed = np.zeros((T, Hout), dtype=np.float64)
    per_slot = np.zeros((T, k, Hout), dtype=np.float64) if return_parts else None

    def expert_rows(e):
        tt, jj = np.nonzero(ids == e)
        w13, w2 = expert_weights(int(e))
        if fp8:
            out = _swiglu_fp8(xd[tt], np.asarray(w13, np.float32), np.asarray(w2, np.float32),
                              out_features)
        else:
            w2s = w2 if out_features is None else np.asarray(w2)[out_features]
            out = swiglu_ffn(x[tt], w13, w2s)
        return tt, jj, out

    for tt, jj, out in map_fn(expert_rows, np.unique(ids)):
        contrib = route.weights[tt, jj][:, None] * out
        np.add.at(routed, tt, contrib)
        if return_parts:
            per_slot[tt, jj] = out
    sh = np.zeros((T, Hout), dtype=np.float64)
    if shared is not None:
        if fp8:
            sh = _swiglu_fp8(xd, np.asarray(shared[0], np.float32),
                             np.asarray(shared[1], np.float32), out_features)
        else:
            s2 = shared[1] if out_features is None else np.asarray(shared[1])[out_features]
            sh = swiglu_ffn(x, shared[0], s2)
    y = routed + sh
    if return_parts:
        return y, routed, sh, per_slot
    return y


def combine(expert_out: np.ndarray, slot_to_row: np.ndarray, k: int,
            weights: Optional[np.ndarray] = None, shared: Optional[np.ndarray] = None) -> np.ndarray:
    """Unpermute and combine ([MoE-walk] §3.4): token t's output is its shared
    expert row plus the sum over its k slots j of w_tj times the expert output
    row that slot's copy was computed in, row slot_to_row[t*k + j] of
    expert_out. weights = None: the rows already carry their routing weight
    (w = 1). Slots whose row is negative (dropped) contribute nothing."""
    eo = np.asarray(expert_out, np.float64)
    s2r = np.asarray(slot_to_row).reshape(-1, k)
    T = s2r.shape[0]
    w = np.ones((T, k)) if weights is None else np.asarray(weights, np.float64).reshape(T, k)
    y = np.zeros((T, eo.shape[1])) if shared is None else np.array(shared, np.float64)
    for t in range(T):
        for j in range(k):
            if s2r[t, j] >= 0:
                y[t] += w[t, j] * eo[s2r[t, j]]
    return y


# --------------------------------------------------------------------------
# Aux-loss-free balancing ([V3-digest] §2.2; load statistic [V3-teardown] §4).
# --------------------------------------------------------------------------
def bias_update(counts: np.ndarray, bias32: np.ndarray, gamma: float,
                T: int, k: int) -> np.ndarray:
    """Overloaded experts' bias goes down, underloaded up, by gamma.
    Load is compared with the mean T*k/E exactly, as c_e*E vs T*k."""
    c = np.asarray(counts, dtype=np.int64)
    E = c.shape[0]
    s = np.sign(c * E - int(T) * int(k)).astype(np.float32)
    b = np.asarray(bias32, dtype=np.float32)
    return (b - np.float32(gamma) * s).astype(np.float32)


def load_cv(counts: np.ndarray) -> float:
    """Coefficient of variation of expert loads: sample standard deviation
    (divisor E-1) over the mean."""
    c = np.asarray(counts, dtype=np.float64)
    E = c.shape[0]
    mean = c.sum() / E
    var = ((c - mean) ** 2).sum() / (E - 1)
    return float(np.sqrt(var) / mean)


# --------------------------------------------------------------------------
# Sequence-level auxiliary balance loss ([MoE-walk §6.2]; seq_aux and
# aux_loss_alpha also appear in [V3-teardown] §3 moe_router.json).
# --------------------------------------------------------------------------
def seq_aux_loss(logits32: np.ndarray, ids: np.ndarray, E: int, k: int, scoring: str,
                 seq_len: int, alpha: float) -> float:
    """alpha * mean over sequences of E * sum_e f_e * P_e, where f_e is the
    fraction of the sequence's seq_len * k assignments that go to expert e
    and P_e the mean of the tokens' normalised scores for e. Forward value
    only; fp64 throughout."""
    L = np.asarray(logits32, dtype=np.float32).astype(np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    T = L.shape[0]
    if seq_len <= 0 or T % seq_len:
        raise ValueError("seq_len must divide T")
    if scoring == "softmax":
        z = np.exp(L - L.max(axis=1, keepdims=True))
    elif scoring == "sigmoid":
        z = 1.0 / (1.0 + np.exp(-L))
    else:
        raise ValueError(scoring)
    p = z / z.sum(axis=1, keepdims=True)          # per-token scores summing to 1
    total = 0.0
    n_seq = T // seq_len
    for b in range(n_seq):
        rows = slice(b * seq_len, (b + 1) * seq_len)
        f = np.bincount(ids[rows].ravel(), minlength=E).astype(np.float64) / (seq_len * k)
        P = p[rows].mean(axis=0)
        total += E * float(np.dot(f, P))
    return alpha * total / n_seq

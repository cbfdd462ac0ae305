"""CPU oracle for the single-GPU Mixture-of-Experts layer forward.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
calls it and it never calls the CUDA library; the two share no code.

It is a plain, slow, obviously-correct restatement of what the layer computes,
in float64 numpy (a library matmul is the only borrowed step).  Sources, all
extracted web pages about MoE inference:

* jsqmd.com, "第11章 MoE模型推理" (chapter 11, MoE model inference):
  - 11.1.1 "稀疏激活原理": the layer y = sum_i R(x)_i * E_i(x), the router
    R(x) = Softmax(W_r x) and the TopK(s, K) sparsifier that sets every
    non-selected score to -inf before the softmax;
  - 11.1.2 "专家网络与门控机制": the expert E_i(x) = GeLU(x W1 + b1) W2 + b2
    and the statement that the B*L*K expert forwards are grouped by expert;
  - 11.2.1: gather into per-expert sub-sequences, then restore token order;
  - 11.2.3: the max/mean expert-load ratio (ideal 1, 3-5 in practice);
  - 11.3.1, step 6 of the expert-parallel layer: weighted sum of the K
    expert outputs by their top-k probabilities.
* ybb.press, "MoE 推理工程深层实战":
  - 2.2 (expert-parallel dispatch, capacity paragraph): tokens above a
    capacity go to an overflow buffer and are processed later, none dropped;
  - 2.3 "DeepSeek-V3 的 256 专家路由机制": aux-loss-free bias that steers
    selection only, node(group)-limited routing: sum of biased scores per
    group, top-2 groups, top-8 experts inside them.
* plumephp.com, "MoE 混合专家推理", routing worked example ("路由打分示意"):
  scores e0 .55, e3 .30, e5 .08, e7 .03 -> top-2 = {e0, e3}, output
  .55*e0(x) + .30*e3(x), marked as a normalised weighting.

Readings taken where the pages are silent or disagree (each is listed, with
its reason, in the design notes):

* gates are renormalised over the K selected experts when ``renormalize`` is
  set (the -inf TopK form of 11.1.1 gives exactly that); with it unset they
  are the full softmax probabilities (the 11.3.1 code);
* ties go to the lower expert (and lower group) index; output slots are in
  descending key order; NaN keys rank below every number;
* in the sigmoid/grouped variant the selection bias is added to sigmoid
  scores, gates use the unbiased scores, and a group's score is the sum of all
  its biased scores;
* GeLU is the exact erf form; SwiGLU is silu(x Wg) * (x Wu) followed by Wd;
* weights are stored "out x in" (K-major): w1/w_gate/w_up [E][h][d],
  w2/w_down [E][d][h], w_router [E][d];
* capacity: the first C rows of an expert in (token, k) order are primary,
  the rest overflow; the layer result does not depend on the split.

Routing decisions are integer results decided by floating point, so they are
taken in the precision the method works in (float32 keys).  The sigmoid used
for selection is defined operationally (``sigmoid_f32``) so that any
implementation following the same sequence of float32 operations reaches the
same bits.
"""

from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64.

    bfloat16 is the upper half of an IEEE binary32, so the value is the
    float32 whose bits are ``bits << 16``.
    """
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns, round to nearest, ties to even.

    Rounds in two steps through float32 only when that is exact; to avoid
    double rounding it works on the float64 value directly: the bf16 grid
    near |x| has spacing 2**(e-7) for x in [2**e, 2**(e+1)).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat = x.reshape(-1)
    o = out.reshape(-1)
    for i, v in enumerate(flat):
        o[i] = _round_to_bf16_scalar(float(v))
    return out


def _round_to_bf16_scalar(v: float) -> int:
    if math.isnan(v):
        return 0x7FC0
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    a = abs(v)
    if a == 0.0:
        return sign
    if math.isinf(a):
        return sign | 0x7F80
    m, e = math.frexp(a)  # a = m * 2**e, m in [0.5, 1)
    ebits = e - 1 + 127  # biased exponent of a in binary32 terms
    if ebits >= 1:
        # normal: 8 significant bits -> quantum 2**(e-1-7)
        q = math.ldexp(1.0, e - 1 - 7)
    else:
        # subnormal bf16: quantum is 2**(-126-7)
        q = math.ldexp(1.0, -133)
    n = a / q  # exact (power-of-two scaling)
    r = math.floor(n)
    frac = n - r
    if frac > 0.5 or (frac == 0.5 and (r % 2 == 1)):
        r += 1
    val = r * q
    if val >= math.ldexp(1.0, 128):
        return sign | 0x7F80
    f32 = np.float32(val)  # exact: val is on the bf16 grid
    bits = int(np.array([f32], dtype=np.float32).view(np.uint32)[0])
    return sign | (bits >> 16)


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """FP8 E4M3 ("fn" variant: no infinities) bit patterns -> float64.

    Layout: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
    Exponent field 0 encodes subnormals m/8 * 2**-6; the pattern with every
    exponent and mantissa bit set is NaN; the largest finite value is 448.
    """
    b = np.asarray(bits).astype(np.int64)
    s = np.where((b >> 7) & 1, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int32))
    sub = (m / 8.0) * math.ldexp(1.0, -6)
    v = np.where(e == 0, sub, normal) * s
    v = np.where((e == 0xF) & ((b & 0x7) == 0x7), np.nan, v)
    return v


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------


def router_logits(x: np.ndarray, w_router: np.ndarray, router_bias=None) -> np.ndarray:
    """l[t, e] = sum_k x[t, k] * W_r[e, k] (+ router_bias[e]), float64 sum,
    rounded once to float32.

    Chapter 11 (jsqmd.com), 11.1.1 and 11.1.2: R(x) = Softmax(W_r x), row
    form s = Softmax(x W_r).  ``w_router`` is stored [E][d].
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    logits = x @ w.T
    if router_bias is not None:
        logits = logits + np.asarray(router_bias, dtype=np.float64)[None, :]
    return logits.astype(np.float32)


# float32 constants of the exponential below, derived here from ln 2
_LN2 = math.log(2.0)
_LOG2E_F32 = np.float32(1.0 / _LN2)
# ln 2 cut to its leading 16 significant bits, so that n * _LN2_HI is exact
# in float32 for |n| < 256; the remainder carries the rest.
_LN2_HI_F32 = np.float32(math.ldexp(math.floor(math.ldexp(_LN2, 16)), -16))
_LN2_LO_F32 = np.float32(_LN2 - float(_LN2_HI_F32))
# Taylor coefficients 1/j!, j = 7 .. 1, rounded to float32
_INV_FACT_F32 = [np.float32(1.0 / math.factorial(j)) for j in range(7, 0, -1)]


def exp_f32(z: np.ndarray) -> np.ndarray:
    """exp(z) in float32 by Cody-Waite range reduction and a Taylor polynomial.

    n = rint(z * log2(e)); r = (z - n*ln2_hi) - n*ln2_lo; exp(r) by the
    degree-7 Taylor polynomial in Horner form; result = ldexp(p, n).  Every
    step is one float32 IEEE operation (round to nearest even).  z > 88
    returns +inf and z < -30 returns 0 (there 1 + exp(z) == 1 in float32, so
    the sigmoid below is unaffected).  This is the selection-time exponential
    of the sigmoid router; its accuracy (<= 2 ulp) is pinned against math.exp.
    """
    z = np.asarray(z, dtype=np.float32)
    f = np.float32
    big = z > f(88.0)
    tiny = z < f(-30.0)
    zc = np.where(big | tiny, f(0.0), z).astype(np.float32)
    n = np.rint(np.multiply(zc, _LOG2E_F32, dtype=np.float32)).astype(np.float32)
    r = np.subtract(zc, np.multiply(n, _LN2_HI_F32, dtype=np.float32), dtype=np.float32)
    r = np.subtract(r, np.multiply(n, _LN2_LO_F32, dtype=np.float32), dtype=np.float32)
    p = np.full(r.shape, _INV_FACT_F32[0], dtype=np.float32)
    for c in _INV_FACT_F32[1:]:
        p = np.add(np.multiply(p, r, dtype=np.float32), c, dtype=np.float32)
    p = np.add(np.multiply(p, r, dtype=np.float32), f(1.0), dtype=np.float32)
    out = np.ldexp(p, n.astype(np.int32)).astype(np.float32)
    out = np.where(big, f(np.inf), out)
    out = np.where(tiny, f(0.0), out)
    return out.astype(np.float32)


def sigmoid_f32(l: np.ndarray) -> np.ndarray:
    """sigma(l) = 1 / (1 + exp(-l)), every step a float32 IEEE operation,
    with exp from ``exp_f32``."""
    l = np.asarray(l, dtype=np.float32)
    e = exp_f32(np.negative(l))
    d = np.add(np.float32(1.0), e, dtype=np.float32)
    return np.divide(np.float32(1.0), d, dtype=np.float32)


def _nan_to_neginf(keys: np.ndarray) -> np.ndarray:
    k = np.asarray(keys, dtype=np.float32)
    return np.where(np.isnan(k), np.float32(-np.inf), k).astype(np.float32)


def _order_desc(keys: np.ndarray) -> np.ndarray:
    """Row-wise order of float32 keys: descending, ties to the lower index;
    a NaN key counts as -inf.  A stable sort of the negated keys gives
    exactly this order (the sort is the library step)."""
    neg = -_nan_to_neginf(keys).astype(np.float64)
    return np.argsort(neg, axis=-1, kind="stable")


def group_sums_f32(v: np.ndarray) -> np.ndarray:
    """Group scores (ybb.press 2.3: a group's score is the sum of its
    members' biased scores) as float32 sums along the last axis, vectorised
    over the leading axes.  The order of the float32 additions is fixed: a
    power-of-two number n of members is halved repeatedly, member j adding
    member j + n/2 (for 32 members: strides 16, 8, 4, 2, 1), until one value
    is left."""
    v = np.asarray(v, dtype=np.float32)
    n = v.shape[-1]
    assert n & (n - 1) == 0, "group size must be a power of two"
    while n > 1:
        h = n // 2
        v = np.add(v[..., :h], v[..., h:], dtype=np.float32)
        n = h
    return v[..., 0]


def select_experts(
    logits: np.ndarray,
    top_k: int,
    score_fn: str = "softmax",
    renormalize: bool = True,
    sel_bias=None,
    num_groups: int = 1,
    topk_groups: int = 1,
    temperature: float = 1.0,
):
    """Top-K expert selection and gate weights for every token.

    logits: float32 [S, E] (router output, router bias already added).
    score_fn 'softmax' (chapter 11, 11.1.1): the score is the tempered logit
        z = l / temperature (chapter 11, 11.3.3, soft routing with
        softmax(s / tau); one float32 division, z = l for temperature 1);
        key = z (+ sel_bias); the gate is exp(z_k - m) / sum_{j in TopK}
        exp(z_j - m) when renormalised -- the softmax of the TopK(-inf)
        sparsified scores -- else the full softmax probability of expert k.
    score_fn 'sigmoid' (ybb.press 2.3, bias moved onto the sigmoid scores):
        s = sigmoid_f32(l), key = s + sel_bias in float32; the gate is
        s_k / sum_j s_j (renormalised) or s_k.
    Groups (ybb.press 2.3): E experts in ``num_groups`` consecutive groups;
        group score = float32 halving-tree sum of its keys; the
        ``topk_groups`` best groups (ties to the lower group) hold the
        candidates, the others are excluded.
    A NaN key or group score counts as -inf.
    Returns topk_idx int32 [S, K] (descending key), topk_w float64 [S, K].
    """
    logits = np.asarray(logits, dtype=np.float32)
    S, E = logits.shape
    scores, keys, cand = selection_keys(logits, score_fn, sel_bias, num_groups, topk_groups, temperature)
    # candidates first, each part in descending key order, ties to lower index
    neg = -keys.astype(np.float64)
    order = np.lexsort((np.broadcast_to(np.arange(E), (S, E)), neg, ~cand), axis=-1)
    idx = order[:, :top_k].astype(np.int32)
    return idx, gate_weights(scores, idx, score_fn, renormalize)


def selection_keys(logits, score_fn="softmax", sel_bias=None, num_groups=1, topk_groups=1, temperature=1.0):
    """The quantities selection works on (see ``select_experts``): scores
    (float32 logits divided by the temperature, or their sigmoid), keys
    (scores + sel_bias in float32, NaN -> -inf) and the candidate mask
    (experts of the token's kept groups; all experts without groups)."""
    logits = np.asarray(logits, dtype=np.float32)
    S, E = logits.shape
    if score_fn == "softmax":
        scores = np.divide(logits, np.float32(temperature), dtype=np.float32)
    elif score_fn == "sigmoid":
        assert temperature == 1.0, "the temperature applies to the softmax router"
        scores = sigmoid_f32(logits)
    else:
        raise ValueError(score_fn)
    keys = scores
    if sel_bias is not None:
        keys = np.add(scores, np.asarray(sel_bias, dtype=np.float32)[None, :], dtype=np.float32)
    keys = _nan_to_neginf(keys)
    gs = E // num_groups
    assert gs * num_groups == E
    if num_groups > 1:
        gscore = group_sums_f32(keys.reshape(S, num_groups, gs))
        gorder = _order_desc(gscore)[:, :topk_groups]
        keep = np.zeros((S, num_groups), dtype=bool)
        np.put_along_axis(keep, gorder, True, axis=1)
        cand = np.repeat(keep, gs, axis=1)
    else:
        cand = np.ones((S, E), dtype=bool)
    return scores, keys, cand


def gate_weights(scores, idx, score_fn="softmax", renormalize=True):
    """Gates of the experts idx [S, K] from the float32 scores [S, E]
    (``select_experts``): softmax over the K selected logits, or the full
    softmax probability; sigmoid scores normalised over the K, or as they are.
    float64."""
    idx = np.asarray(idx)
    if score_fn == "softmax":
        l = np.asarray(scores, np.float32).astype(np.float64)
        sel = np.take_along_axis(l, idx, axis=1)
        if renormalize:
            m = sel.max(axis=1, keepdims=True)
            ex = np.exp(sel - m)
            return ex / ex.sum(axis=1, keepdims=True)
        m = l.max(axis=1, keepdims=True)
        ex = np.exp(l - m)
        return np.take_along_axis(ex, idx, axis=1) / ex.sum(axis=1, keepdims=True)
    s = np.take_along_axis(np.asarray(scores, np.float32).astype(np.float64), idx, axis=1)
    return s / s.sum(axis=1, keepdims=True) if renormalize else s


def selection_margin(logits, top_k, score_fn="softmax", sel_bias=None, num_groups=1, topk_groups=1,
                     temperature=1.0):
    """Per token, the smaller of (a) the gap between the K-th and (K+1)-th
    candidate key and (b) the gap between the last kept and the first dropped
    group score.  A path that computes its own logits in another summation
    order may legitimately route a token with a tiny margin differently."""
    logits = np.asarray(logits, dtype=np.float32)
    S, E = logits.shape
    if score_fn == "softmax":
        scores = np.divide(logits, np.float32(temperature), dtype=np.float32)
    else:
        scores = sigmoid_f32(logits)
    keys = scores if sel_bias is None else np.add(scores, np.asarray(sel_bias, np.float32)[None, :],
                                                  dtype=np.float32)
    keys = _nan_to_neginf(keys).astype(np.float64)
    gs = E // num_groups
    margin = np.full(S, np.inf)
    cand = np.ones((S, E), dtype=bool)
    if num_groups > 1:
        g = group_sums_f32(keys.astype(np.float32).reshape(S, num_groups, gs)).astype(np.float64)
        gsorted = -np.sort(-g, axis=1)
        if topk_groups < num_groups:
            margin = np.minimum(margin, gsorted[:, topk_groups - 1] - gsorted[:, topk_groups])
        keep = np.zeros((S, num_groups), dtype=bool)
        np.put_along_axis(keep, _order_desc(g)[:, :topk_groups], True, axis=1)
        cand = np.repeat(keep, gs, axis=1)
    ks = -np.sort(-np.where(cand, keys, -np.inf), axis=1)
    n_cand = cand.sum(axis=1)
    has_next = n_cand > top_k
    gap = ks[:, top_k - 1] - ks[:, min(top_k, E - 1)]
    margin = np.where(has_next, np.minimum(margin, gap), margin)
    return margin


# ----------------------------------------------------------------------------
# grouping by expert
# ----------------------------------------------------------------------------


def expert_counts(topk_idx: np.ndarray, num_experts: int) -> np.ndarray:
    """counts[e] = number of (token, k) slots routed to expert e."""
    return np.bincount(np.asarray(topk_idx).reshape(-1), minlength=num_experts).astype(np.int32)


def exclusive_prefix(counts: np.ndarray) -> np.ndarray:
    """offsets[e] = sum_{j<e} counts[j]; offsets[E] = total."""
    c = np.asarray(counts, dtype=np.int64)
    out = np.zeros(len(c) + 1, dtype=np.int64)
    out[1:] = np.cumsum(c)
    return out.astype(np.int32)


def expert_permutation(topk_idx: np.ndarray, num_experts: int, capacity: int = 0):
    """Stable grouping of the S*K slots by expert (chapter 11, 11.2.1: regroup
    the sequence into per-expert sub-sequences, restore order afterwards).

    Slots are taken in flattened order t*K + k.  A stable sort of the slots by
    expert id gives every slot its rank r inside its expert.  Without
    capacity its row is offsets[e] + r.  With capacity C (ybb.press 2.2,
    overflow buffering) the first C slots of expert e land in the primary
    block at row e*C + r; the others go to the overflow region that starts at
    row E*C, expert after expert (exclusive prefix of the overflow counts), at
    E*C + ovf_offsets[e] + (r - C).  Nothing is dropped.

    Returns a dict: counts, offsets, row_of_slot [S*K], token_of_row [R] (-1
    for unused primary rows), num_rows R; with capacity also prim_counts,
    ovf_counts, ovf_offsets.
    """
    idx = np.asarray(topk_idx)
    S, K = idx.shape
    E = num_experts
    flat = idx.reshape(-1).astype(np.int64)
    counts = expert_counts(idx, E)
    offsets = exclusive_prefix(counts)
    order = np.argsort(flat, kind="stable")  # slots grouped by expert, slot order kept
    rank = np.empty(S * K, dtype=np.int64)
    rank[order] = np.arange(S * K) - offsets[flat[order]]
    out = {"counts": counts, "offsets": offsets}
    if capacity <= 0:
        R = S * K
        row_of_slot = offsets[flat] + rank
    else:
        C = capacity
        prim = np.minimum(counts, C).astype(np.int32)
        ovf = (counts - prim).astype(np.int32)
        ovf_off = exclusive_prefix(ovf)
        R = E * C + S * K
        row_of_slot = np.where(rank < C, flat * C + rank, E * C + ovf_off[flat] + (rank - C))
        out.update(prim_counts=prim, ovf_counts=ovf, ovf_offsets=ovf_off)
    token_of_row = np.full(R, -1, dtype=np.int64)
    token_of_row[row_of_slot] = np.arange(S * K) // K
    out.update(row_of_slot=row_of_slot.astype(np.int32), token_of_row=token_of_row.astype(np.int32), num_rows=R)
    return out


def reroute_over_capacity(topk_idx, keys, cand, capacity: int):
    """Over-capacity re-routing (jsqmd.com chapter 11, 11.3.3, expert-dropping paragraph:
    when an expert is overloaded, its excess tokens go to their next-best
    expert).  The page gives the rule in one sentence; the reading taken:

    1. every expert keeps the first ``capacity`` slots routed to it, slots in
       (token, k) order;
    2. the remaining (excess) slots are visited in (token, k) order; each
       moves to the best expert by the token's selection key among the
       token's candidates (its kept groups) that still has room and that the
       token does not hold already (ties to the lower index), taking one unit
       of that expert's room;
    3. an excess slot with no such expert keeps its expert (it then goes to
       the overflow region, as without re-routing).

    Returns (new topk_idx int32 [S, K], moved bool [S, K]).  Gates are then
    recomputed over the final experts (``gate_weights``)."""
    idx = np.array(topk_idx, dtype=np.int32, copy=True)
    S, K = idx.shape
    E = keys.shape[1]
    kept = np.zeros(E, dtype=np.int64)
    excess = []
    for t in range(S):
        for k in range(K):
            e = idx[t, k]
            if kept[e] < capacity:
                kept[e] += 1
            else:
                excess.append((t, k))
    room = capacity - kept
    moved = np.zeros((S, K), dtype=bool)
    for t, k in excess:
        best, best_key = -1, -np.inf
        held = set(idx[t].tolist())
        for e in range(E):
            if room[e] <= 0 or e in held or not cand[t, e] or keys[t, e] == -np.inf:
                continue
            if best < 0 or keys[t, e] > best_key:
                best, best_key = e, keys[t, e]
        if best >= 0:
            idx[t, k] = best
            room[best] -= 1
            moved[t, k] = True
    return idx, moved


def load_stats(counts: np.ndarray, top_k: int, num_tokens: int, capacity: int = 0) -> dict:
    """Load report of one routing, from the per-expert counts (plumephp.com
    verification block: the routing histogram is the first thing to check):

    * max_over_mean: max_e count_e / (S*K/E), the max/mean expert load of
      chapter 11, 11.2.3 (1 when balanced, 3-5 in practice);
    * std: population standard deviation of the counts (ybb.press 1.2,
      expert load balance row of the table);
    * overflow_rows: rows above the capacity, sum_e max(count_e - C, 0)
      (ybb.press 2.2 overflow buffering; 0 without a capacity);
    * dropped: (token, k) slots without an expert row, S*K - sum_e count_e
      (ybb.press 1.2, token drop rate; the layer drops nothing, so 0 unless
      an expert id was out of range);
    * mean = S*K/E and max = max_e count_e."""
    c = np.asarray(counts, dtype=np.float64)
    mean = num_tokens * top_k / len(c)
    over = float(np.maximum(c - capacity, 0).sum()) if capacity > 0 else 0.0
    return {"max_over_mean": float(c.max() / mean) if mean > 0 else 0.0,
            "std": float(c.std()), "mean": mean, "max": float(c.max()), "overflow_rows": over,
            "dropped": float(num_tokens * top_k - c.sum())}


# ----------------------------------------------------------------------------
# experts
# ----------------------------------------------------------------------------


def gelu_erf(z: np.ndarray) -> np.ndarray:
    """GeLU(z) = 0.5 z (1 + erf(z / sqrt 2)), the exact form."""
    z = np.asarray(z, dtype=np.float64)
    erf = np.vectorize(math.erf)
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)), float64."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def expert_gelu(x, w1, b1, w2, b2):
    """E(x) = GeLU(x W1 + b1) W2 + b2 (chapter 11, 11.1.2) for rows x [n, d];
    w1 [h, d], b1 [h], w2 [d, h], b2 [d] (stored out x in)."""
    x = np.asarray(x, dtype=np.float64)
    hid = gelu_erf(x @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64)[None, :])
    return hid @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)[None, :]


def expert_swiglu(x, w_gate, w_up, w_down, round_hidden_bf16: bool = False,
                  s_gate=None, s_up=None, s_down=None):
    """E(x) = (SiLU(x Wg) * (x Wu)) Wd for rows x [n, d]; w_gate/w_up [h, d],
    w_down [d, h].  Optional per-output-channel scales multiply the weight rows
    (FP8 weights: w = s_n * decode(q_n)).  ``round_hidden_bf16`` rounds the
    hidden activation to bfloat16 before the down projection, as a stored
    bf16 intermediate would."""
    x = np.asarray(x, dtype=np.float64)
    wg = np.asarray(w_gate, np.float64)
    wu = np.asarray(w_up, np.float64)
    wd = np.asarray(w_down, np.float64)
    if s_gate is not None:
        wg = wg * np.asarray(s_gate, np.float64)[:, None]
        wu = wu * np.asarray(s_up, np.float64)[:, None]
        wd = wd * np.asarray(s_down, np.float64)[:, None]
    hid = silu(x @ wg.T) * (x @ wu.T)
    if round_hidden_bf16:
        hid = bf16_bits_to_f64(f64_to_bf16_bits_fast(hid))
    return hid @ wd.T


def f64_to_bf16_bits_fast(x: np.ndarray) -> np.ndarray:
    """Vectorised round-to-nearest-even float64 -> bfloat16 for finite values
    inside the float32 normal range; falls back to the scalar routine for
    anything else.  Rounding is done on the float64 value (no double
    rounding): the bf16 quantum of |x| in [2**e, 2**(e+1)) is 2**(e-7)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    ok = np.isfinite(x) & ((a == 0) | ((a >= 2.0 ** -126) & (a < 2.0 ** 127)))
    if not np.all(ok):
        return f64_to_bf16_bits(x)
    m, e = np.frexp(a)
    q = np.ldexp(1.0, (e - 8).astype(np.int32))
    n = a / q
    r = np.floor(n)
    frac = n - r
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2) == 1))
    r = r + up
    v = np.copysign(r * q, x)
    v = np.where(a == 0, x, v)
    bits = v.astype(np.float32).view(np.uint32) >> np.uint32(16)
    return bits.astype(np.uint16)


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------


def combine(y_rows: np.ndarray, row_of_slot: np.ndarray, topk_w: np.ndarray, y_shared=None) -> np.ndarray:
    """y[t] = sum_k g[t,k] * y_rows[row_of_slot[t*K + k]] (+ y_shared[t]),
    summed in k order (chapter 11, 11.3.1 step 6; plumephp.com worked
    example: the output is the gate-weighted sum of the chosen experts)."""
    w = np.asarray(topk_w, np.float64)
    S, K = w.shape
    y_rows = np.asarray(y_rows, np.float64)
    ros = np.asarray(row_of_slot).reshape(S, K)
    out = np.zeros((S, y_rows.shape[1]), dtype=np.float64)
    for k in range(K):
        out += w[:, k:k + 1] * y_rows[ros[:, k]]
    if y_shared is not None:
        out += np.asarray(y_shared, np.float64)
    return out


def moe_layer(x, topk_idx, topk_w, expert_fn, num_experts, shared_fn=None):
    """y_t = sum_{k} g_{t,k} E_{e_{t,k}}(x_t) (+ shared expert E_s(x_t), gate 1).

    Chapter 11, 11.1.1: y = sum_i R(x)_i E_i(x) with R zero outside TopK;
    chapter 11, 11.1.2: the S*K expert forwards are evaluated grouped by
    expert (one matrix product per expert), which is how this loop runs:
    expert_fn(e, rows) -> outputs for those rows.
    """
    x = np.asarray(x, dtype=np.float64)
    S = x.shape[0]
    idx = np.asarray(topk_idx)
    w = np.asarray(topk_w, np.float64)
    y = None
    for e in range(num_experts):
        ts, ks = np.nonzero(idx == e)
        if len(ts) == 0:
            continue
        out = expert_fn(e, x[ts])
        if y is None:
            y = np.zeros((S, out.shape[1]))
        for j in range(len(ts)):
            y[ts[j]] += w[ts[j], ks[j]] * out[j]
    if y is None:
        y = np.zeros_like(x)
    if shared_fn is not None:
        y = y + shared_fn(x)
    return y


def moe_layer_dense(x, topk_idx, topk_w, expert_fn, num_experts, shared_fn=None):
    """The same layer computed densely: every expert on every token, then the
    outputs weighted by R(x)_i, which is zero outside the TopK set (chapter
    11, 11.1.1 with the -inf sparsifier).  Must agree with ``moe_layer``."""
    x = np.asarray(x, dtype=np.float64)
    S = x.shape[0]
    idx = np.asarray(topk_idx)
    w = np.asarray(topk_w, np.float64)
    dense_w = np.zeros((S, num_experts))
    for t in range(S):
        for k in range(idx.shape[1]):
            dense_w[t, idx[t, k]] = w[t, k]
    y = 0.0
    for e in range(num_experts):
        y = y + dense_w[:, e:e + 1] * expert_fn(e, x)
    if shared_fn is not None:
        y = y + shared_fn(x)
    return y


def soft_routing(x, logits, expert_fn, num_experts, tau=1.0):
    """Soft routing (chapter 11, 11.3.3): y = sum_i softmax(s/tau)_i E_i(x)
    over all experts."""
    l = np.asarray(logits, np.float64) / tau
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    y = 0.0
    for e in range(num_experts):
        y = y + p[:, e:e + 1] * expert_fn(e, np.asarray(x, np.float64))
    return y


# ----------------------------------------------------------------------------
# aux-loss-free bias update (NEXT row: the selection bias follows the load)
# ----------------------------------------------------------------------------


class WindowBias:
    """Sliding-window expert counts and the selection-bias update of
    ybb.press 2.3 (aux-loss-free routing: the bias added to the selection
    keys is recomputed from a sliding window of recent tokens' expert
    choices; the page's window holds 1000 tokens).

    The page does not print the update rule.  Reading taken: after each
    batch, b_e <- b_e + gamma * sign(mean - count_e) in float32, where count_e
    is expert e's number of (token, k) slots among the last `window` tokens and
    mean = tokens_in_window * K / E; under-loaded experts move up, over-loaded
    ones down.

    The window is a ring of `window` token positions filled from position 0;
    a batch of S tokens occupies the next S positions (only its last `window`
    tokens when S >= window).
    """

    def __init__(self, num_experts: int, top_k: int, window: int):
        self.E, self.K, self.W = num_experts, top_k, window
        self.ring = np.full((window, top_k), -1, dtype=np.int64)
        self.filled = 0
        self.head = 0

    def counts(self) -> np.ndarray:
        ids = self.ring[self.ring >= 0]
        return np.bincount(ids, minlength=self.E).astype(np.int32)

    def update(self, topk_idx: np.ndarray, sel_bias: np.ndarray, gamma: float):
        idx = np.asarray(topk_idx, dtype=np.int64)
        idx = np.where((idx >= 0) & (idx < self.E), idx, -1)  # ids outside [0, E) are not counted
        S = idx.shape[0]
        if S >= self.W:
            self.ring[:] = idx[S - self.W:]
            self.filled, self.head = self.W, 0
        else:
            for i in range(S):
                self.ring[(self.head + i) % self.W] = idx[i]
            self.filled = min(self.W, self.filled + S)
            self.head = (self.head + S) % self.W
        c = self.counts()
        mean = np.float32(self.filled * self.K) / np.float32(self.E)
        b = np.asarray(sel_bias, dtype=np.float32).copy()
        g = np.float32(gamma)
        for e in range(self.E):
            diff = np.float32(mean - np.float32(c[e]))
            if diff > 0:
                b[e] = np.float32(b[e] + g)
            elif diff < 0:
                b[e] = np.float32(b[e] - g)
        return b, c


# ----------------------------------------------------------------------------
# W8A8: E4M3 activations with per-row scales (NEXT row)
# ----------------------------------------------------------------------------


def f32_to_e4m3_bits(v: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 bit patterns, round to nearest, ties to even,
    saturating at +-448 (the largest finite E4M3 value); NaN -> 0x7F.

    The E4M3 grid: exponent e in [-6, 8] with 3 mantissa bits (spacing
    2**(e-3)); below 2**-6 the subnormal spacing is 2**-9.  Rounding is done
    on the exact float64 value of the float32 input (no double rounding).
    """
    x = np.asarray(v, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    flat, o = x.reshape(-1), out.reshape(-1)
    for i, val in enumerate(flat):
        if math.isnan(val):
            o[i] = 0x7F
            continue
        sign = 0x80 if math.copysign(1.0, val) < 0 else 0
        a = abs(val)
        if a >= 448.0:
            o[i] = sign | 0x7E
            continue
        if a == 0.0:
            o[i] = sign
            continue
        e = max(math.frexp(a)[1] - 1, -6)  # exponent of the grid containing a
        q = math.ldexp(1.0, e - 3)         # spacing of that grid
        n = a / q
        r = math.floor(n)
        frac = n - r
        if frac > 0.5 or (frac == 0.5 and r % 2 == 1):
            r += 1
        val_r = r * q
        if val_r > 448.0:
            val_r = 448.0
        # encode val_r exactly
        if val_r < math.ldexp(1.0, -6):
            o[i] = sign | int(round(val_r / math.ldexp(1.0, -9)))
        else:
            m, ee = math.frexp(val_r)  # val_r = m * 2**ee, m in [0.5, 1)
            exp_field = ee - 1 + 7
            mant = int(round((m * 2.0 - 1.0) * 8.0))
            if mant == 8:  # rounding carried into the next binade
                mant, exp_field = 0, exp_field + 1
            o[i] = sign | (exp_field << 3) | mant
    return out


def quantize_rows_e4m3(rows: np.ndarray):
    """Per-row E4M3 quantisation of float32 rows (the W8A8 activations):
    amax = max_j |x_j|; scale s = amax / 448 as one float32 division (1 when
    the row is all zero); codes q_j = E4M3(x_j / s), the quotient a float32
    division, rounded to nearest even.  Returns (codes uint8 [n, d], s float32
    [n]); the dequantised row is q * s."""
    x = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    s = np.where(amax > 0, np.divide(amax, np.float32(448.0), dtype=np.float32), np.float32(1.0)).astype(np.float32)
    ratio = np.divide(x, s[:, None], dtype=np.float32)
    return f32_to_e4m3_bits(ratio), s


def split_rows_e4m3(rows: np.ndarray):
    """Two-term E4M3 codes of float32 rows holding bf16 values: the
    activation operand of E4M3-weight layers with bf16 activations.  The
    pages give E4M3 only as the expert weights' storage format (ybb.press
    3.3); the library's tensor-core GEMMs have no bf16 x E4M3 product, so it
    writes each bf16 value as a power-of-two multiple of the sum of two E4M3
    values.  Per row:

        k  = the largest integer with amax * 2**k <= 448 (0 for an all-zero
             row), clamped to [-126, 126]
        v  = x * 2**k                 (float32 product)
        c1 = E4M3(v)                  (round to nearest even)
        c2 = E4M3(v - value(c1))      (float32 difference)
        scale = 2**-k                 (NaN when the row holds an inf or NaN;
                                       its codes are then all zero)

    Returns (c1 uint8 [n, d], c2 uint8 [n, d], scale float32 [n]); the row is
    (value(c1) + value(c2)) * scale."""
    x = np.asarray(rows, dtype=np.float32)
    n, d = x.shape
    c1 = np.zeros((n, d), dtype=np.uint8)
    c2 = np.zeros((n, d), dtype=np.uint8)
    scale = np.zeros(n, dtype=np.float32)
    for i in range(n):
        row = x[i]
        if not np.all(np.isfinite(row)):
            scale[i] = np.float32(np.nan)  # the row's outputs are NaN through its scale
            continue
        else:
            amax = float(np.max(np.abs(row.astype(np.float64)))) if d else 0.0
            k = 0
            if amax > 0.0:
                f, ex = math.frexp(amax)  # amax = f * 2**ex, f in [0.5, 1); 448 = 0.875 * 2**9
                k = (9 if f <= 0.875 else 8) - ex
                k = max(-126, min(126, k))
            mult, scale[i] = np.float32(math.ldexp(1.0, k)), np.float32(math.ldexp(1.0, -k))
        v = np.multiply(row, mult, dtype=np.float32)
        c1[i] = f32_to_e4m3_bits(v)
        rest = np.subtract(v, e4m3_bits_to_f64(c1[i]).astype(np.float32), dtype=np.float32)
        c2[i] = f32_to_e4m3_bits(rest)
    return c1, c2, scale


def expert_swiglu_w8a8(x, q_gate, q_up, q_down, s_gate, s_up, s_down, round_hidden_bf16=True):
    """SwiGLU expert with E4M3 weights (per-output-channel scales) applied to
    E4M3-quantised activations: x rows are quantised per row
    (``quantize_rows_e4m3``), the hidden rows are rounded to bfloat16 and
    quantised per row again before the down projection.  float64 sums."""
    x = np.asarray(x, dtype=np.float64)
    qx, sx = quantize_rows_e4m3(x.astype(np.float32))
    xq = e4m3_bits_to_f64(qx) * sx[:, None].astype(np.float64)
    wg = e4m3_bits_to_f64(q_gate) * np.asarray(s_gate, np.float64)[:, None]
    wu = e4m3_bits_to_f64(q_up) * np.asarray(s_up, np.float64)[:, None]
    wd = e4m3_bits_to_f64(q_down) * np.asarray(s_down, np.float64)[:, None]
    hid = silu(xq @ wg.T) * (xq @ wu.T)
    if round_hidden_bf16:
        hid = bf16_bits_to_f64(f64_to_bf16_bits_fast(hid))
    qh, sh = quantize_rows_e4m3(hid.astype(np.float32))
    hq = e4m3_bits_to_f64(qh) * sh[:, None].astype(np.float64)
    return hq @ wd.T

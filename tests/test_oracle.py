"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests restates the oracle's own formulas: each compares it with
a printed worked example, a brute-force enumeration, a closed form, a special
case that reduces to a textbook routine, or an invariant stated on the pages.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# worked example (plumephp.com, routing worked example block)
# ----------------------------------------------------------------------------


def _worked_example():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


def test_worked_example_top2_and_gates():
    ex = _worked_example()
    p = np.array(ex["probabilities"])
    # any logits whose softmax is p: log p (softmax is shift invariant)
    logits = np.log(p).astype(np.float32)[None, :]
    idx, w = O.select_experts(logits, 2, renormalize=True)
    assert idx[0].tolist() == ex["expected_top2"]
    np.testing.assert_allclose(w[0], ex["expected_gates_normalised"], rtol=1e-6)
    idx, w = O.select_experts(logits, 2, renormalize=False)
    assert idx[0].tolist() == ex["expected_top2"]
    np.testing.assert_allclose(w[0], ex["expected_gates_unnormalised"], rtol=1e-6)


def test_worked_example_output_is_weighted_sum():
    """Output = 0.55*e0(x) + 0.30*e3(x) (unnormalised) with experts whose
    outputs are known in closed form: expert e maps x to (e + 1) * x."""
    ex = _worked_example()
    logits = np.log(np.array(ex["probabilities"])).astype(np.float32)[None, :]
    x = np.array([[1.0, -2.0, 0.5]])
    expert = lambda e, rows: (e + 1.0) * rows
    for renorm, gates in ((False, ex["expected_gates_unnormalised"]), (True, ex["expected_gates_normalised"])):
        idx, w = O.select_experts(logits, 2, renormalize=renorm)
        y = O.moe_layer(x, idx, w, expert, 8)
        expect = gates[0] * 1.0 * x + gates[1] * 4.0 * x  # e0 -> 1x, e3 -> 4x
        np.testing.assert_allclose(y, expect, rtol=1e-6)


# ----------------------------------------------------------------------------
# top-k selection against brute force
# ----------------------------------------------------------------------------


def _brute_topk(keys_row, k, cand=None):
    """Plain repeated selection: scan for the best remaining key (strict '>'
    keeps the lower index on ties; NaN counts as -inf)."""
    n = len(keys_row)
    kv = [(-math.inf if math.isnan(float(v)) else float(v)) for v in keys_row]
    taken = [False] * n
    out = []
    for _ in range(k):
        best = -1
        for j in range(n):
            if taken[j] or (cand is not None and not cand[j]):
                continue
            if best < 0 or kv[j] > kv[best]:
                best = j
        taken[best] = True
        out.append(best)
    return out


@pytest.mark.parametrize("E,K", [(8, 2), (64, 8), (256, 8), (5, 5), (32, 1)])
def test_softmax_topk_matches_brute_force_with_ties(E, K):
    rng = np.random.default_rng(E * 100 + K)
    # small integer logits force many ties
    logits = rng.integers(-3, 4, size=(40, E)).astype(np.float32)
    logits[0, :] = 1.0  # all tied
    logits[1, 0] = np.nan
    logits[2, :] = -np.inf
    idx, w = O.select_experts(logits, K)
    for t in range(logits.shape[0]):
        assert idx[t].tolist() == _brute_topk(logits[t], K), t
    assert np.all(np.isfinite(w[3:]))
    np.testing.assert_allclose(w[3:].sum(axis=1), 1.0, rtol=1e-12)


def test_softmax_gates_textbook():
    """Unnormalised gates equal the textbook softmax probability of each
    chosen expert; normalised gates equal the softmax of the chosen logits."""
    rng = np.random.default_rng(1)
    l = rng.normal(size=(20, 8)).astype(np.float32)
    idx, w = O.select_experts(l, 2, renormalize=False)
    p = torch.softmax(torch.tensor(l, dtype=torch.float64), dim=1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=1e-12)
    idx2, w2 = O.select_experts(l, 2, renormalize=True)
    assert (idx2 == idx).all()
    sel = torch.tensor(np.take_along_axis(l, idx, 1), dtype=torch.float64)
    np.testing.assert_allclose(w2, torch.softmax(sel, dim=1).numpy(), rtol=1e-12)
    # TopK(-inf) then softmax over all E (chapter 11, 11.1.1 as written)
    masked = np.full_like(l, -np.inf, dtype=np.float64)
    np.put_along_axis(masked, idx, np.take_along_axis(l, idx, 1).astype(np.float64), 1)
    pm = torch.softmax(torch.tensor(masked), dim=1).numpy()
    np.testing.assert_allclose(w2, np.take_along_axis(pm, idx, 1), rtol=1e-12)


# ----------------------------------------------------------------------------
# group-limited sigmoid selection against brute-force enumeration
# ----------------------------------------------------------------------------


def test_grouped_selection_brute_force_dyadic():
    """Keys on a coarse dyadic grid make every float32 sum exact, so the group
    scores can be summed in any order.  The chosen groups must be the pair of
    groups with the largest total among all C(8,2)=28 pairs (lexicographically
    first on ties), and the top-8 the best keys inside them."""
    rng = np.random.default_rng(7)
    E, G, TG, K = 256, 8, 2, 8
    gs = E // G
    n_tok = 60
    # sigmoid keys: choose the selection bias so that s + b lands on a grid
    logits = rng.normal(size=(n_tok, E)).astype(np.float32)
    s = O.sigmoid_f32(logits)
    target = (rng.integers(0, 16, size=(n_tok, E)) / 16.0).astype(np.float32)
    for t in range(n_tok):
        # per-token bias is not allowed (bias is per expert), so check each
        # token with its own bias vector
        bias = (target[t] - s[t]).astype(np.float32)
        keys = np.add(s[t], bias, dtype=np.float32)
        idx, w = O.select_experts(logits[t:t + 1], K, score_fn="sigmoid", sel_bias=bias, num_groups=G,
                                  topk_groups=TG)
        gsum = [float(np.sum(keys[g * gs:(g + 1) * gs].astype(np.float64))) for g in range(G)]
        best_pair = max(itertools.combinations(range(G), TG), key=lambda pr: (sum(gsum[g] for g in pr),
                                                                              [-g for g in pr]))
        cand = np.zeros(E, dtype=bool)
        for g in best_pair:
            cand[g * gs:(g + 1) * gs] = True
        assert idx[0].tolist() == _brute_topk(keys, K, cand), t
        assert all(cand[i] for i in idx[0])  # chosen experts lie inside chosen groups
        # gates: unbiased sigmoid scores, normalised
        sk = s[t][idx[0]].astype(np.float64)
        np.testing.assert_allclose(w[0], sk / sk.sum(), rtol=1e-12)


def _group_row_with_cancellation():
    """32 float32 members: 2**25 at member 0, -2**25 at member 16, and
    c = float32(0.7) (not dyadic) everywhere else."""
    v = np.full(32, np.float32(0.7), dtype=np.float32)
    v[0], v[16] = np.float32(2.0 ** 25), np.float32(-2.0 ** 25)
    return v


def test_group_sums_f32_is_the_halving_tree():
    """The group score of the grouped selection adds member j + 16 to member
    j, then j + 8, j + 4, j + 2, j + 1 (a fixed float32 order).  On the row
    of ``_group_row_with_cancellation`` that order gives exactly 21, by hand:
    with c = 11744051 * 2**-24 (float32(0.7)),
      stride 16: 2**25 - 2**25 = 0 and fifteen sums 2c (exact);
      stride 8:  0 + 2c = 2c and seven sums 4c (exact);
      stride 4:  2c + 4c = 70464306 * 2**-24, rounded to the 2**-21 grid
                 -> 70464304 * 2**-24; three sums 8c (exact);
      stride 2:  70464304 + 93952408 = 164416712 (units of 2**-24), a tie on
                 the 2**-20 grid -> even -> 164416704; one sum 16c;
      stride 1:  164416704 + 187904816 = 352321520, a tie on the 2**-19 grid
                 -> even -> 352321536 = 21 * 2**24, i.e. 21.0.
    A left-to-right sum or adjacent pairing (j with j + 1) gives other
    float32 values on the same row, so either slip fails here."""
    v = _group_row_with_cancellation()
    assert O.group_sums_f32(v) == np.float32(21.0)
    # vectorised over leading axes: the same row in a [2, 3, 32] batch
    batch = np.broadcast_to(v, (2, 3, 32)).copy()
    batch[1, 2] = np.float32(0.5)  # 32 * 0.5 = 16 exactly in any order
    got = O.group_sums_f32(batch)
    assert got.shape == (2, 3)
    assert got[1, 2] == np.float32(16.0)
    assert np.all(np.delete(got.reshape(-1), 5) == np.float32(21.0))
    # the row discriminates: the two other plausible orders differ from 21
    ltr = np.float32(0.0)
    for m in v:
        ltr = np.float32(ltr + m)
    adj = v.copy()
    while len(adj) > 1:
        adj = np.add(adj[0::2], adj[1::2], dtype=np.float32)
    assert ltr != np.float32(21.0) and adj[0] != np.float32(21.0) and ltr != adj[0]


def test_group_limited_selection_uses_the_halving_order():
    """Two groups of 32 softmax keys, keep one group, top-1.  Group 0 holds
    the cancellation row (halving sum 21, see above); group 1 holds 32 keys
    0.609375 (exact dyadic sum 19.5 in any order).  The halving order keeps
    group 0, whose best key (2**25, expert 0) wins; a left-to-right or
    adjacent-pair group sum (both below 19.5 on this row) would keep group 1
    and pick expert 32."""
    keys = np.concatenate([_group_row_with_cancellation(), np.full(32, np.float32(0.609375))])[None, :]
    idx, w = O.select_experts(keys, 1, num_groups=2, topk_groups=1)
    assert idx.tolist() == [[0]]
    np.testing.assert_allclose(w, [[1.0]])
    # and when group 1's exact sum is above 21 (0.671875 * 32 = 21.5), group 1 wins
    keys2 = np.concatenate([_group_row_with_cancellation(), np.full(32, np.float32(0.671875))])[None, :]
    idx2, _ = O.select_experts(keys2, 1, num_groups=2, topk_groups=1)
    assert idx2.tolist() == [[32]]


# ----------------------------------------------------------------------------
# float32 sigmoid / exponential against the mathematics
# ----------------------------------------------------------------------------


def test_exp_f32_within_two_ulp_of_math_exp():
    z = np.concatenate([np.linspace(-30, 88, 400001), np.array([0.0, 1.0, -1.0, 0.5])]).astype(np.float32)
    e = O.exp_f32(z).astype(np.float64)
    ref = np.array([math.exp(float(v)) for v in z[::37]])
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(e[::37] - ref) / ulp) <= 2.0
    assert O.exp_f32(np.float32(0.0)) == 1.0


def test_sigmoid_f32_special_values():
    assert O.sigmoid_f32(np.float32(0.0)) == np.float32(0.5)
    big = O.sigmoid_f32(np.array([100.0, -100.0, np.inf, -np.inf], dtype=np.float32))
    assert big.tolist() == [1.0, 0.0, 1.0, 0.0]
    x = np.linspace(-20, 20, 10001).astype(np.float32)
    s = O.sigmoid_f32(x).astype(np.float64)
    ref = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    assert np.max(np.abs(s - ref) / np.maximum(ref, 1e-30)) < 4e-7
    assert np.all(np.diff(s) >= 0)  # monotone


# ----------------------------------------------------------------------------
# histogram, scan, permutation: invariants from the pages
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("capacity", [0, 3, 1])
def test_permutation_invariants(capacity):
    rng = np.random.default_rng(3)
    S, E, K = 50, 8, 3
    logits = rng.normal(size=(S, E)).astype(np.float32)
    logits[:, 2] += 2.0  # a hot expert
    idx, _ = O.select_experts(logits, K)
    P = O.expert_permutation(idx, E, capacity)
    # every token goes to K experts (chapter 11, 11.1.2): counts sum to S*K
    assert P["counts"].sum() == S * K
    assert P["counts"].tolist() == [int((idx == e).sum()) for e in range(E)]
    off = P["offsets"]
    assert off[0] == 0 and off[-1] == S * K and np.all(np.diff(off) >= 0)
    ros, tor = P["row_of_slot"], P["token_of_row"]
    # bijection between slots and used rows; no token dropped (ybb.press 2.2)
    assert len(set(ros.tolist())) == S * K
    assert np.all(ros >= 0) and np.all(ros < P["num_rows"])
    for slot in range(S * K):
        assert tor[ros[slot]] == slot // K
    assert (tor >= 0).sum() == S * K
    # stable: within each expert, rows follow slot order
    flat = idx.reshape(-1)
    for e in range(E):
        rows = ros[flat == e]
        assert np.all(np.diff(rows) > 0)
    if capacity:
        C = capacity
        assert np.all(P["prim_counts"] <= C)
        assert (P["prim_counts"] + P["ovf_counts"] == P["counts"]).all()
        for e in range(E):
            rows = ros[flat == e]
            prim = rows[rows < E * C]
            assert np.all((prim >= e * C) & (prim < (e + 1) * C))
    else:
        for e in range(E):
            rows = ros[flat == e]
            assert np.all((rows >= off[e]) & (rows < off[e + 1]))


def test_overflow_region_is_expert_major():
    """ybb.press 2.2 (overflow buffering), with the layout read as: the E*C
    primary rows first, then the overflow rows expert by expert, each
    expert's in slot order.  Hand-built case, E = 3, C = 1, K = 2:
        token 0 -> (e0, e2), token 1 -> (e2, e0), token 2 -> (e1, e2)
    slots 0..5 = e0, e2, e2, e0, e1, e2; counts (2, 1, 3).
    Primary rows: e0 keeps slot 0 (row 0), e1 slot 4 (row 1), e2 slot 1
    (row 2).  Overflow counts (1, 0, 2) -> overflow offsets (0, 1, 1, 3):
    e0's excess slot 3 -> row 3 + 0 = 3; e2's excess slots 2, 5 -> rows
    3 + 1 = 4 and 5.  A token-major overflow layout would put slot 2 at row 3
    and slot 3 at row 4 instead."""
    idx = np.array([[0, 2], [2, 0], [1, 2]], dtype=np.int32)
    P = O.expert_permutation(idx, 3, capacity=1)
    assert P["counts"].tolist() == [2, 1, 3]
    assert P["prim_counts"].tolist() == [1, 1, 1]
    assert P["ovf_counts"].tolist() == [1, 0, 2]
    assert P["ovf_offsets"].tolist() == [0, 1, 1, 3]
    assert P["num_rows"] == 3 * 1 + 3 * 2
    assert P["row_of_slot"].tolist() == [0, 2, 4, 3, 1, 5]
    assert P["token_of_row"].tolist() == [0, 2, 0, 1, 1, 2, -1, -1, -1]
    # without capacity: plain stable grouping, offsets (0, 2, 3, 6)
    Q = O.expert_permutation(idx, 3)
    assert Q["offsets"].tolist() == [0, 2, 3, 6]
    assert Q["row_of_slot"].tolist() == [0, 3, 4, 1, 2, 5]
    assert Q["token_of_row"].tolist() == [0, 1, 2, 0, 1, 2]


def test_load_stats_uniform_and_skewed():
    st = O.load_stats(np.array([4, 4, 4, 4]), 2, 8)
    assert st["max_over_mean"] == 1.0 and st["std"] == 0.0
    assert st["overflow_rows"] == 0 and st["dropped"] == 0
    # S*K = 16 slots over 4 experts: mean 4; deviations 9, -3, -3, -3 -> variance
    # (81 + 27) / 4 = 27, std = 3 * sqrt(3); capacity 3 leaves 13 - 3 = 10 rows over
    st = O.load_stats(np.array([13, 1, 1, 1]), 2, 8, capacity=3)
    assert st["max_over_mean"] == pytest.approx(3.25)
    assert st["std"] == pytest.approx(3.0 * math.sqrt(3.0), rel=1e-15)
    assert st["mean"] == 4.0 and st["max"] == 13.0
    assert st["overflow_rows"] == 10.0 and st["dropped"] == 0.0
    # one slot with an out-of-range id is counted nowhere: dropped = 1
    st = O.load_stats(np.array([12, 1, 1, 1]), 2, 8)
    assert st["dropped"] == 1.0 and st["overflow_rows"] == 0.0


# ----------------------------------------------------------------------------
# experts: closed forms and special cases
# ----------------------------------------------------------------------------


def test_gelu_erf_textbook_values():
    # GeLU(z) = z * Phi(z); Phi(1) = 0.8413447460685429 (normal table)
    g = O.gelu_erf(np.array([0.0, 1.0, -1.0, 8.0, -8.0]))
    np.testing.assert_allclose(g[:3], [0.0, 0.8413447460685429, -1 + 0.8413447460685429], rtol=1e-15, atol=1e-16)
    assert g[3] == pytest.approx(8.0) and abs(g[4]) < 1e-12


def test_silu_values():
    s = O.silu(np.array([0.0, 1.0, -1.0]))
    np.testing.assert_allclose(s, [0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1))], rtol=1e-15)


def test_expert_gelu_one_hot_weights():
    """W1 = identity-like, b1 = 0, W2 = identity, b2 = c: output is
    GeLU(x) + c elementwise."""
    d = 4
    x = np.array([[0.5, -1.0, 2.0, 0.0]])
    w1 = np.eye(d)
    w2 = np.eye(d)
    c = np.array([0.1, 0.2, 0.3, 0.4])
    y = O.expert_gelu(x, w1, np.zeros(d), w2, c)
    np.testing.assert_allclose(y, O.gelu_erf(x) + c, rtol=1e-15)
    # W1 stored out x in: a permutation matrix routes input j to hidden p(j)
    perm = np.eye(d)[[2, 0, 3, 1]]
    y2 = O.expert_gelu(x, perm, np.zeros(d), np.eye(d), np.zeros(d))
    np.testing.assert_allclose(y2[0], O.gelu_erf(x[0][[2, 0, 3, 1]]), rtol=1e-15)


def test_expert_swiglu_closed_form():
    """h=1: Wg row a, Wu row b, Wd column c -> y = silu(x.a) * (x.b) * c."""
    x = np.array([[1.0, 2.0], [-1.0, 0.5]])
    a, b, c = np.array([[0.5, -0.25]]), np.array([[1.0, 1.0]]), np.array([[2.0], [-3.0]])
    y = O.expert_swiglu(x, a, b, c)
    for t in range(2):
        za, zb = float(x[t] @ a[0]), float(x[t] @ b[0])
        hval = za / (1 + math.exp(-za)) * zb
        np.testing.assert_allclose(y[t], [2.0 * hval, -3.0 * hval], rtol=1e-14)
    # per-channel scales multiply the weight rows
    y2 = O.expert_swiglu(x, a, b, c, s_gate=np.array([2.0]), s_up=np.array([0.5]), s_down=np.array([1.0, 1.0]))
    y3 = O.expert_swiglu(x, 2 * a, 0.5 * b, c)
    np.testing.assert_allclose(y2, y3, rtol=1e-14)


def _rand_gelu_experts(rng, E, d, h):
    w1 = rng.normal(size=(E, h, d)) / math.sqrt(d)
    b1 = rng.normal(size=(E, h)) * 0.1
    w2 = rng.normal(size=(E, d, h)) / math.sqrt(h)
    b2 = rng.normal(size=(E, d)) * 0.1
    return (lambda e, rows: O.expert_gelu(rows, w1[e], b1[e], w2[e], b2[e])), (w1, b1, w2, b2)


def test_sparse_layer_equals_dense_then_mask():
    rng = np.random.default_rng(11)
    S, d, E, K, h = 30, 16, 8, 2, 24
    fn, _ = _rand_gelu_experts(rng, E, d, h)
    x = rng.normal(size=(S, d))
    l = rng.normal(size=(S, E)).astype(np.float32)
    idx, w = O.select_experts(l, K)
    np.testing.assert_allclose(O.moe_layer(x, idx, w, fn, E), O.moe_layer_dense(x, idx, w, fn, E),
                               rtol=1e-12, atol=1e-13)
    # and through the permute/combine route with a shared expert
    P = O.expert_permutation(idx, E)
    y_rows = np.zeros((P["num_rows"], d))
    for e in range(E):
        rows = np.arange(P["offsets"][e], P["offsets"][e + 1])
        if len(rows):
            y_rows[rows] = fn(e, x[P["token_of_row"][rows]])
    shared = fn(0, x)
    np.testing.assert_allclose(O.combine(y_rows, P["row_of_slot"], w, shared),
                               O.moe_layer(x, idx, w, fn, E, shared_fn=lambda z: fn(0, z)), rtol=1e-12,
                               atol=1e-13)


def test_single_expert_is_dense_ffn():
    """E = 1, K = 1: the layer is the plain FFN of that expert (gate 1)."""
    rng = np.random.default_rng(2)
    fn, (w1, b1, w2, b2) = _rand_gelu_experts(rng, 1, 8, 12)
    x = rng.normal(size=(5, 8))
    idx, w = O.select_experts(rng.normal(size=(5, 1)).astype(np.float32), 1)
    assert (idx == 0).all() and np.all(w == 1.0)
    hid = x @ w1[0].T + b1[0]
    hid = 0.5 * hid * (1 + np.vectorize(math.erf)(hid / math.sqrt(2)))
    np.testing.assert_allclose(O.moe_layer(x, idx, w, fn, 1), hid @ w2[0].T + b2[0], rtol=1e-12)


def test_k_equals_e_is_soft_routing():
    """K = E with renormalised softmax gates is soft routing with tau = 1
    (chapter 11, 11.3.3)."""
    rng = np.random.default_rng(4)
    S, d, E = 12, 8, 6
    fn, _ = _rand_gelu_experts(rng, E, d, 10)
    x = rng.normal(size=(S, d))
    l = rng.normal(size=(S, E)).astype(np.float32)
    idx, w = O.select_experts(l, E)
    np.testing.assert_allclose(O.moe_layer(x, idx, w, fn, E), O.soft_routing(x, l, fn, E, 1.0), rtol=1e-12)


@pytest.mark.parametrize("tau", [0.5, 2.0, 0.7, 3.0])
def test_temperature_k_equals_e_is_soft_routing(tau):
    """With a temperature, K = E renormalised selection is the soft routing
    y = sum_i softmax(s / tau)_i E_i(x) of chapter 11, 11.3.3 (computed there
    in float64; here the tempered logit is one float32 division, so the two
    agree to float32 rounding)."""
    rng = np.random.default_rng(40)
    S, d, E = 12, 8, 6
    fn, _ = _rand_gelu_experts(rng, E, d, 10)
    x = rng.normal(size=(S, d))
    l = (3.0 * rng.normal(size=(S, E))).astype(np.float32)
    idx, w = O.select_experts(l, E, temperature=tau)
    np.testing.assert_allclose(O.moe_layer(x, idx, w, fn, E), O.soft_routing(x, l, fn, E, tau), rtol=2e-6)
    # the gates themselves: softmax of l / tau over all experts, in each token's slot order
    p = torch.softmax(torch.tensor(l, dtype=torch.float64) / tau, dim=1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=2e-6)


def test_temperature_keeps_the_order_and_sharpens_or_flattens_the_gates():
    """tau > 0 divides every key alike, so the selected experts are those of
    tau = 1 (keys far apart here); tau < 1 moves the top gate up and tau > 1
    moves it toward 1/K, the limits of a softmax temperature."""
    rng = np.random.default_rng(41)
    l = rng.normal(size=(50, 16)).astype(np.float32) * 4.0
    idx1, w1 = O.select_experts(l, 4)
    for tau in (0.25, 4.0):
        idx, w = O.select_experts(l, 4, temperature=tau)
        np.testing.assert_array_equal(idx, idx1)
        if tau < 1:
            assert np.all(w[:, 0] >= w1[:, 0])
        else:
            assert np.all(w[:, 0] <= w1[:, 0]) and np.all(w[:, 0] >= 0.25)
    assert np.array_equal(O.select_experts(l, 4, temperature=1.0)[1], w1)


def test_capacity_does_not_change_the_layer():
    rng = np.random.default_rng(5)
    S, d, E, K = 40, 8, 4, 2
    fn, _ = _rand_gelu_experts(rng, E, d, 8)
    x = rng.normal(size=(S, d))
    l = rng.normal(size=(S, E)).astype(np.float32)
    l[:, 1] += 3.0
    idx, w = O.select_experts(l, K)
    outs = []
    for cap in (0, 5, 17):
        P = O.expert_permutation(idx, E, cap)
        y_rows = np.zeros((P["num_rows"], d))
        tor = P["token_of_row"]
        flat = idx.reshape(-1)
        for slot in range(S * K):
            y_rows[P["row_of_slot"][slot]] = fn(flat[slot], x[slot // K:slot // K + 1])[0]
        assert (tor >= 0).sum() == S * K
        outs.append(O.combine(y_rows, P["row_of_slot"], w))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-13)
    np.testing.assert_allclose(outs[0], outs[2], rtol=1e-13)


# ----------------------------------------------------------------------------
# number formats against torch's converters (library routines)
# ----------------------------------------------------------------------------


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(mine) & np.isnan(ref)
    assert np.all(both_nan | (mine == ref))
    assert mine[0x7E] == 448.0 and mine[0x38] == 1.0 and mine[0xB8] == -1.0 and mine[0x01] == 2.0 ** -9


def test_bf16_round_trip_matches_torch():
    rng = np.random.default_rng(9)
    v = (rng.normal(size=4000) * np.exp(rng.normal(size=4000) * 5)).astype(np.float32)
    v[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # exact ties
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (O.f64_to_bf16_bits(v.astype(np.float64)) == ref).all()
    assert (O.f64_to_bf16_bits_fast(v.astype(np.float64)) == ref).all()
    back = O.bf16_bits_to_f64(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_router_logits_definition():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(3, 5)).astype(np.float32)
    w = rng.normal(size=(4, 5)).astype(np.float32)
    b = np.array([0.5, 0.0, -0.5, 1.0], dtype=np.float32)
    l = O.router_logits(x, w, b)
    for t in range(3):
        for e in range(4):
            exact = math.fsum(float(x[t, k]) * float(w[e, k]) for k in range(5)) + float(b[e])
            assert abs(float(l[t, e]) - exact) <= np.spacing(np.float32(abs(exact)))


# ----------------------------------------------------------------------------
# sliding-window bias update (aux-loss-free routing, ybb.press 2.3)
# ----------------------------------------------------------------------------


def test_window_bias_hand_computed():
    """E=4, K=1, window 4, gamma 0.5: tokens [0,0,0,1] -> counts [3,1,0,0],
    mean 1 -> bias [-0.5, 0, +0.5, +0.5]; then [2,2] replaces the two oldest
    -> window [2,2,0,1], counts [1,1,2,0] -> bias [-0.5, 0, 0, 1.0]."""
    wb = O.WindowBias(4, 1, 4)
    b = np.zeros(4, np.float32)
    b, c = wb.update(np.array([[0], [0], [0], [1]]), b, 0.5)
    assert c.tolist() == [3, 1, 0, 0] and b.tolist() == [-0.5, 0.0, 0.5, 0.5]
    b, c = wb.update(np.array([[2], [2]]), b, 0.5)
    assert c.tolist() == [1, 1, 2, 0] and b.tolist() == [-0.5, 0.0, 0.0, 1.0]
    # a batch longer than the window keeps only its last `window` tokens
    b, c = wb.update(np.array([[3]] * 3 + [[1]] * 4), b, 0.5)
    assert c.tolist() == [0, 4, 0, 0]


def test_window_counts_sum_and_partial_fill():
    wb = O.WindowBias(8, 2, 10)
    rng = np.random.default_rng(0)
    b = np.zeros(8, np.float32)
    seen = []
    for S in (3, 4, 5, 1, 12, 2):
        ridx, _ = O.select_experts(rng.normal(size=(S, 8)).astype(np.float32), 2)
        seen.extend(ridx.tolist())
        b, c = wb.update(ridx, b, 0.01)
        last = np.array(seen[-10:])
        assert c.sum() == min(len(seen), 10) * 2
        assert c.tolist() == np.bincount(last.reshape(-1), minlength=8).tolist()


def test_bias_update_steers_load_toward_balance():
    """The point of the bias (ybb.press 2.3: steer the routing distribution
    without gradients): repeated routing + update under a skewed router must
    lower the max/mean load.  With the sign flipped the skew would grow."""
    rng = np.random.default_rng(1)
    E, K, S = 16, 2, 512
    offs = (rng.normal(size=E) * 1.5).astype(np.float32)
    wb = O.WindowBias(E, K, 1000)
    b = np.zeros(E, np.float32)
    ratios = []
    for it in range(60):
        logits = (rng.normal(size=(S, E)).astype(np.float32) + offs).astype(np.float32)
        idx, _ = O.select_experts(logits, K, "softmax", True, b)
        ratios.append(O.load_stats(O.expert_counts(idx, E), K, S)["max_over_mean"])
        b, _ = wb.update(idx, b, 0.05)
    assert ratios[0] > 2.0 and np.mean(ratios[-10:]) < 0.6 * ratios[0]


# ----------------------------------------------------------------------------
# E4M3 encoder and per-row quantisation (W8A8)
# ----------------------------------------------------------------------------


def test_f32_to_e4m3_matches_torch_rne():
    rng = np.random.default_rng(12)
    v = np.concatenate([
        (rng.normal(size=20000) * np.exp(rng.normal(size=20000) * 3)),
        O.e4m3_bits_to_f64(np.arange(0, 0x7F, dtype=np.uint8)),          # every finite code exactly
        (O.e4m3_bits_to_f64(np.arange(0, 0x7E, dtype=np.uint8)) +
         O.e4m3_bits_to_f64(np.arange(1, 0x7F, dtype=np.uint8))) / 2,   # every tie
    ]).astype(np.float32)
    v = v[np.abs(v) < 464]  # torch's encoder is not saturating past the rounding edge
    mine = O.f32_to_e4m3_bits(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(mine, ref)
    assert O.f32_to_e4m3_bits(np.array([1e6, -500.0], np.float32)).tolist() == [0x7E, 0xFE]  # saturates


def test_quantize_rows_round_trip_error_bound():
    """Dequantised rows are within half an E4M3 step of the input: relative
    2**-4 for normal codes, absolute s * 2**-10 near zero; the row maximum maps
    to 448 exactly."""
    rng = np.random.default_rng(13)
    x = (rng.normal(size=(50, 300)) * np.exp(rng.normal(size=(50, 1)))).astype(np.float32)
    x[3] = 0.0
    q, s = O.quantize_rows_e4m3(x)
    back = O.e4m3_bits_to_f64(q) * s[:, None]
    err = np.abs(back - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * 1.0000001
    assert np.all(err <= bound)
    assert s[3] == 1.0 and np.all(q[3] == 0)
    top = np.argmax(np.abs(x), axis=1)
    nz = np.arange(50) != 3
    assert np.all(np.abs(O.e4m3_bits_to_f64(q[np.arange(50), top]))[nz] == 448.0)


def _bf16_rows(rng, n, d, spread):
    """Random float32 rows holding bf16 values: |x| = amax_row * 2**-u, u
    uniform in [0, spread), random signs, bf16 mantissas."""
    amax = np.exp2(rng.integers(-20, 20, size=(n, 1))) * rng.uniform(1, 2, size=(n, 1))
    x = amax * np.exp2(-rng.uniform(0, spread, size=(n, d))) * rng.choice([-1.0, 1.0], size=(n, d))
    return O.bf16_bits_to_f64(O.f64_to_bf16_bits(x)).astype(np.float32)


def test_split_rows_hand_example():
    """x = [1 + 2**-7, -0.5, 0, 3]: amax 3 = 0.75 * 2**2, so k = 7 (3 * 2**7 =
    384 <= 448 < 768); v = [129, -64, 0, 384].  129 lies on the grid of
    spacing 16 in [128, 256) and rounds to 128 = code 0x70 (exponent field
    14), leaving 1 = code 0x38; -64 = code 0xE8, 384 = 1.5 * 2**8 = code 0x7C,
    all exact; scale 2**-7."""
    c1, c2, s = O.split_rows_e4m3(np.array([[1.0078125, -0.5, 0.0, 3.0]], np.float32))
    assert list(c1[0]) == [0x70, 0xE8, 0x00, 0x7C]
    assert list(c2[0]) == [0x38, 0x00, 0x00, 0x00]
    assert s[0] == np.float32(2.0 ** -7)


def test_split_rows_reconstruct_bf16_exactly():
    """Every bf16 value of at least 2**-9 of its row's largest magnitude is
    the exact sum of its two terms times the row scale (the scaled value is at
    least 224 * 2**-9 > 1/4, so the remainder after the first term, at most 4
    significant bits, lies on the E4M3 grid); the scale is the largest power
    of two bringing the row maximum to at most 448."""
    rng = np.random.default_rng(31)
    x = _bf16_rows(rng, 40, 96, 9.0)
    c1, c2, s = O.split_rows_e4m3(x)
    v1, v2 = O.e4m3_bits_to_f64(c1), O.e4m3_bits_to_f64(c2)
    assert np.array_equal((v1 + v2) * s[:, None].astype(np.float64), x.astype(np.float64))
    top = np.max(np.abs(x.astype(np.float64)), axis=1) / s
    assert np.all((top > 224.0) & (top <= 448.0))
    # the first term alone is the value rounded to 4 significant bits
    assert np.all(np.abs(v2) <= np.abs(v1) * 2.0 ** -4)


def test_split_rows_error_bound_and_special_rows():
    """Values far below the row maximum lose at most 2**-10 of the scaled
    value (half the E4M3 subnormal spacing); a zero row has scale 1 and zero
    codes; a row maximum of exactly 448 * 2**j gives scale 2**j; a row with an
    infinity or a NaN gets the scale NaN and zero codes."""
    rng = np.random.default_rng(32)
    x = _bf16_rows(rng, 30, 128, 30.0)
    c1, c2, s = O.split_rows_e4m3(x)
    v = x.astype(np.float64) / s[:, None]
    err = np.abs(O.e4m3_bits_to_f64(c1) + O.e4m3_bits_to_f64(c2) - v)
    assert np.all(err <= 2.0 ** -10)
    assert np.any(err > 0)  # the spread reaches below the exact range
    y = np.zeros((4, 16), np.float32)
    y[1, 3] = 448.0 * 8
    y[2, 5] = np.inf
    y[3, 0] = np.nan
    c1, c2, s = O.split_rows_e4m3(y)
    assert s[0] == 1.0 and not c1[0].any() and not c2[0].any()
    assert s[1] == 8.0 and c1[1, 3] == 0x7E and c2[1, 3] == 0
    assert np.isnan(s[2]) and np.isnan(s[3])
    assert not c1[2:].any() and not c2[2:].any()


def test_split_rows_expert_equals_bf16_expert_within_bound():
    """A SwiGLU expert fed the two-term reconstruction of bf16 rows
    ((c1 + c2) * scale) equals the expert on the bf16 rows themselves within
    the bound the split guarantees (every element within 2**-10 * scale of its
    value), propagated through the up projections: |x W| changes by at most
    2**-10 * scale * sum_k |W[n, k]|.  On rows of limited spread (every value
    at least 2**-9 of its row maximum) the two agree exactly."""
    rng = np.random.default_rng(33)
    d, h = 48, 40
    wg, wu = rng.normal(size=(h, d)) / 7, rng.normal(size=(h, d)) / 7
    for spread, exact in ((9.0, True), (24.0, False)):
        x = _bf16_rows(rng, 25, d, spread).astype(np.float64)
        c1, c2, sc = O.split_rows_e4m3(x.astype(np.float32))
        xr = (O.e4m3_bits_to_f64(c1) + O.e4m3_bits_to_f64(c2)) * sc[:, None].astype(np.float64)
        if exact:
            assert np.array_equal(xr, x)
        bound_x = 2.0 ** -10 * sc[:, None].astype(np.float64)
        assert np.all(np.abs(xr - x) <= bound_x)
        g, u = x @ wg.T, x @ wu.T
        gr, ur = xr @ wg.T, xr @ wu.T
        bg = bound_x * np.abs(wg).sum(axis=1)[None, :]
        bu = bound_x * np.abs(wu).sum(axis=1)[None, :]
        assert np.all(np.abs(gr - g) <= bg * (1 + 1e-9) + 1e-300)
        assert np.all(np.abs(ur - u) <= bu * (1 + 1e-9) + 1e-300)


def test_w8a8_expert_close_to_exact_expert():
    """With 8-bit activations the expert output stays within the quantisation
    noise of the same expert on unquantised activations (relative L2 a few
    percent), and equals it exactly when activations are E4M3-representable
    multiples of their row scale."""
    rng = np.random.default_rng(14)
    d, h = 64, 96
    wg, wu, wd = (rng.normal(size=(h, d)) / 8, rng.normal(size=(h, d)) / 8, rng.normal(size=(d, h)) / 10)
    qg, sg = (lambda q: (q[0], q[1]))(O.quantize_rows_e4m3(wg.astype(np.float32)))
    qu, su = O.quantize_rows_e4m3(wu.astype(np.float32))
    qd, sd = O.quantize_rows_e4m3(wd.astype(np.float32))
    x = rng.normal(size=(20, d))
    y8 = O.expert_swiglu_w8a8(x, qg, qu, qd, sg, su, sd, round_hidden_bf16=False)
    yref = O.expert_swiglu(x, O.e4m3_bits_to_f64(qg), O.e4m3_bits_to_f64(qu), O.e4m3_bits_to_f64(qd),
                           s_gate=sg, s_up=su, s_down=sd)
    rel = np.linalg.norm(y8 - yref) / np.linalg.norm(yref)
    assert 1e-4 < rel < 5e-2


def test_w8a8_expert_exact_on_representable_rows():
    """With x rows that are E4M3 codes times a power of two (the row maximum
    coding to 448) the activation quantisation is lossless, and with d_ff = 1
    each hidden row has one element, which quantises to +-448 times |h|/448,
    i.e. back to h up to one float32 rounding.  So the W8A8 expert must equal
    the plain SwiGLU expert on the dequantised weights; a wrong activation or
    hidden scale, or swapped weight scales, breaks the equality."""
    rng = np.random.default_rng(15)
    d, n = 32, 12
    codes = rng.integers(0, 0x7F, size=(n, d)).astype(np.uint8) | (rng.integers(0, 2, size=(n, d)) << 7).astype(
        np.uint8)
    codes[:, 0] = 0x7E  # 448: the row maximum
    x = O.e4m3_bits_to_f64(codes) * (2.0 ** rng.integers(-12, 4, size=(n, 1)))
    wg, wu, wd = rng.normal(size=(1, d)) / 4, rng.normal(size=(1, d)) / 4, rng.normal(size=(d, 1))
    qg, sg = O.quantize_rows_e4m3(wg.astype(np.float32))
    qu, su = O.quantize_rows_e4m3(wu.astype(np.float32))
    qd, sd = O.quantize_rows_e4m3(wd.astype(np.float32))
    su = su * 3.0  # distinct gate and up scales, so that swapping them shows
    y8 = O.expert_swiglu_w8a8(x, qg, qu, qd, sg, su, sd, round_hidden_bf16=False)
    yref = O.expert_swiglu(x, O.e4m3_bits_to_f64(qg), O.e4m3_bits_to_f64(qu), O.e4m3_bits_to_f64(qd),
                           s_gate=sg, s_up=su, s_down=sd)
    np.testing.assert_allclose(y8, yref, rtol=1e-6, atol=1e-12 * np.abs(yref).max())


# ----------------------------------------------------------------------------
# over-capacity re-routing (jsqmd.com chapter 11, 11.3.3)
# ----------------------------------------------------------------------------


def _reroute(keys, K, C, cand=None):
    keys = np.asarray(keys, np.float32)
    if cand is None:
        cand = np.ones(keys.shape, bool)
    idx, _ = O.select_experts(keys, K)
    return idx, O.reroute_over_capacity(idx, keys, cand, C)


def test_reroute_hand_computed():
    """E=4, K=1, C=1.  Three tokens all prefer e0: t0 keeps it; t1 (excess)
    takes its best expert with room, e1; t2 then finds e1 full and takes e3
    (key 2 beats e2's 1)."""
    idx, (new, moved) = _reroute([[4, 3, 2, 1], [4, 3, 2, 1], [4, 3, 1, 2]], 1, 1)
    assert idx[:, 0].tolist() == [0, 0, 0]
    assert new[:, 0].tolist() == [0, 1, 3]
    assert moved[:, 0].tolist() == [False, True, True]
    # a slot that finds no room keeps its expert (and its overflow row)
    idx, (new, moved) = _reroute([[2, 1], [2, 1], [2, 1]], 1, 1)
    assert new[:, 0].tolist() == [0, 1, 0] and moved[:, 0].tolist() == [False, True, False]


def test_reroute_skips_held_and_non_candidate_experts():
    """E=4, K=2, C=2: t2's excess slot (e0) cannot take e2, which t2 already
    holds, nor e1 (full), nor e3 outside its candidates; nothing is left, so
    it stays.  With e3 a candidate it moves there."""
    keys = [[4, 3, 2, 1], [4, 3, 1, 2], [4, 1, 3, 2]]
    cand = np.ones((3, 4), bool)
    cand[2, 3] = False
    idx, (new, moved) = _reroute(keys, 2, 2, cand)
    assert idx.tolist() == [[0, 1], [0, 1], [0, 2]]
    assert new.tolist() == idx.tolist() and not moved.any()
    idx, (new, moved) = _reroute(keys, 2, 2)
    assert new.tolist() == [[0, 1], [0, 1], [3, 2]] and moved.tolist() == [[False] * 2, [False] * 2, [True, False]]


def test_reroute_invariants_on_a_skewed_batch():
    rng = np.random.default_rng(21)
    S, E, K = 600, 16, 4
    keys = (rng.normal(size=(S, E)) + 1.5 * rng.normal(size=E)[None, :]).astype(np.float32)
    C = O_cap = int(np.ceil(1.1 * S * K / E))
    idx, (new, moved) = _reroute(keys, K, C)
    counts0 = O.expert_counts(idx, E)
    assert counts0.max() > C                                     # the batch really overflows
    # slots are moved only out of overloaded experts, never within a token twice
    assert all(len(set(r.tolist())) == K for r in new)
    P0 = O.expert_permutation(idx, E, C)
    excess = (P0["row_of_slot"] >= E * C).reshape(S, K)
    assert not (moved & ~excess).any()
    assert (new[~moved] == idx[~moved]).all()
    # every expert that received moved slots stays within its capacity
    counts1 = O.expert_counts(new, E)
    recv = np.bincount(new[moved], minlength=E)
    assert (counts1[recv > 0] <= C).all()
    # a moved slot's new expert ranks below all of the token's original K
    t, k = np.nonzero(moved)
    kth = np.sort(np.take_along_axis(keys, idx, 1), axis=1)[:, 0]
    assert (keys[t, new[t, k]] <= kth[t]).all()
    # the total room is large enough here, so every excess slot finds an expert
    assert moved.sum() == excess.sum()
    # unbounded capacity changes nothing
    _, (same, none) = _reroute(keys, K, S)
    assert (same == idx).all() and not none.any()
    assert O_cap == C


def test_reroute_visit_order_is_slot_order():
    """Two excess slots compete for the last unit of room: the earlier slot
    in (token, k) order wins, the later one takes the next best."""
    keys = [[9, 1, 5, 4], [9, 2, 5, 4], [9, 3, 5, 4]]
    idx, (new, moved) = _reroute(keys, 1, 1)
    # t0 keeps e0; t1 -> e2 (5); t2 -> e2 full -> e3 (4)
    assert new[:, 0].tolist() == [0, 2, 3]


def test_gate_weights_match_selection():
    rng = np.random.default_rng(22)
    logits = rng.normal(size=(50, 12)).astype(np.float32)
    for fn in ("softmax", "sigmoid"):
        for renorm in (True, False):
            idx, w = O.select_experts(logits, 3, fn, renorm)
            scores, _, _ = O.selection_keys(logits, fn)
            np.testing.assert_allclose(O.gate_weights(scores, idx, fn, renorm), w, rtol=0, atol=0)


def test_selection_margin_hand_computed_and_stability():
    """The margin is the gap between the K-th and (K+1)-th candidate keys
    (and between the last kept and first dropped group score with groups);
    any perturbation of the keys smaller than half of it leaves the selection
    unchanged, and one slightly larger can change it."""
    l = np.array([[3.0, 1.0, 2.0, 0.5]], np.float32)
    assert O.selection_margin(l, 1)[0] == 1.0              # 3 vs 2
    assert O.selection_margin(l, 2)[0] == 1.0              # 2 vs 1
    assert O.selection_margin(l, 3)[0] == 0.5              # 1 vs 0.5
    # groups of 2: group sums (3+1, 2+0.5) = (4, 2.5): keep 1 group -> margin min(1.5, key gap inside)
    assert O.selection_margin(l, 1, num_groups=2, topk_groups=1)[0] == 1.5
    rng = np.random.default_rng(23)
    logits = rng.normal(size=(400, 16)).astype(np.float32)
    idx, _ = O.select_experts(logits, 4)
    m = O.selection_margin(logits, 4)
    noise = (rng.uniform(-1, 1, size=logits.shape) * (0.49 * m[:, None])).astype(np.float32)
    idx2, _ = O.select_experts((logits.astype(np.float64) + noise).astype(np.float32), 4)
    assert (np.sort(idx, 1) == np.sort(idx2, 1)).all()
    # closing the gap of one token flips its K-th choice
    t = int(np.argmin(m))
    order = np.argsort(-logits[t])
    bumped = logits.copy()
    bumped[t, order[4]] += np.float32(m[t] * 1.01)
    idx3, _ = O.select_experts(bumped, 4)
    assert set(idx3[t].tolist()) != set(idx[t].tolist())


def _reroute_in_epochs(topk_idx, keys, cand, capacity, nsegs):
    """The epoch structure the GPU assignment uses, restated on the host.

    Every excess slot first picks against the starting room (a token's slots
    in k order, each excluding the token's experts and its earlier picks).
    Then, per epoch: the first slot whose pick is the (room+1)-th pick of its
    expert among the uncommitted slots is found through per-expert counts by
    token segment (nsegs segments), then sub-ranges of that segment, then a
    scan of one sub-range; the picks before it are committed; the experts
    left without room drop out; the uncommitted slots that picked one of them
    pick again, in k order per token, with the token's later slots that now
    clash with a new pick.  Returns (topk_idx, epochs)."""
    KEPT, NONE = -2, -1
    idx = np.array(topk_idx, dtype=np.int64, copy=True).reshape(-1)
    S, K = np.asarray(topk_idx).shape
    E = keys.shape[1]
    key = np.where(cand, keys, -np.inf)
    counts = O.expert_counts(np.asarray(topk_idx), E)
    ros = O.expert_permutation(np.asarray(topk_idx), E, capacity)["row_of_slot"]
    room = capacity - np.minimum(counts, capacity)
    avail = room > 0

    def best(t, held):
        bv, be = -np.inf, NONE
        for e in range(E):
            if key[t, e] > bv and not held[e] and avail[e]:
                bv, be = key[t, e], e
        return be

    pick = np.full(S * K, KEPT)
    for t in range(S):
        held = np.zeros(E, bool)
        held[idx[t * K:(t + 1) * K]] = True
        for k in range(K):
            if ros[t * K + k] >= E * capacity:
                pick[t * K + k] = best(t, held)
                if pick[t * K + k] >= 0:
                    held[pick[t * K + k]] = True
    seg_len = -(-S // nsegs)
    seg_of = lambda s: (s // K) // seg_len
    seg_begin = lambda w: min(S, w * seg_len) * K
    cnt = np.zeros((nsegs, E), np.int64)
    for s in np.nonzero(pick >= 0)[0]:
        cnt[seg_of(s), pick[s]] += 1

    def first_over(counts_by_part, limit):  # part holding the (limit+1)-th pick, picks before it there
        acc = 0
        for w, c in enumerate(counts_by_part):
            if acc + c > limit:
                return w, limit - acc
            acc += c
        return len(counts_by_part), 0

    start, epochs = 0, 0
    for _ in range(E + 2):
        epochs += 1
        seg_e, need_e = np.full(E, nsegs), np.zeros(E, np.int64)
        for e in np.nonzero(avail)[0]:
            seg_e[e], need_e[e] = first_over(cnt[:, e], room[e])
        ms, P = int(seg_e.min()), S * K
        if ms < nsegs:
            a, b = max(seg_begin(ms), start), seg_begin(ms + 1)
            span = -(-(b - a) // nsegs)
            sub = np.zeros((nsegs, E), np.int64)
            for w in range(nsegs):
                lo = min(b, a + w * span)
                for s in range(lo, min(b, lo + span)):
                    if pick[s] >= 0 and seg_e[pick[s]] == ms:
                        sub[w, pick[s]] += 1
            sub_e, need2 = np.full(E, nsegs), np.zeros(E, np.int64)
            for e in np.nonzero(seg_e == ms)[0]:
                sub_e[e], need2[e] = first_over(sub[:, e], need_e[e])
            wm = int(sub_e.min())
            lo = min(b, a + wm * span)
            run, P = np.zeros(E, np.int64), None
            for s in range(lo, min(b, lo + span)):
                p = pick[s]
                if p >= 0 and seg_e[p] == ms and sub_e[p] == wm:
                    if run[p] == need2[p]:
                        P = s
                        break
                    run[p] += 1
            assert P is not None
        for s in range(start, P):
            if pick[s] >= 0:
                idx[s] = pick[s]
                room[pick[s]] -= 1
                cnt[seg_of(s), pick[s]] -= 1
        start = P
        if P >= S * K:
            break
        full = avail & (room <= 0)
        avail &= ~full
        done = set()
        for s in range(P, S * K):
            t = s // K
            if pick[s] < 0 or not full[pick[s]] or t in done:
                continue
            done.add(t)
            held = np.zeros(E, bool)
            held[idx[t * K:(t + 1) * K]] = True
            for k in range(max(P, t * K) - t * K, K):
                p = pick[t * K + k]
                if p >= 0 and (full[p] or held[p]):
                    q = best(t, held)
                    cnt[seg_of(t * K), p] -= 1
                    if q >= 0:
                        cnt[seg_of(t * K), q] += 1
                    pick[t * K + k] = p = q
                if p >= 0:
                    held[p] = True
    assert start >= S * K
    return idx.reshape(S, K).astype(np.int32), epochs


@pytest.mark.parametrize("nsegs", [1, 3, 16])
def test_reroute_epochs_equal_the_serial_assignment(nsegs):
    """The epoch structure reproduces reroute_over_capacity exactly, for any
    number of token segments, with ties in the keys, and with at most one
    epoch per expert that runs out of room, plus one."""
    rng = np.random.default_rng(24 + nsegs)
    for trial in range(12):
        S, E, K = int(rng.integers(20, 300)), int(rng.choice([4, 8, 16, 32])), int(rng.integers(1, 5))
        keys = (rng.normal(size=(S, E)) + 1.5 * rng.normal(size=E)[None, :]).astype(np.float32)
        if trial % 3 == 0:
            keys = np.round(keys).astype(np.float32)         # many equal keys
        cand = rng.random((S, E)) > 0.1
        idx, _ = O.select_experts(np.where(cand, keys, -np.inf).astype(np.float32), K)
        C = max(1, int(np.ceil(rng.uniform(0.7, 1.3) * S * K / E)))
        ref, _ = O.reroute_over_capacity(idx, keys, cand, C)
        got, epochs = _reroute_in_epochs(idx, keys, cand, C, nsegs)
        np.testing.assert_array_equal(got, ref)
        room = C - np.minimum(O.expert_counts(idx, E), C)
        filled = int(((room > 0) & (O.expert_counts(ref, E) >= C)).sum())
        assert epochs <= filled + 1, (epochs, filled)


def test_skew_recipe_gives_max_over_mean_near_four():
    """The skewed FP8 workload's router offsets (scale SKEW_OFFSET_SCALE, the
    value tests/golden/calibrate_skew.py finds) give a max/mean expert load of
    about 4 under the oracle's routing of the full-size inputs, drawn on the
    CPU (the top of the 3-5 range of jsqmd.com chapter 11, 11.2.3)."""
    import torch
    from mixture_experts_layer_bias_b200 import synthetic as syn
    cfg = syn.CONFIGS["fp8_skew_capacity"]
    x = syn.make_inputs(cfg, "cpu", seed=0, x_only=True)["x"].float().numpy()
    cpu = torch.device("cpu")
    w_r = syn._normal((cfg.E, cfg.d), 1.0 / cfg.d, syn._gen(cpu, 0, 2), cpu, torch.bfloat16).float().numpy()
    rb = syn.router_offsets(cfg, 0).numpy().astype(np.float64)
    logits = O.router_logits(x.astype(np.float64), w_r.astype(np.float64), rb)
    idx, _ = O.select_experts(logits, cfg.K)
    ratio = O.load_stats(O.expert_counts(idx, cfg.E), cfg.K, cfg.S)["max_over_mean"]
    assert 3.8 <= ratio <= 4.2, ratio
    # and the capacity of 1.25 S K / E really overflows on the hot experts
    assert cfg.capacity == syn.capacity_for(cfg.S, cfg.K, cfg.E) and ratio * cfg.S * cfg.K / cfg.E > cfg.capacity

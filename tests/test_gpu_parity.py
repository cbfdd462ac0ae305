"""Parity of every stage of the CUDA path with the CPU oracle, through the C ABI.

Routing indices, counts, offsets and the permutation are compared bit for bit
(on oracle-supplied float32 logits); float outputs within the contract's
tolerances: fp32 max-abs <= 1e-4 * max|ref|, bf16 relative L2 <= 1e-2, FP8
weights relative L2 <= 3e-2 against the oracle on the same decoded weights.
Sizes span several tiles and ragged tails.
"""

import dataclasses

import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

from parity import (BF16_REL_L2, F32_MAXABS_REL, FP8_REL_L2, OracleExperts, assert_status_clean, compare_layer,
                    ffn_case, max_abs_rel, new_ws, np64, rel_l2, run_layer, skewed_logits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ops.lib()
    torch.cuda.init()


def _route_gpu(desc_fields, logits, router_bias=None, sel_bias=None):
    desc = ops.make_desc(**desc_fields)
    ws = new_ws(desc)
    S, K = desc.num_tokens, desc.top_k
    tens = {}
    if router_bias is not None:
        tens["router_bias"] = torch.tensor(router_bias, dtype=torch.float32, device="cuda")
    if sel_bias is not None:
        tens["sel_bias"] = torch.tensor(sel_bias, dtype=torch.float32, device="cuda")
    w = ops.make_weights(tens)
    lg = torch.tensor(logits, dtype=torch.float32, device="cuda")
    idx = torch.full((S, K), -7, dtype=torch.int32, device="cuda")
    gw = torch.zeros((S, K), dtype=torch.float32, device="cuda")
    ops.moe_route(desc, w, None, lg, idx, gw, ws)
    torch.cuda.synchronize()
    code, flags, counters = ops.moe_get_status(ws)
    return idx.cpu().numpy(), gw.cpu().numpy().astype(np.float64), flags, counters


def _fields(S, E, K, **kw):
    f = dict(num_tokens=S, d_model=64, num_experts=E, top_k=K, d_ff=64)
    f.update(kw)
    return f


# ----------------------------------------------------------------------------
# routing: bit-exact indices on oracle logits
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("S,E,K,renorm", [(64, 8, 2, 1), (4096, 8, 2, 1), (300, 8, 2, 0), (1000, 64, 8, 1),
                                          (257, 256, 8, 1), (77, 5, 3, 1), (33, 32, 1, 1), (50, 40, 6, 0)])
def test_route_softmax_bit_exact(S, E, K, renorm):
    rng = np.random.default_rng(S * 7 + E)
    logits = skewed_logits(rng, S, E)
    logits[: S // 4] = np.round(logits[: S // 4] * 2) / 2  # ties
    rb = rng.normal(size=E).astype(np.float32) * 0.5
    idx, gw, flags, _ = _route_gpu(_fields(S, E, K, renormalize=renorm), logits, router_bias=rb)
    l_eff = np.add(logits, rb[None, :], dtype=np.float32)  # bias added to the logits in float32
    ridx, rw = O.select_experts(l_eff, K, "softmax", bool(renorm))
    np.testing.assert_array_equal(idx, ridx)
    assert max_abs_rel(gw, rw) <= F32_MAXABS_REL
    assert flags == 0


def test_route_nonfinite_logits_flagged_and_ranked_last():
    rng = np.random.default_rng(3)
    S, E, K = 40, 8, 2
    logits = rng.normal(size=(S, E)).astype(np.float32)
    logits[0, 3] = np.nan
    logits[1, :] = -np.inf
    logits[2, 5] = np.inf
    idx, gw, flags, counters = _route_gpu(_fields(S, E, K), logits)
    ridx, _ = O.select_experts(logits, K)
    np.testing.assert_array_equal(idx, ridx)
    assert flags & ops.MOE_STATUS_NONFINITE_LOGIT
    assert counters["nonfinite"] == 3


@pytest.mark.parametrize("E,G,TG,K", [(256, 8, 2, 8), (256, 16, 4, 8), (256, 4, 2, 8), (64, 8, 3, 6),
                                      (32, 4, 2, 4), (128, 2, 1, 8)])
def test_route_sigmoid_grouped_bit_exact(E, G, TG, K):
    rng = np.random.default_rng(E + G + TG)
    S = 700
    logits = rng.normal(size=(S, E)).astype(np.float32) * 2
    sb = (rng.normal(size=E) * 0.1).astype(np.float32)
    f = _fields(S, E, K, score_fn=1, num_groups=G, topk_groups=TG)
    idx, gw, flags, _ = _route_gpu(f, logits, sel_bias=sb)
    ridx, rw = O.select_experts(logits, K, "sigmoid", True, sb, G, TG)
    np.testing.assert_array_equal(idx, ridx)
    assert max_abs_rel(gw, rw) <= F32_MAXABS_REL
    # unnormalised gates are the sigmoid scores themselves
    f["renormalize"] = 0
    idx2, gw2, _, _ = _route_gpu(f, logits, sel_bias=sb)
    np.testing.assert_array_equal(idx2, ridx)
    np.testing.assert_array_equal(gw2.astype(np.float32), np.take_along_axis(O.sigmoid_f32(logits), ridx, 1))


def test_route_worked_example():
    """plumephp.com worked example: probabilities .55/.30/.08/.03 -> top-2
    {e0, e3} with gates .55/.85, .30/.85 (normalised) or .55, .30."""
    p = np.array([0.55, 0.01, 0.01, 0.30, 0.01, 0.08, 0.01, 0.03])
    logits = np.log(p).astype(np.float32)[None, :]
    idx, gw, _, _ = _route_gpu(_fields(1, 8, 2), logits)
    assert idx[0].tolist() == [0, 3]
    np.testing.assert_allclose(gw[0], [0.55 / 0.85, 0.30 / 0.85], rtol=1e-6)
    idx, gw, _, _ = _route_gpu(_fields(1, 8, 2, renormalize=0), logits)
    np.testing.assert_allclose(gw[0], [0.55, 0.30], rtol=1e-6)


@pytest.mark.parametrize("name,S,over", [("tiny_f32", 64, {}), ("mixtral_prefill", 512, {}),
                                         ("mixtral_prefill", 1500, {}), ("fp8_skew_capacity", 1024, {}),
                                         ("dsv3_grouped", 256, {}),
                                         ("dsv3_grouped", 1024, dict(E=32, num_groups=4, topk_groups=2)),
                                         ("mixtral_prefill", 1000, dict(d=520, E=6)),
                                         ("mixtral_prefill", 777, dict(d=1000, E=13, K=3)),
                                         ("mixtral_prefill", 2049, dict(d=264, E=32, K=4))])
def test_route_computed_logits_within_margin(name, S, over):
    """The router computes its own logits: a CTA per token (S <= 512), for
    S > 512, E <= 32 and W_r of at most 64 KB tensor-core products over 16
    tokens per CTA (bf16: the Mixtral-shaped case at S = 1500, and ragged
    cases with d not a multiple of 32, E not a multiple of 8 and S not a
    multiple of 16) or warps streaming token rows against W_r in shared memory
    (fp32), or the logits GEMM then the selection (E > 32, or a larger W_r:
    32 experts x 7168 here);
    indices must agree with the oracle wherever the selection margin is
    >= 1e-4 (excluded tokens are counted), and the gates within the fp32
    tolerance."""
    cfg = syn.scaled(syn.CONFIGS[name], S=S, **over)
    # routing only reads x and the router; small experts keep the draw cheap
    inp = syn.make_inputs(syn.scaled(cfg, h=8), "cuda", seed=1)
    desc = ops.make_desc(**syn.desc_dict(cfg, S))
    ws = new_ws(desc)
    idx = torch.empty((S, cfg.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, cfg.K), dtype=torch.float32, device="cuda")
    ops.moe_route(desc, ops.make_weights(inp), inp["x"], None, idx, gw, ws)
    torch.cuda.synchronize()
    from parity import oracle_routing
    _, ridx, rw, margin = oracle_routing(inp, cfg)
    keep = margin >= 1e-4
    assert keep.sum() >= 0.9 * S
    np.testing.assert_array_equal(idx.cpu().numpy()[keep], ridx[keep])
    # the gates are fp32 outputs: the fp32 contract, max-abs <= 1e-4 * max|ref|
    assert max_abs_rel(gw.cpu().numpy()[keep], rw[keep]) <= F32_MAXABS_REL
    print(f"{name}: excluded {int((~keep).sum())} of {S} tokens (margin < 1e-4)")


# ----------------------------------------------------------------------------
# histogram / scan / permutation: bit-exact
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("S,E,K,cap,dt", [(1, 8, 2, 0, 1), (5000, 8, 2, 0, 1), (3000, 64, 8, 0, 1),
                                          (777, 256, 8, 0, 1), (2000, 64, 8, -1, 1), (1000, 8, 3, 0, 0),
                                          (4099, 16, 5, -1, 0), (64, 8, 2, 0, 0), (2048, 8, 1, 9, 1)])
def test_permute_bit_exact(S, E, K, cap, dt):
    rng = np.random.default_rng(S + E + K)
    logits = skewed_logits(rng, S, E, spread=2.0)
    ridx, _ = O.select_experts(logits, K)
    if cap < 0:
        cap = syn.capacity_for(S, K, E)
    d = 64 if dt == 0 else 136  # 136: not a multiple of the 16-byte vector count per warp
    desc = ops.make_desc(num_tokens=S, d_model=d, num_experts=E, top_k=K, d_ff=64, capacity=cap, act_dtype=dt,
                         activation=0 if dt == 0 else 1, weight_dtype=0 if dt == 0 else 1)
    ws = new_ws(desc)
    R = ops.moe_routed_rows(desc)
    tdt = torch.float32 if dt == 0 else torch.bfloat16
    x = torch.randn((S, d), device="cuda").to(tdt)
    counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((2 * (E + 1),), -1, dtype=torch.int32, device="cuda")
    ros = torch.full((S * K,), -5, dtype=torch.int32, device="cuda")
    tor = torch.full((R,), -5, dtype=torch.int32, device="cuda")
    xp = torch.zeros((R, d), dtype=tdt, device="cuda")
    idx_t = torch.tensor(ridx, dtype=torch.int32, device="cuda")
    ops.moe_permute(desc, x, idx_t, counts, offsets, ros, tor, xp, ws)
    torch.cuda.synchronize()
    P = O.expert_permutation(ridx, E, cap)
    np.testing.assert_array_equal(counts.cpu().numpy(), P["counts"])
    np.testing.assert_array_equal(offsets.cpu().numpy()[: E + 1], P["offsets"])
    if cap:
        np.testing.assert_array_equal(offsets.cpu().numpy()[E + 1:], P["ovf_offsets"])
    np.testing.assert_array_equal(ros.cpu().numpy(), P["row_of_slot"])
    tor_np = tor.cpu().numpy()
    if cap:
        np.testing.assert_array_equal(tor_np, P["token_of_row"])
    else:
        np.testing.assert_array_equal(tor_np, P["token_of_row"])
    used = P["token_of_row"] >= 0
    # gathered rows are bit copies of the token rows
    assert torch.equal(xp[torch.tensor(np.nonzero(used)[0], device="cuda")],
                       x[torch.tensor(P["token_of_row"][used], device="cuda", dtype=torch.long)])
    counters = assert_status_clean(ws)
    if cap:
        assert counters["overflow_rows"] == int(P["ovf_counts"].sum())


def test_permute_bad_ids_flagged():
    S, E, K = 100, 8, 2
    rng = np.random.default_rng(0)
    ridx, _ = O.select_experts(rng.normal(size=(S, E)).astype(np.float32), K)
    ridx[5, 1] = 9
    ridx[7, 0] = -1
    desc = ops.make_desc(num_tokens=S, d_model=64, num_experts=E, top_k=K, d_ff=64)
    ws = new_ws(desc)
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    offsets = torch.empty((E + 1,), dtype=torch.int32, device="cuda")
    ros = torch.empty((S * K,), dtype=torch.int32, device="cuda")
    tor = torch.empty((S * K,), dtype=torch.int32, device="cuda")
    ops.moe_permute(desc, None, torch.tensor(ridx, device="cuda", dtype=torch.int32), counts, offsets, ros, tor,
                    None, ws)
    code, flags, counters = ops.moe_get_status(ws)
    assert code == ops.MOE_ERR_DEVICE_STATUS and flags & ops.MOE_STATUS_BAD_EXPERT_ID
    assert counters["bad_id"] == 2
    assert int(counts.sum()) == S * K - 2
    r = ros.cpu().numpy().reshape(S, K)
    assert r[5, 1] == -1 and r[7, 0] == -1


# ----------------------------------------------------------------------------
# combine
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("dt,shared,K,S", [(0, 0, 2, 333), (1, 0, 2, 333), (1, 1, 8, 333), (0, 1, 3, 333),
                                           (1, 1, 8, 5), (0, 0, 2, 1), (1, 0, 2, 256)])
def test_combine(dt, shared, K, S):
    E, d = 16, 264
    rng = np.random.default_rng(K + dt)
    ridx, rw = O.select_experts(rng.normal(size=(S, E)).astype(np.float32), K)
    P = O.expert_permutation(ridx, E)
    R = P["num_rows"]
    tdt = torch.float32 if dt == 0 else torch.bfloat16
    yp = torch.randn((R + shared * S, d), device="cuda").to(tdt)
    desc = ops.make_desc(num_tokens=S, d_model=d, num_experts=E, top_k=K, d_ff=64, num_shared=shared,
                         act_dtype=dt, activation=0 if dt == 0 else 1, weight_dtype=0 if dt == 0 else 1)
    ws = new_ws(desc)
    y = torch.empty((S, d), dtype=tdt, device="cuda")
    ops.moe_combine(desc, yp, torch.tensor(P["row_of_slot"], device="cuda"),
                    torch.tensor(rw, dtype=torch.float32, device="cuda"), y, ws)
    torch.cuda.synchronize()
    ypn = np64(yp)
    ref = O.combine(ypn[:R], P["row_of_slot"], rw.astype(np.float32), ypn[R:] if shared else None)
    if dt == 0:
        assert max_abs_rel(np64(y), ref) <= F32_MAXABS_REL
    else:
        assert rel_l2(np64(y), ref) <= BF16_REL_L2 / 4


# ----------------------------------------------------------------------------
# grouped expert FFN
# ----------------------------------------------------------------------------


_ffn_case = ffn_case


def test_grouped_ffn_f32_tiny():
    got, ref = _ffn_case(syn.CONFIGS["tiny_f32"])
    assert max_abs_rel(got, ref) <= F32_MAXABS_REL


@pytest.mark.parametrize("S,d,h,E,K,extra", [
    (300, 256, 384, 8, 2, {}),            # several m-blocks, partial tiles
    (200, 320, 200, 8, 2, {}),            # N and K tails in both projections
    (1, 512, 256, 8, 2, {}),              # a single token
    (513, 384, 256, 16, 4, {"num_shared": 1}),
    (700, 256, 128, 64, 8, {"capacity": -1}),
    (600, 256, 128, 256, 8, {"capacity": -1, "num_shared": 1}),  # 2 x 256 + 1 groups in one launch
])
def test_grouped_ffn_bf16_swiglu(S, d, h, E, K, extra):
    extra = dict(extra)
    cap = extra.pop("capacity", 0)
    cfg = syn.LayerConfig("t", S=S, d=d, E=E, K=K, h=h, router_offset_var=1.0, **extra)
    if cap:
        cfg = syn.scaled(cfg, capacity=syn.capacity_for(S, K, E))
    got, ref = _ffn_case(cfg)
    assert rel_l2(got, ref) <= BF16_REL_L2


@pytest.mark.parametrize("S,d,h,E,K", [(400, 256, 384, 8, 2), (600, 512, 176, 16, 4),
                                       (300, 96, 192, 8, 2)])   # d < 128: decoded by a pass, not in the GEMM
def test_grouped_ffn_fp8_weights(S, d, h, E, K):
    cfg = syn.LayerConfig("t", S=S, d=d, E=E, K=K, h=h, weight_dtype=syn.E4M3, router_offset_var=1.0,
                          capacity=syn.capacity_for(S, K, E))
    got, ref = _ffn_case(cfg)
    assert rel_l2(got, ref) <= FP8_REL_L2


@pytest.mark.parametrize("S,d,h,E,K,extra", [
    (2, 2048, 1024, 8, 2, {}),                                   # few tiles, long K: split-K on both GEMMs
    (3, 1024, 2048, 8, 2, {"activation": syn.GELU}),              # GeLU + bias applied after the split sum
    (4, 2048, 1408, 8, 2, {"weight_dtype": syn.E4M3}),            # FP8 scales applied after the split sum
    (5, 1024, 512, 16, 4, {"num_shared": 1}),                     # shared expert group in the split GEMMs
    (128, 4096, 1024, 8, 2, {}),                                  # decode-sized batch, full model width
])
def test_grouped_ffn_split_k(S, d, h, E, K, extra):
    cfg = syn.LayerConfig("t", S=S, d=d, E=E, K=K, h=h, router_offset_var=0.5, **extra)
    got, ref = _ffn_case(cfg)
    lim = FP8_REL_L2 if cfg.weight_dtype == syn.E4M3 else BF16_REL_L2
    assert rel_l2(got, ref) <= lim


def test_grouped_ffn_bf16_gelu_bias():
    cfg = syn.LayerConfig("t", S=150, d=256, E=8, K=2, h=256, activation=syn.GELU)
    got, ref = _ffn_case(cfg)
    assert rel_l2(got, ref) <= BF16_REL_L2


# ----------------------------------------------------------------------------
# the whole layer
# ----------------------------------------------------------------------------


def test_layer_tiny_f32_full_size():
    cfg = syn.CONFIGS["tiny_f32"]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    gpu = run_layer(inp, cfg)
    rep = compare_layer(gpu, inp, cfg)
    assert rep["ok"], rep
    assert_status_clean(gpu["ws"])


@pytest.mark.parametrize("name,over", [
    ("mixtral_prefill", dict(S=384, d=512, h=768)),
    ("mixtral_decode", dict(S=8, d=512, h=768)),
    ("dsv3_grouped", dict(S=256, d=512, h=256)),
    ("fp8_skew_capacity", dict(S=1024, d=256, h=384)),
])
def test_layer_scaled_down(name, over):
    cfg = syn.scaled(syn.CONFIGS[name], **over)
    inp = syn.make_inputs(cfg, "cuda", seed=2)
    gpu = run_layer(inp, cfg)
    rep = compare_layer(gpu, inp, cfg)
    print(name, rep)
    assert rep["ok"], rep
    # the histogram output agrees with the GPU's own routing
    idx = gpu["idx"].cpu().numpy()
    np.testing.assert_array_equal(gpu["counts"].cpu().numpy(), O.expert_counts(idx, cfg.E))


def test_layer_dense_cross_check_tiny():
    """Sparse output equals every expert on every token, masked by TopK."""
    cfg = syn.CONFIGS["tiny_f32"]
    inp = syn.make_inputs(cfg, "cuda", seed=5)
    gpu = run_layer(inp, cfg)
    from parity import oracle_routing
    x, ridx, rw, margin = oracle_routing(inp, cfg)
    fn = OracleExperts(inp, cfg)
    dense = O.moe_layer_dense(x, ridx, rw, fn, cfg.E)
    keep = margin >= 1e-4
    assert max_abs_rel(np64(gpu["y"])[keep], dense[keep]) <= F32_MAXABS_REL


@pytest.mark.parametrize("tau", [1.0, 2.0, 0.5, 0.7])
def test_soft_routing_with_temperature(tau):
    """Soft routing (jsqmd.com chapter 11, 11.3.3): y = sum_i softmax(s/tau)_i
    E_i(x) over all experts.  The layer with K = E, renormalised gates and
    desc.temperature = tau computes it from the unscaled router weights."""
    cfg = dataclasses.replace(syn.scaled(syn.CONFIGS["tiny_f32"], K=8), temperature=tau)
    inp = syn.make_inputs(cfg, "cuda", seed=4)
    gpu = run_layer(inp, cfg)
    x = np64(inp["x"])
    logits = O.router_logits(x, np64(inp["w_router"]))
    fn = OracleExperts(inp, cfg)
    ref = O.soft_routing(x, logits, fn, cfg.E, tau)
    assert max_abs_rel(np64(gpu["y"]), ref) <= F32_MAXABS_REL
    # the gates: every expert's softmax(l / tau) probability in the slot order
    p = torch.softmax(torch.tensor(logits, dtype=torch.float64) / tau, dim=1).numpy()
    idx = gpu["idx"].cpu().numpy()
    assert max_abs_rel(gpu["w"].cpu().numpy(), np.take_along_axis(p, idx, 1)) <= F32_MAXABS_REL


@pytest.mark.parametrize("tau", [0.5, 0.7, 2.0])
def test_route_temperature_bit_exact_on_oracle_logits(tau):
    """Top-8 of 64 with a temperature on oracle logits: indices bit-exact
    (keys l / tau in float32 on both sides), gates within the fp32 bar."""
    rng = np.random.default_rng(int(tau * 10))
    S, E, K = 2000, 64, 8
    logits = skewed_logits(rng, S, E, spread=2.0)
    idx, gw, flags, _ = _route_gpu(_fields(S, E, K, temperature=tau), logits)
    ridx, rw = O.select_experts(logits, K, temperature=tau)
    np.testing.assert_array_equal(idx, ridx)
    assert max_abs_rel(gw, rw) <= F32_MAXABS_REL
    assert flags == 0

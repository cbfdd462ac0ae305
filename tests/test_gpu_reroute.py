"""Over-capacity re-routing (jsqmd.com chapter 11, 11.3.3) against the oracle.

The re-routed indices are compared bit for bit on oracle-supplied float32
logits (the keys are then the same bits on both sides), the recomputed gates
within 1e-5 of the largest gate, the counters exactly; the layer output
within the FP8 tolerance, computed the same way.  moe_layer_forward must give
the same bits as the stage calls it chains.
"""
import gc

import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

from parity import (FP8_REL_L2, SCORE, OracleExperts, assert_status_clean, new_ws, np64, oracle_reroute, rel_l2,
                    run_layer)

pytestmark = pytest.mark.gpu


def _bufs(cfg, desc):
    S, E, K = cfg.S, cfg.E, cfg.K
    R = ops.moe_routed_rows(desc)
    dev = "cuda"
    return dict(idx=torch.empty((S, K), dtype=torch.int32, device=dev),
                gw=torch.empty((S, K), dtype=torch.float32, device=dev),
                counts=torch.empty((E,), dtype=torch.int32, device=dev),
                offsets=torch.empty((2 * (E + 1),), dtype=torch.int32, device=dev),
                ros=torch.empty((S * K,), dtype=torch.int32, device=dev),
                tor=torch.empty((R,), dtype=torch.int32, device=dev))


def _route_reroute(cfg, logits, sel_bias=None, router_bias=None):
    """moe_route on the given float32 logits, capacity ranks, moe_reroute.
    Returns the buffers, the workspace and the descriptor."""
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    b = _bufs(cfg, desc)
    w = ops.MoeWeights()
    w.sel_bias = None if sel_bias is None else sel_bias.data_ptr()
    w.router_bias = None if router_bias is None else router_bias.data_ptr()
    ops.moe_route(desc, w, None, torch.tensor(logits, device="cuda"), b["idx"], b["gw"], ws)
    first = b["idx"].clone()
    ops.moe_permute(desc, None, b["idx"], b["counts"], b["offsets"], b["ros"], b["tor"], None, ws)
    ops.moe_reroute(desc, b["idx"], b["gw"], b["counts"], b["ros"], ws)
    torch.cuda.synchronize()
    return b, ws, desc, first


CASES = [
    # S, E, K, capacity factor, score, groups, sel_bias var
    (2048, 64, 8, 1.25, syn.SOFTMAX, (1, 1), 0.0),   # the skewed FP8 layer's shape of routing
    (1000, 16, 4, 1.1, syn.SIGMOID, (4, 2), 0.01),   # sigmoid keys with bias, group-limited candidates
    (700, 8, 2, 0.8, syn.SOFTMAX, (1, 1), 0.0),      # total room below the excess: some slots stay
    (3000, 256, 8, 1.0, syn.SIGMOID, (8, 2), 0.01),  # 256 experts (the key rows span 8 registers)
]


@pytest.mark.parametrize("S,E,K,factor,score,groups,sbv", CASES)
def test_reroute_bit_exact_on_oracle_logits(S, E, K, factor, score, groups, sbv):
    rng = np.random.default_rng(S + E)
    logits = (rng.normal(size=(S, E)) + 1.2 * rng.normal(size=E)[None, :]).astype(np.float32)
    C = syn.capacity_for(S, K, E, factor)
    cfg = syn.LayerConfig("t", S=S, d=64, E=E, K=K, h=64, score_fn=score, num_groups=groups[0],
                          topk_groups=groups[1], capacity=C, reroute=1)
    sb = None
    if sbv > 0:
        sb = (rng.normal(size=E) * np.sqrt(sbv)).astype(np.float32)
    b, ws, desc, first = _route_reroute(cfg, logits, None if sb is None else torch.tensor(sb, device="cuda"))
    idx0, _ = O.select_experts(logits, K, SCORE[score], True, sb, groups[0], groups[1])
    np.testing.assert_array_equal(first.cpu().numpy(), idx0)
    ref_idx, ref_w = oracle_reroute(logits, idx0, cfg, sb)
    got_idx = b["idx"].cpu().numpy()
    np.testing.assert_array_equal(got_idx, ref_idx)
    np.testing.assert_allclose(b["gw"].cpu().numpy(), ref_w, rtol=0, atol=1e-5 * np.abs(ref_w).max())
    moved = int((got_idx != idx0).sum())
    code, flags, counters = ops.moe_get_status(ws)
    assert flags == 0 and counters["rerouted"] == moved
    # the second permutation: counts of the final choices; only slots without room overflow
    ops.moe_permute(desc, None, b["idx"], b["counts"], b["offsets"], b["ros"], b["tor"], None, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(b["counts"].cpu().numpy(), O.expert_counts(ref_idx, E))
    P = O.expert_permutation(ref_idx, E, C)
    np.testing.assert_array_equal(b["ros"].cpu().numpy(), P["row_of_slot"])
    if factor >= 1.0:
        assert moved > 0
    print(S, E, K, C, "moved", moved, "still over capacity", int(P["ovf_counts"].sum()))


def test_reroute_nothing_to_move():
    """Capacity above every count: the indices and gates are left as routed."""
    S, E, K = 500, 8, 2
    rng = np.random.default_rng(3)
    logits = rng.normal(size=(S, E)).astype(np.float32)
    cfg = syn.LayerConfig("t", S=S, d=64, E=E, K=K, h=64, capacity=S, reroute=1)
    b, ws, desc, first = _route_reroute(cfg, logits)
    assert torch.equal(first, b["idx"])
    assert ops.moe_get_status(ws)[2]["rerouted"] == 0


def _staged_layer(cfg, inp, logits=None):
    """route (oracle logits if given) -> permute (ranks) -> reroute ->
    permute -> grouped FFN -> combine."""
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    b = _bufs(cfg, desc)
    S, d = cfg.S, cfg.d
    R = ops.moe_routed_rows(desc)
    w = ops.make_weights(inp)
    xp = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    yp = torch.empty((R + cfg.num_shared * S, d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    lg = None if logits is None else torch.tensor(logits, device="cuda")
    ops.moe_route(desc, w, inp["x"], lg, b["idx"], b["gw"], ws)
    ops.moe_permute(desc, None, b["idx"], b["counts"], b["offsets"], b["ros"], b["tor"], None, ws)
    ops.moe_reroute(desc, b["idx"], b["gw"], b["counts"], b["ros"], ws)
    ops.moe_permute(desc, inp["x"], b["idx"], b["counts"], b["offsets"], b["ros"], b["tor"], xp, ws)
    ops.moe_grouped_ffn(desc, w, xp, b["offsets"], inp["x"], yp, ws)
    ops.moe_combine(desc, yp, b["ros"], b["gw"], y, ws)
    torch.cuda.synchronize()
    assert_status_clean(ws)
    return y, b


def _oracle_layer_on_logits(cfg, inp, logits, tokens):
    x = np64(inp["x"])
    idx0, _ = O.select_experts(logits, cfg.K, SCORE[cfg.score_fn], bool(cfg.renormalize))
    idx, w = oracle_reroute(logits, idx0, cfg)
    fn = OracleExperts(inp, cfg)
    return O.moe_layer(x[tokens], idx[tokens], w[tokens], fn, cfg.E), idx


def _oracle_logits(inp):
    x = np64(inp["x"])
    rb = None if inp.get("router_bias") is None else np64(inp["router_bias"])
    logits = O.router_logits(x, np64(inp["w_router"]), rb)
    return logits


@pytest.mark.parametrize("over", [dict(S=1024, d=256, h=384), dict(S=2000, d=128, h=256, K=4, E=16)])
def test_layer_with_reroute_scaled(over):
    cfg = syn.scaled(syn.VARIANTS["fp8_skew_capacity_reroute"], **over)
    inp = syn.make_inputs(cfg, "cuda", seed=7)
    logits = _oracle_logits(inp)
    # the bias is already inside the oracle logits: route on them without it
    inp_nb = dict(inp)
    inp_nb["router_bias"] = None
    y, b = _staged_layer(cfg, inp_nb, logits)
    tokens = np.arange(cfg.S)
    ref, ref_idx = _oracle_layer_on_logits(cfg, inp_nb, logits, tokens)
    np.testing.assert_array_equal(b["idx"].cpu().numpy(), ref_idx)
    err = rel_l2(np64(y), ref)
    print(over, "rel_l2", err)
    assert err <= FP8_REL_L2


@pytest.mark.parametrize("over", [dict(S=1024, d=256, h=384), dict(S=300, d=128, h=128, E=8, K=2)])
def test_layer_forward_equals_stage_calls(over):
    """moe_layer_forward chains route -> permute -> reroute -> permute -> FFN
    -> combine itself: the same bits as the stage calls."""
    cfg = syn.scaled(syn.VARIANTS["fp8_skew_capacity_reroute"], **over)
    inp = syn.make_inputs(cfg, "cuda", seed=8)
    fused = run_layer(inp, cfg)
    y, b = _staged_layer(cfg, inp)
    assert torch.equal(fused["idx"], b["idx"])
    assert torch.equal(fused["y"].view(torch.int16), y.view(torch.int16))
    code, flags, counters = ops.moe_get_status(fused["ws"])
    assert flags == 0 and counters["rerouted"] > 0


def test_reroute_full_size():
    """The skewed FP8 layer with re-routing at full size: routing bit-exact on
    oracle logits, outputs on sampled tokens (every expert, moved slots)."""
    cfg = syn.VARIANTS["fp8_skew_capacity_reroute"]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    logits = _oracle_logits(inp)
    inp_nb = dict(inp)
    inp_nb["router_bias"] = None
    y, b = _staged_layer(cfg, inp_nb, logits)
    idx0, _ = O.select_experts(logits, cfg.K, "softmax", True)
    rng = np.random.default_rng(0)
    got = b["idx"].cpu().numpy()
    moved_tok = np.nonzero((got != idx0).any(axis=1))[0]
    assert len(moved_tok) > 0
    toks = np.unique(np.concatenate([rng.choice(cfg.S, 24, replace=False), moved_tok[:16]]))
    ref, ref_idx = _oracle_layer_on_logits(cfg, inp_nb, logits, toks)
    np.testing.assert_array_equal(got, ref_idx)
    err = rel_l2(np64(y)[toks], ref)
    print("full size: moved slots", int((got != idx0).sum()), "rel_l2", err)
    assert err <= FP8_REL_L2
    del inp, inp_nb
    gc.collect()
    torch.cuda.empty_cache()

"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (moe_layer_forward / the four stage calls on one stream).

Every token's routing and the whole permutation are checked bit for bit
(oracle logits fed through moe_route's logits input; the oracle's indices fed
to moe_permute); layer outputs are checked on a sample of at least 1024 tokens the oracle
computes one by one, chosen to cover every expert that receives tokens (and
tokens with overflow rows for the capacity-bounded workload), with tokens whose
selection margin is below 1e-4 excluded and counted.
"""
import gc

import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

from parity import SCORE, compare_layer, new_ws, np64, oracle_routing, run_layer

pytestmark = pytest.mark.gpu


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _sample_tokens(idx_ref, E, n_random, rng, extra=()):
    """Random tokens plus, for every expert with tokens, one token routed to
    it."""
    S = idx_ref.shape[0]
    toks = set(rng.choice(S, size=min(n_random, S), replace=False).tolist())
    for e in range(E):
        hit = np.nonzero((idx_ref == e).any(axis=1))[0]
        if len(hit) and not toks.intersection(hit.tolist()):
            toks.add(int(hit[0]))
    toks.update(int(t) for t in extra)
    return np.array(sorted(toks))


def _routing_bit_exact(inp, cfg, S=None):
    """moe_route on the oracle's float32 logits (router bias added in float32
    by both sides) reproduces the oracle's indices for every token."""
    S = cfg.S if S is None else S
    x = np64(inp["x"])
    logits = O.router_logits(x, np64(inp["w_router"]))
    rb = inp.get("router_bias")
    l_eff = logits if rb is None else np.add(logits, rb.cpu().numpy().astype(np.float32)[None, :],
                                             dtype=np.float32)
    sb = None if inp.get("sel_bias") is None else inp["sel_bias"].cpu().numpy().astype(np.float32)
    ridx, rw = O.select_experts(l_eff, cfg.K, SCORE[cfg.score_fn], bool(cfg.renormalize), sb, cfg.num_groups,
                                cfg.topk_groups)
    desc = ops.make_desc(**syn.desc_dict(cfg, S))
    ws = new_ws(desc)
    idx = torch.empty((S, cfg.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, cfg.K), dtype=torch.float32, device="cuda")
    ops.moe_route(desc, ops.make_weights(inp), None, torch.tensor(logits, device="cuda"), idx, gw, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(gw.cpu().numpy(), rw, rtol=0, atol=1e-4 * np.abs(rw).max())
    return ridx


def _permute_bit_exact(cfg, ridx):
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    R = ops.moe_routed_rows(desc)
    E, S, K = cfg.E, cfg.S, cfg.K
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    offsets = torch.empty((2 * (E + 1),), dtype=torch.int32, device="cuda")
    ros = torch.empty((S * K,), dtype=torch.int32, device="cuda")
    tor = torch.empty((R,), dtype=torch.int32, device="cuda")
    ops.moe_permute(desc, None, torch.tensor(ridx, device="cuda", dtype=torch.int32), counts, offsets, ros, tor,
                    None, ws)
    torch.cuda.synchronize()
    P = O.expert_permutation(ridx, E, cfg.capacity)
    np.testing.assert_array_equal(counts.cpu().numpy(), P["counts"])
    np.testing.assert_array_equal(offsets.cpu().numpy()[: E + 1], P["offsets"])
    if cfg.capacity:
        np.testing.assert_array_equal(offsets.cpu().numpy()[E + 1:], P["ovf_offsets"])
    np.testing.assert_array_equal(ros.cpu().numpy(), P["row_of_slot"])
    np.testing.assert_array_equal(tor.cpu().numpy(), P["token_of_row"])
    return P


def _check_layer(cfg, inp, n_random=48, extra=(), seed=0):
    gpu = run_layer(inp, cfg)
    code, flags, counters = ops.moe_get_status(gpu["ws"])
    assert flags == 0, (flags, counters)
    _, ridx_full, _, _ = oracle_routing(inp, cfg)
    toks = _sample_tokens(ridx_full, cfg.E, n_random, np.random.default_rng(seed), extra)
    rep = compare_layer(gpu, inp, cfg, toks)
    # the load report computed on the device from the layer's counts
    counts = gpu["counts"].cpu().numpy()
    stats = torch.full((ops.MOE_NUM_LOAD_STATS,), -1.0, dtype=torch.float64, device="cuda")
    ops.moe_load_stats(gpu["desc"], gpu["counts"], stats)
    got = dict(zip(ops.LOAD_STAT_NAMES, stats.cpu().tolist()))
    ref = O.load_stats(counts, cfg.K, cfg.S, cfg.capacity)
    for k in ops.LOAD_STAT_NAMES:
        assert got[k] == pytest.approx(ref[k], rel=1e-12, abs=1e-9), (k, got, ref)
    assert got["dropped"] == 0.0
    rep["max_over_mean"] = got["max_over_mean"]
    rep["load_std"] = got["std"]
    rep["overflow_rows"] = counters["overflow_rows"]
    if cfg.capacity and not cfg.reroute:
        assert got["overflow_rows"] == counters["overflow_rows"]
    print(cfg.name, rep)
    assert rep["ok"], rep
    return gpu, rep


def test_mixtral_prefill_full_size():
    cfg = syn.CONFIGS["mixtral_prefill"]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    ridx = _routing_bit_exact(inp, cfg)
    _permute_bit_exact(cfg, ridx)
    _check_layer(cfg, inp, n_random=1024)
    del inp
    _free()


def test_mixtral_decode_sweep_full_weights():
    base = syn.CONFIGS["mixtral_decode"]
    weights = syn.make_inputs(syn.scaled(base, S=1), "cuda", seed=0)
    for S in syn.DECODE_SIZES:
        cfg = syn.scaled(base, S=S)
        inp = dict(weights)
        inp["x"] = syn.make_inputs(cfg, "cuda", seed=S, x_only=True)["x"]
        _routing_bit_exact(inp, cfg)
        gpu = run_layer(inp, cfg)
        rep = compare_layer(gpu, inp, cfg)  # every token
        print(cfg.name, S, rep)
        assert rep["ok"], rep
    del weights
    _free()


def test_mixtral_decode_e4m3_weights_full_size():
    """The decode sizes on the Mixtral-shaped weights stored as E4M3 with
    per-channel scales and bf16 activations: the GEMMs multiply the weight
    codes by two-term codes of the activations (both terms in one MMA, in
    64-row m-blocks at S = 128).  Every token against the oracle (FP8
    tolerance)."""
    base = syn.VARIANTS["mixtral_decode_e4m3"]
    weights = syn.make_inputs(syn.scaled(base, S=1), "cuda", seed=0)
    for S in (1, 8, 32, 128):
        cfg = syn.scaled(base, S=S)
        inp = dict(weights)
        inp["x"] = syn.make_inputs(cfg, "cuda", seed=S, x_only=True)["x"]
        gpu = run_layer(inp, cfg)
        code, flags, counters = ops.moe_get_status(gpu["ws"])
        assert flags == 0, (flags, counters)
        rep = compare_layer(gpu, inp, cfg)
        print(cfg.name, S, rep)
        assert rep["ok"], rep
    del weights
    _free()


def test_dsv3_grouped_full_size():
    cfg = syn.CONFIGS["dsv3_grouped"]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    ridx = _routing_bit_exact(inp, cfg)
    # every chosen expert lies in one of the two chosen groups
    groups = ridx // (cfg.E // cfg.num_groups)
    assert all(len(set(r.tolist())) <= cfg.topk_groups for r in groups)
    _permute_bit_exact(cfg, ridx)
    _check_layer(cfg, inp, n_random=1024)
    del inp
    _free()


def test_fp8_skew_capacity_full_size():
    cfg = syn.CONFIGS["fp8_skew_capacity"]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    ridx = _routing_bit_exact(inp, cfg)
    P = _permute_bit_exact(cfg, ridx)
    assert P["ovf_counts"].sum() > 0  # the skew really overflows the capacity
    # a few tokens whose slots land in the overflow region
    ovf_slots = np.nonzero(P["row_of_slot"] >= cfg.E * cfg.capacity)[0]
    extra = np.unique(ovf_slots // cfg.K)[:64]
    gpu, rep = _check_layer(cfg, inp, n_random=1024, extra=extra)
    assert rep["overflow_rows"] == int(P["ovf_counts"].sum())
    assert 3.5 <= rep["max_over_mean"] <= 4.5
    del inp
    _free()


def test_tiny_f32_capacity_equals_unbounded():
    """Capacity changes the layout only: outputs with and without it agree."""
    cfg = syn.CONFIGS["tiny_f32"]
    inp = syn.make_inputs(cfg, "cuda", seed=3)
    inp["router_bias"] = torch.tensor([2.0, 0, 0, 0, 0, 0, 0, -1.0], device="cuda")
    a = run_layer(inp, cfg)["y"]
    b = run_layer(inp, syn.scaled(cfg, capacity=5))["y"]
    assert torch.allclose(a, b, rtol=0, atol=1e-6 * float(a.abs().max()))

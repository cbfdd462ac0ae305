"""Decode-sized layer calls (S <= 16 tokens): the layer call must give
exactly the outputs of the separate stage calls (moe_route -> moe_permute ->
moe_grouped_ffn -> moe_combine), match the oracle within the contract's
tolerances, repeat bit-identically, and let one workspace serve several batch
sizes.
"""
import dataclasses

import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn

from parity import assert_status_clean, compare_layer, new_ws, run_layer

pytestmark = pytest.mark.gpu


def _stages(inp, cfg, S):
    desc = ops.make_desc(**syn.desc_dict(cfg, S))
    ws = new_ws(desc)
    w = ops.make_weights(inp)
    R = ops.moe_routed_rows(desc)
    adt = torch.float32 if cfg.act_dtype == syn.F32 else torch.bfloat16
    idx = torch.empty((S, cfg.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, cfg.K), dtype=torch.float32, device="cuda")
    counts = torch.empty((cfg.E,), dtype=torch.int32, device="cuda")
    offsets = torch.empty((2 * (cfg.E + 1),), dtype=torch.int32, device="cuda")
    ros = torch.empty((S * cfg.K,), dtype=torch.int32, device="cuda")
    tor = torch.empty((R,), dtype=torch.int32, device="cuda")
    xp = torch.zeros((R, cfg.d), dtype=adt, device="cuda")
    yp = torch.zeros((R + cfg.num_shared * S, cfg.d), dtype=adt, device="cuda")
    y = torch.empty((S, cfg.d), dtype=adt, device="cuda")
    ops.moe_route(desc, w, inp["x"], None, idx, gw, ws)
    ops.moe_permute(desc, inp["x"], idx, counts, offsets, ros, tor, xp, ws)
    ops.moe_grouped_ffn(desc, w, xp, offsets, inp["x"], yp, ws)
    ops.moe_combine(desc, yp, ros, gw, y, ws)
    torch.cuda.synchronize()
    assert_status_clean(ws)
    return dict(idx=idx, w=gw, counts=counts, y=y)


CASES = [
    ("mixtral_decode", dict(S=1, d=1024, h=1024)),
    ("mixtral_decode", dict(S=5, d=1024, h=512)),
    ("mixtral_decode", dict(S=16, d=512, h=512)),
    ("tiny_f32", dict(S=3)),
    ("tiny_f32", dict(S=16, E=32, K=4)),
    ("mixtral_decode", dict(S=7, d=512, h=512, E=32, K=4, capacity=1)),   # capacity with overflow rows
    ("mixtral_prefill_w8a8", dict(S=9, d=512, h=512)),                  # quantising gather
    ("mixtral_decode", dict(S=120, d=512, h=512, E=2, K=2)),            # groups of 120 rows: two 64-row blocks
    ("mixtral_decode_e4m3", dict(S=120, d=512, h=512, E=2, K=2)),       # the same, both E4M3 terms in one MMA
    ("mixtral_prefill_w8a8", dict(S=120, d=512, h=512, E=2, K=2)),      # the same with one E4M3 term
]


@pytest.mark.parametrize("name,kw", CASES)
def test_small_layer_equals_stage_calls_and_oracle(name, kw):
    base = syn.CONFIGS.get(name) or syn.VARIANTS[name]
    cfg = syn.scaled(base, **kw)
    inp = syn.make_inputs(cfg, "cuda", seed=11)
    if cfg.router_offset_var:
        inp["router_bias"] = syn.router_offsets(cfg, seed=0).to("cuda")
    gpu = run_layer(inp, cfg)
    code, flags, counters = ops.moe_get_status(gpu["ws"])
    assert flags == 0, (flags, counters)
    ref = _stages(inp, cfg, cfg.S)
    assert torch.equal(gpu["idx"], ref["idx"])
    assert torch.equal(gpu["w"], ref["w"])
    assert torch.equal(gpu["counts"], ref["counts"])
    assert torch.equal(gpu["y"], ref["y"])
    rep = compare_layer(gpu, inp, cfg)
    print(name, kw, rep)
    assert rep["ok"], rep
    if cfg.capacity:
        assert counters["overflow_rows"] == int(np.maximum(ref["counts"].cpu().numpy() - cfg.capacity, 0).sum())


def test_small_layer_repeats_bit_identically():
    """Repeated layer calls on one workspace give the same bits (split-K
    slices are summed in a fixed order)."""
    cfg = syn.scaled(syn.CONFIGS["mixtral_decode"], S=2, d=1024, h=2048)
    inp = syn.make_inputs(cfg, "cuda", seed=12)
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    w = ops.make_weights(inp)
    ys = []
    for _ in range(3):
        y = torch.empty((cfg.S, cfg.d), dtype=torch.bfloat16, device="cuda")
        ops.moe_layer_forward(desc, w, inp["x"], y, None, None, None, ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    assert_status_clean(ws)


def test_one_workspace_serves_several_batch_sizes():
    """A workspace sized for the largest batch serves smaller ones."""
    base = syn.scaled(syn.CONFIGS["mixtral_decode"], d=1024, h=2048)
    inp = syn.make_inputs(syn.scaled(base, S=128), "cuda", seed=13)
    big = ops.make_desc(**syn.desc_dict(base, 128))
    ws = new_ws(big)
    w = ops.make_weights(inp)
    for S in (128, 1, 32, 8, 128, 3):
        desc = ops.make_desc(**syn.desc_dict(base, S))
        y = torch.empty((S, base.d), dtype=torch.bfloat16, device="cuda")
        ops.moe_layer_forward(desc, w, inp["x"][:S], y, None, None, None, ws)
        sub = dict(inp)
        sub["x"] = inp["x"][:S]
        ref = run_layer(sub, dataclasses.replace(base, S=S))["y"]
        torch.cuda.synchronize()
        assert torch.equal(y, ref), S
    assert_status_clean(ws)

"""W8A8 path: per-row E4M3 activation quantisation and the expert GEMMs on
8-bit operands (kind::f8f6f4), against the oracle.

The quantiser is compared bit for bit (codes and scales) with the oracle's
``quantize_rows_e4m3``; the FFN and the layer are compared with the oracle's
``expert_swiglu_w8a8``, which quantises the same rows the same way, within
the FP8 tolerance (relative L2 <= 3e-2).
"""
import gc

import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

from parity import FP8_REL_L2, assert_status_clean, compare_layer, ffn_case, oracle_routing, rel_l2, run_layer

pytestmark = pytest.mark.gpu


def _quant_rows(x_bf16: torch.Tensor):
    rows, d = x_bf16.shape
    q = torch.empty((rows, d), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows,), dtype=torch.float32, device="cuda")
    ops.moe_quantize_rows_e4m3(x_bf16, q, s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def _rows_with_edge_cases(rows, d, seed):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(rows, d)) * (10.0 ** rng.uniform(-3, 3, size=(rows, 1)))
    x[0] = 0.0                          # all zero: scale 1, codes 0
    x[1, 5] = np.nan                    # a NaN: scale 1, that code 0x7F
    x[2, 7] = np.inf                    # an infinity: scale inf
    x[3] = rng.normal(size=d) * 1e-38   # scale below the float32 normal range
    x[4] = rng.normal(size=d) * 1e38    # near the bf16 maximum
    x[5, ::3] = -x[5, ::3]
    x[6] = 0.0
    x[6, d - 1] = -2.0                  # one value, in the row's last column
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("rows,d", [(1, 16), (37, 1040), (300, 4096), (9, 7168), (2050, 48)])
def test_quantize_rows_bit_exact(rows, d):
    rows = max(rows, 7)
    xb = _rows_with_edge_cases(rows, d, seed=rows + d)
    q, s = _quant_rows(xb.cuda())
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        q_ref, s_ref = O.quantize_rows_e4m3(xb.float().numpy())
    np.testing.assert_array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q, q_ref)


def test_quantize_rows_empty_and_errors():
    x = torch.zeros((0, 32), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((0, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty((0,), dtype=torch.float32, device="cuda")
    ops.moe_quantize_rows_e4m3(x, q, s)  # no-op
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.MoeError):
        ops.moe_quantize_rows_e4m3(x, torch.empty((4, 24), dtype=torch.uint8, device="cuda"),
                                   torch.empty((4,), dtype=torch.float32, device="cuda"))


def _w8a8(**kw):
    return syn.LayerConfig("t", weight_dtype=syn.E4M3, act_quant=1, router_offset_var=1.0, **kw)


@pytest.mark.parametrize("cfg", [
    _w8a8(S=300, d=256, h=384, E=8, K=2),                         # several m-blocks, partial tiles
    _w8a8(S=200, d=320, h=208, E=8, K=2),                         # N and K tails (K not a multiple of 128)
    _w8a8(S=513, d=384, h=256, E=16, K=4, num_shared=1),          # shared expert reads x through its own scales
    syn.scaled(_w8a8(S=700, d=256, h=128, E=64, K=8), capacity=syn.capacity_for(700, 8, 64)),  # overflow pass
    _w8a8(S=4, d=2048, h=1408, E=8, K=2),                         # split-K: row scales applied after the sum
    _w8a8(S=5, d=1024, h=512, E=16, K=4, num_shared=1),           # split-K with the shared group
], ids=["tiles", "tails", "shared", "capacity", "splitk", "splitk_shared"])
def test_grouped_ffn_w8a8(cfg):
    got, ref = ffn_case(cfg)
    err = rel_l2(got, ref)
    print(cfg, err)
    assert err <= FP8_REL_L2


@pytest.mark.parametrize("name,over", [
    ("fp8_skew_capacity_w8a8", dict(S=1024, d=256, h=384)),
    ("mixtral_prefill_w8a8", dict(S=384, d=512, h=768)),
])
def test_layer_w8a8_scaled_down(name, over):
    cfg = syn.scaled(syn.VARIANTS[name], **over)
    inp = syn.make_inputs(cfg, "cuda", seed=2)
    gpu = run_layer(inp, cfg)
    assert_status_clean(gpu["ws"])
    rep = compare_layer(gpu, inp, cfg)
    print(name, rep)
    assert rep["ok"], rep


def test_w8a8_deviation_from_bf16_activations_is_the_rounding_error():
    """Against the layer that keeps bf16 activations (same E4M3 weights) the
    W8A8 output moves by the E4M3 rounding of its activations: each
    quantisation rounds to 3 mantissa bits (relative error <= 2^-4 per element,
    about 2^-4 / sqrt(3) RMS), applied twice in sequence (tokens, then hidden
    rows).  The deviation must be of that size: clearly non-zero (the
    activations really were quantised) and below 2 * 2^-4."""
    cfg = syn.scaled(syn.VARIANTS["mixtral_prefill_w8a8"], S=256, d=512, h=512)
    inp = syn.make_inputs(cfg, "cuda", seed=4)
    y8 = run_layer(inp, cfg)["y"].double().cpu().numpy()
    y16 = run_layer(inp, syn.scaled(cfg, act_quant=0))["y"].double().cpu().numpy()
    dev = rel_l2(y8, y16)
    print("W8A8 vs bf16 activations", dev)
    assert 2.0 ** -6 < dev < 2 * 2.0 ** -4


def _sample(idx, E, n, rng, extra=()):
    S = idx.shape[0]
    toks = set(rng.choice(S, size=min(n, S), replace=False).tolist())
    for e in range(E):
        hit = np.nonzero((idx == e).any(axis=1))[0]
        if len(hit) and not toks.intersection(hit.tolist()):
            toks.add(int(hit[0]))
    toks.update(int(t) for t in extra)
    return np.array(sorted(toks))


@pytest.mark.parametrize("name", ["fp8_skew_capacity_w8a8", "mixtral_prefill_w8a8"])
def test_layer_w8a8_full_size(name):
    """Full-size W8A8 layers, outputs checked on sampled tokens covering every
    expert with tokens (and overflow rows for the capacity-bounded one)."""
    cfg = syn.VARIANTS[name]
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    gpu = run_layer(inp, cfg)
    code, flags, counters = ops.moe_get_status(gpu["ws"])
    assert flags == 0, (flags, counters)
    _, ridx, _, _ = oracle_routing(inp, cfg)
    extra = ()
    if cfg.capacity:
        P = O.expert_permutation(ridx, cfg.E, cfg.capacity)
        ovf_slots = np.nonzero(P["row_of_slot"] >= cfg.E * cfg.capacity)[0]
        extra = np.unique(ovf_slots // cfg.K)[:16]
        assert len(extra) > 0
    toks = _sample(ridx, cfg.E, 32, np.random.default_rng(0), extra)
    rep = compare_layer(gpu, inp, cfg, toks)
    print(name, rep)
    assert rep["ok"], rep
    del inp, gpu
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,over", [
    ("fp8_skew_capacity_w8a8", dict(S=1024, d=256, h=384)),
    ("mixtral_prefill_w8a8", dict(S=300, d=512, h=256, num_shared=1)),
])
def test_fused_gather_quantisation_matches_stage_calls(name, over):
    """moe_layer_forward quantises the token rows inside the row gather; the
    four stage calls quantise the gathered bf16 rows in moe_grouped_ffn.  Both
    encode the same rows the same way, so the outputs are bit-identical."""
    cfg = syn.scaled(syn.VARIANTS[name], **over)
    inp = syn.make_inputs(cfg, "cuda", seed=6)
    fused = run_layer(inp, cfg)
    desc = fused["desc"]
    w = ops.make_weights(inp)
    ws = torch.empty(ops.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
    ops.moe_workspace_init(ws)
    S, E, K = cfg.S, cfg.E, cfg.K
    R = ops.moe_routed_rows(desc)
    idx = torch.empty((S, K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, K), dtype=torch.float32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    offsets = torch.empty((2 * (E + 1),), dtype=torch.int32, device="cuda")
    ros = torch.empty((S * K,), dtype=torch.int32, device="cuda")
    tor = torch.empty((R,), dtype=torch.int32, device="cuda")
    xp = torch.empty((R, cfg.d), dtype=torch.bfloat16, device="cuda")
    yp = torch.empty((R + cfg.num_shared * S, cfg.d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((S, cfg.d), dtype=torch.bfloat16, device="cuda")
    ops.moe_route(desc, w, inp["x"], None, idx, gw, ws)
    ops.moe_permute(desc, inp["x"], idx, counts, offsets, ros, tor, xp, ws)
    ops.moe_grouped_ffn(desc, w, xp, offsets, inp["x"], yp, ws)
    ops.moe_combine(desc, yp, ros, gw, y, ws)
    torch.cuda.synchronize()
    assert_status_clean(ws)
    assert torch.equal(y.view(torch.int16), fused["y"].view(torch.int16))

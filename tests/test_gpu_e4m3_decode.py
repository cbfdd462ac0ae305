"""E4M3 expert weights with bf16 activations: while the experts have at most
1024 routed rows each on average, the GEMM decodes every landed E4M3 weight
tile to bf16 itself (no separate decode pass); above that, one decode pass
writes the bf16 weights to the workspace first.

With all channel scales 1, the layer on E4M3 weights must give exactly the
layer on the same weights decoded to bf16 beforehand (E4M3 -> bf16 is exact,
and both run the same MMAs on the same bf16 values in the same order), with
every finite E4M3 code present in the weights.  The decode is also checked
against the oracle within the FP8 tolerance at the skewed workload's shape
(capacity, overflow rows), small batches (split-K) included.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn

from parity import compare_layer, new_ws, run_layer

pytestmark = pytest.mark.gpu


def _all_codes(shape, seed):
    """uint8 E4M3 codes covering every finite code (0x7F / 0xFF are NaN)."""
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 256, shape, generator=g, dtype=torch.int32)
    flat = codes.view(-1)
    flat[:256] = torch.arange(256, dtype=torch.int32)
    codes = torch.where((codes & 0x7F) == 0x7F, codes - 1, codes)  # NaN codes -> the largest finite ones
    return codes.to(torch.uint8)


@pytest.mark.parametrize("S,E,K,cap", [(256, 8, 2, 0), (5, 8, 2, 0), (700, 16, 4, 180),
                                       (4200, 4, 1, 0)])   # 1050 rows per expert: the decode pass
def test_e4m3_layer_equals_bf16_layer_on_decoded_weights(S, E, K, cap):
    d, h = 256, 384
    cfg8 = syn.LayerConfig("e4m3_exact", S=S, d=d, E=E, K=K, h=h, weight_dtype=syn.E4M3, capacity=cap)
    inp = syn.make_inputs(cfg8, "cuda", seed=21)
    for j, name in enumerate(("w_gate", "w_up", "w_down")):
        inp[name] = _all_codes(tuple(inp[name].shape), 100 + j).cuda()
        inp["s_" + name[2:]] = torch.ones_like(inp["s_" + name[2:]])
    # the same weights decoded exactly to bf16 (E4M3 -> float32 -> bf16 is exact)
    inp16 = dict(inp)
    for name in ("w_gate", "w_up", "w_down"):
        inp16[name] = inp[name].view(torch.float8_e4m3fn).to(torch.float32).to(torch.bfloat16)
        inp16["s_" + name[2:]] = None
    cfg16 = syn.LayerConfig("bf16_exact", S=S, d=d, E=E, K=K, h=h, weight_dtype=syn.BF16, capacity=cap)
    a = run_layer(inp, cfg8)
    b = run_layer(inp16, cfg16)
    for r in (a, b):
        code, flags, counters = ops.moe_get_status(r["ws"])
        assert flags == 0, (flags, counters)
    assert torch.equal(a["idx"], b["idx"])
    assert torch.isfinite(a["y"].float()).all()
    assert torch.equal(a["y"], b["y"])


@pytest.mark.parametrize("S", [16384, 64, 3])
def test_e4m3_skewed_layer_against_oracle(S):
    cfg = syn.scaled(syn.CONFIGS["fp8_skew_capacity"], S=S)
    inp = syn.make_inputs(cfg, "cuda", seed=0)
    gpu = run_layer(inp, cfg)
    code, flags, counters = ops.moe_get_status(gpu["ws"])
    assert flags == 0, (flags, counters)
    toks = np.unique(np.linspace(0, S - 1, num=min(S, 256)).astype(np.int64))
    rep = compare_layer(gpu, inp, cfg, tokens=toks)
    print(S, rep)
    assert rep["ok"], rep

"""E4M3 expert weights with bf16 activations.

With d and h multiples of 16 the expert GEMMs multiply the stored E4M3 weight
codes (kind::f8f6f4) by two-term E4M3 codes of the bf16 activation rows
(moe_split_rows_e4m3: x * 2^k = c1 + c2, exact but for elements far below the
row maximum); otherwise one exact decode pass writes the weights to the
workspace as bf16 first.

Checks: the two-term codes bit-exact against the oracle on rows with every
kind of value; the layer on E4M3 weights against the layer on the same
weights decoded to bf16 beforehand (within the two-term bound and the fp32
summation order: relative L2 1e-3; exactly equal on the decode-pass path),
with every finite E4M3 code present in the weights; and the skewed workload
against the oracle within the FP8 tolerance (capacity, overflow rows, small
batches with split-K).
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn

from oracle import moe_oracle as O
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


def _edge_rows(d, n=40):
    """bf16 rows with every kind of value: spreads from 2**-30 to 1 of the row
    maximum, bf16 subnormals, huge and tiny maxima, maxima of exactly
    448 * 2**j, a zero row, rows holding an infinity or a NaN."""
    rng = np.random.default_rng(77 + n)
    amax = np.exp2(rng.integers(-30, 30, size=(n, 1))).astype(np.float64) * rng.uniform(1, 2, size=(n, 1))
    x = amax * np.exp2(-rng.uniform(0, 30, size=(n, d))) * rng.choice([-1.0, 1.0], size=(n, d))
    x[0] = 0.0
    x[1, :] = 1e-40                       # bf16 subnormals
    x[2, 7] = 448.0 * 2.0 ** 5
    x[3, 0] = 3.0e38
    x[4, 5] = np.inf
    x[5, 9] = np.nan
    x[6] = rng.normal(size=d)
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t


@pytest.mark.parametrize("n,d", [(40, 16), (40, 272), (40, 4096), (1500, 272), (700, 2048)])
def test_split_rows_bit_exact(n, d):
    """Few rows (a CTA per row) and many rows (rows staged in shared memory by
    bulk copies)."""
    x = _edge_rows(d, n)
    xd = x.cuda()
    q = torch.empty((x.shape[0], 2 * d), dtype=torch.uint8, device="cuda")
    s = torch.empty((x.shape[0],), dtype=torch.float32, device="cuda")
    ops.moe_split_rows_e4m3(xd, q, s)
    torch.cuda.synchronize()
    c1, c2, sr = O.split_rows_e4m3(x.float().numpy())
    qh = q.cpu().numpy()
    assert np.array_equal(qh[:, :d], c1)
    assert np.array_equal(qh[:, d:], c2)
    sg = s.cpu().numpy()
    assert np.array_equal(np.isnan(sg), np.isnan(sr))
    fin = ~np.isnan(sr)
    assert np.array_equal(sg[fin], sr[fin])


@pytest.mark.parametrize("S,E,K,cap,d,h", [(256, 8, 2, 0, 256, 384), (5, 8, 2, 0, 256, 384),
                                           (100, 4, 2, 0, 256, 384),   # groups up to 100 rows: 64-row m-blocks
                                           (700, 16, 4, 180, 256, 384), (4200, 4, 1, 0, 256, 384),
                                           (64, 8, 2, 0, 264, 392)])   # d, h not multiples of 16: decode pass
def test_e4m3_layer_against_bf16_layer_on_decoded_weights(S, E, K, cap, d, h):
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
    ya, yb = a["y"].double(), b["y"].double()
    assert torch.isfinite(ya).all()
    if d % 16 or h % 16:
        assert torch.equal(a["y"], b["y"])   # decode pass: the same bf16 GEMMs
    else:
        rel = float(torch.linalg.norm(ya - yb) / torch.linalg.norm(yb))
        assert rel <= 1e-3, rel


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

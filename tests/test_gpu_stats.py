"""The load report (moe_load_stats) and the stage-timed layer call
(moe_layer_forward_timed) on the GPU.

The load report is checked against the oracle's load_stats on hand-built and
random counts; the timed layer call must produce exactly what
moe_layer_forward produces, with its stage events in stream order.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

from parity import new_ws

pytestmark = pytest.mark.gpu


def _stats_gpu(desc, counts_np):
    counts = torch.tensor(counts_np, dtype=torch.int32, device="cuda")
    out = torch.full((ops.MOE_NUM_LOAD_STATS,), -1.0, dtype=torch.float64, device="cuda")
    ops.moe_load_stats(desc, counts, out)
    torch.cuda.synchronize()
    return dict(zip(ops.LOAD_STAT_NAMES, out.cpu().tolist()))


def test_load_stats_hand_built():
    # 16 slots over 4 experts, capacity 3: max/mean 13/4, std 3*sqrt(3), 10 rows over
    desc = ops.make_desc(num_tokens=8, d_model=64, num_experts=4, top_k=2, d_ff=64, capacity=3)
    got = _stats_gpu(desc, [13, 1, 1, 1])
    assert got["max_over_mean"] == 3.25 and got["mean"] == 4.0 and got["max"] == 13.0
    assert got["std"] == pytest.approx(3.0 * np.sqrt(3.0), rel=1e-15)
    assert got["overflow_rows"] == 10.0 and got["dropped"] == 0.0
    # one slot lost to an out-of-range id
    got = _stats_gpu(desc, [12, 1, 1, 1])
    assert got["dropped"] == 1.0


@pytest.mark.parametrize("S,E,K,cap", [(1, 8, 2, 0), (4096, 8, 2, 0), (8192, 256, 8, 0), (16384, 64, 8, 2560),
                                       (100, 1, 1, 0), (3000, 96, 6, 200)])
def test_load_stats_matches_oracle(S, E, K, cap):
    rng = np.random.default_rng(S + E)
    # a skewed multinomial split of the S*K slots
    p = rng.dirichlet(np.full(E, 0.5))
    counts = rng.multinomial(S * K, p).astype(np.int32)
    desc = ops.make_desc(num_tokens=S, d_model=64, num_experts=E, top_k=K, d_ff=64, capacity=cap)
    got = _stats_gpu(desc, counts)
    ref = O.load_stats(counts, K, S, cap)
    for k in ops.LOAD_STAT_NAMES:
        assert got[k] == pytest.approx(ref[k], rel=1e-12, abs=1e-9), (k, got, ref)


@pytest.mark.parametrize("name", ["tiny_f32", "fp8_skew_capacity", "mixtral_prefill_w8a8"])
def test_layer_forward_timed_matches_layer_forward(name):
    cfg = syn.CONFIGS.get(name) or syn.VARIANTS[name]
    cfg = syn.scaled(cfg, S=min(cfg.S, 512), d=min(cfg.d, 512), h=min(cfg.h, 512))
    inp = syn.make_inputs(cfg, "cuda", seed=5)
    desc = ops.make_desc(**syn.desc_dict(cfg))
    w = ops.make_weights(inp)
    adt = torch.float32 if cfg.act_dtype == syn.F32 else torch.bfloat16
    outs = []
    st = torch.cuda.current_stream()
    events = [torch.cuda.Event(enable_timing=True) for _ in range(ops.MOE_NUM_STAGE_EVENTS)]
    for ev in events:
        ev.record(st)  # creates the CUDA events
    for timed in (False, True):
        ws = new_ws(desc)
        y = torch.empty((cfg.S, cfg.d), dtype=adt, device="cuda")
        idx = torch.empty((cfg.S, cfg.K), dtype=torch.int32, device="cuda")
        gw = torch.empty((cfg.S, cfg.K), dtype=torch.float32, device="cuda")
        counts = torch.empty((cfg.E,), dtype=torch.int32, device="cuda")
        if timed:
            ops.moe_layer_forward_timed(desc, w, inp["x"], y, idx, gw, counts, ws, events)
        else:
            ops.moe_layer_forward(desc, w, inp["x"], y, idx, gw, counts, ws)
        torch.cuda.synchronize()
        outs.append((y, idx, gw, counts))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    # the stage events were recorded in stream order
    gaps = [events[i].elapsed_time(events[i + 1]) for i in range(ops.MOE_NUM_STAGE_EVENTS - 1)]
    assert all(g >= 0.0 for g in gaps), gaps
    assert events[3].elapsed_time(events[4]) > 0.0 and events[5].elapsed_time(events[6]) > 0.0


def test_layer_forward_timed_skips_null_events():
    cfg = syn.scaled(syn.CONFIGS["tiny_f32"], S=32)
    inp = syn.make_inputs(cfg, "cuda", seed=6)
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    y = torch.empty((cfg.S, cfg.d), dtype=torch.float32, device="cuda")
    ev = torch.cuda.Event(enable_timing=True)
    ev.record()
    events = [None] * ops.MOE_NUM_STAGE_EVENTS
    events[7] = ev
    ops.moe_layer_forward_timed(desc, ops.make_weights(inp), inp["x"], y, None, None, None, ws, events)
    torch.cuda.synchronize()
    assert ev.query()

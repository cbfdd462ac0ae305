"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random tensors and stores them in the layer's
formats; it contains none of the layer's arithmetic, so that the CUDA path
and the CPU oracle can both be fed from it without sharing code.

Workloads (shapes and distributions of the layer variants the pages discuss;
N(0, v) means variance v):

* ``tiny_f32``: S=64 tokens, d=128, E=8, K=2, softmax top-2 renormalised,
  GeLU experts with biases, h=256, all fp32.  W_r ~ N(0, 1/d),
  W1 ~ N(0, 1/d), W2 ~ N(0, 1/h), b1, b2 ~ N(0, 0.01), x ~ N(0, 1).
* ``mixtral_prefill``: S=4096, d=4096, E=8, K=2, softmax top-2 renormalised,
  SwiGLU experts h=14336 (Mixtral-8x7B shapes), bf16 weights and
  activations, W ~ N(0, 1/fan_in), x ~ N(0, 1).
* ``mixtral_decode``: the same weights at S in {1, 8, 32, 128}; the router
  logits get a per-expert offset ~ N(0, 0.5) so expert loads are uneven.
* ``dsv3_grouped``: S=8192, d=7168, 256 routed experts + 1 shared, K=8,
  h=2048 SwiGLU, bf16; sigmoid scores plus a selection bias ~ N(0, 0.01);
  8 groups of 32, top-2 groups, top-8 experts (DeepSeek-V3 shapes).
* ``fp8_skew_capacity``: S=16384, d=2048, E=64, K=8, h=1408 SwiGLU; expert
  weights FP8-E4M3 with per-output-channel fp32 scales, bf16 activations;
  per-expert router offsets c * z_e, z_e ~ N(0, 1), with c chosen so that the
  max/mean expert load is about 4; capacity ceil(1.25 * S * K / E).

Large tensors are drawn on the target device (torch's Philox generator for
CUDA, its CPU generator on the host), so CPU and GPU runs of the same seed
see different values; every comparison feeds one set of tensors to both
sides.  Small per-expert vectors (router offsets, selection bias) are always
drawn on the CPU so their values do not depend on the device.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

SOFTMAX, SIGMOID = 0, 1
GELU, SWIGLU = 0, 1
F32, BF16, E4M3 = 0, 1, 2

# Scale of the fp8_skew_capacity router offsets.  Calibrated on the CPU
# oracle's routing of the full-size workload (the calibration script sits
# next to the golden files) so that max/mean expert load is close to 4.
SKEW_OFFSET_SCALE = 0.463


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    S: int
    d: int
    E: int
    K: int
    h: int
    score_fn: int = SOFTMAX
    renormalize: int = 1
    num_groups: int = 1
    topk_groups: int = 1
    num_shared: int = 0
    activation: int = SWIGLU
    act_dtype: int = BF16
    weight_dtype: int = BF16
    capacity: int = 0
    act_quant: int = 0               # 1: W8A8 (E4M3 activation rows with per-row scales)
    reroute: int = 0                 # 1: over-capacity slots move to the next-best expert with room
    temperature: float = 0.0         # softmax temperature of the router (0 = 1)
    router_offset_var: float = 0.0   # variance of N(0, v) per-expert logit offsets
    skew_offset_scale: float = 0.0   # c of the c * z_e offsets
    sel_bias_var: float = 0.0        # variance of the selection bias
    bias_var: float = 0.01           # GeLU experts' b1, b2


CONFIGS = {
    "tiny_f32": LayerConfig("tiny_f32", S=64, d=128, E=8, K=2, h=256, activation=GELU,
                            act_dtype=F32, weight_dtype=F32),
    "mixtral_prefill": LayerConfig("mixtral_prefill", S=4096, d=4096, E=8, K=2, h=14336),
    "mixtral_decode": LayerConfig("mixtral_decode", S=1, d=4096, E=8, K=2, h=14336, router_offset_var=0.5),
    "dsv3_grouped": LayerConfig("dsv3_grouped", S=8192, d=7168, E=256, K=8, h=2048, score_fn=SIGMOID,
                                num_groups=8, topk_groups=2, num_shared=1, sel_bias_var=0.01),
    "fp8_skew_capacity": LayerConfig("fp8_skew_capacity", S=16384, d=2048, E=64, K=8, h=1408,
                                     weight_dtype=E4M3, capacity=2560,
                                     skew_offset_scale=SKEW_OFFSET_SCALE),
}

# Variants of the workloads.  W8A8: the same inputs with the expert GEMMs run on E4M3
# activations (per-row scales) against E4M3 weights.  The Mixtral-shaped one
# stores its expert weights as E4M3 with per-output-channel scales.
VARIANTS = {
    "fp8_skew_capacity_w8a8": dataclasses.replace(CONFIGS["fp8_skew_capacity"], name="fp8_skew_capacity_w8a8",
                                                  act_quant=1),
    "mixtral_prefill_w8a8": dataclasses.replace(CONFIGS["mixtral_prefill"], name="mixtral_prefill_w8a8",
                                                weight_dtype=E4M3, act_quant=1),
    # the skewed capacity-bounded layer with over-capacity re-routing instead of the overflow pass
    "fp8_skew_capacity_reroute": dataclasses.replace(CONFIGS["fp8_skew_capacity"], name="fp8_skew_capacity_reroute",
                                                     reroute=1),
    # decode with the Mixtral-shaped expert weights stored as E4M3 (per-channel scales), bf16 activations
    "mixtral_decode_e4m3": dataclasses.replace(CONFIGS["mixtral_decode"], name="mixtral_decode_e4m3",
                                               weight_dtype=E4M3),
}

DECODE_SIZES = (1, 8, 32, 128)


def capacity_for(S: int, K: int, E: int, factor: float = 1.25) -> int:
    return int(math.ceil(factor * S * K / E))


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """The same recipe at other sizes (capacity recomputed when S, K or E
    change and the workload is capacity-bounded)."""
    c = dataclasses.replace(cfg, **kw)
    if cfg.capacity and "capacity" not in kw:
        c = dataclasses.replace(c, capacity=capacity_for(c.S, c.K, c.E))
    return c


def _gen(device, seed: int, stream_id: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + stream_id)
    return g


def _normal(shape, var, g, device, dtype=torch.float32):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if var != 1.0:
        t.mul_(math.sqrt(var))
    return t.to(dtype)


def _act_torch_dtype(code):
    return torch.float32 if code == F32 else torch.bfloat16


def quantize_e4m3_rows(w: torch.Tensor):
    """Per-output-channel (row) FP8-E4M3 encoding of a float32 matrix
    [n, k]: s_n = max_k |w[n, k]| / 448, q = round-to-nearest-even E4M3 of
    w / s_n.  Returns (q as uint8 bit patterns, s fp32 [n])."""
    s = w.abs().amax(dim=1).clamp_min(1e-30) / 448.0
    q = (w / s[:, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), s.to(torch.float32)


def router_offsets(cfg: LayerConfig, seed: int = 0):
    """Per-expert router logit offsets of the workload (CPU tensor), or None."""
    cpu = torch.device("cpu")
    rb = None
    if cfg.router_offset_var > 0:
        rb = _normal((cfg.E,), cfg.router_offset_var, _gen(cpu, seed, 3), cpu)
    if cfg.skew_offset_scale > 0:
        rb = _normal((cfg.E,), 1.0, _gen(cpu, seed, 4), cpu) * cfg.skew_offset_scale
    return rb


def make_inputs(cfg: LayerConfig, device="cpu", seed: int = 0, x_only: bool = False) -> dict:
    """Draw every input of one layer call.  Returns a dict of torch tensors on
    ``device``: x, w_router, router_bias, sel_bias and the expert stacks in the
    library's layouts (out x in, shared expert as the last slab)."""
    dev = torch.device(device)
    S, d, E, h = cfg.S, cfg.d, cfg.E, cfg.h
    adt = _act_torch_dtype(cfg.act_dtype)
    out = {"cfg": cfg}
    out["x"] = _normal((S, d), 1.0, _gen(dev, seed, 1), dev, adt)
    if x_only:
        return out
    cpu = torch.device("cpu")
    out["w_router"] = _normal((E, d), 1.0 / d, _gen(cpu, seed, 2), cpu, adt).to(dev)
    rb = router_offsets(cfg, seed)
    out["router_bias"] = None if rb is None else rb.to(dev)
    out["sel_bias"] = None
    if cfg.sel_bias_var > 0:
        out["sel_bias"] = _normal((E,), cfg.sel_bias_var, _gen(cpu, seed, 5), cpu).to(dev)
    n_slabs = E + cfg.num_shared
    if cfg.activation == GELU:
        wdt = torch.float32 if cfg.weight_dtype == F32 else torch.bfloat16
        out["w1"] = _normal((n_slabs, h, d), 1.0 / d, _gen(dev, seed, 10), dev, wdt)
        out["w2"] = _normal((n_slabs, d, h), 1.0 / h, _gen(dev, seed, 11), dev, wdt)
        out["b1"] = _normal((n_slabs, h), cfg.bias_var, _gen(dev, seed, 12), dev)
        out["b2"] = _normal((n_slabs, d), cfg.bias_var, _gen(dev, seed, 13), dev)
        return out
    shapes = {"w_gate": (h, d, 1.0 / d), "w_up": (h, d, 1.0 / d), "w_down": (d, h, 1.0 / h)}
    for j, (name, (n, k, var)) in enumerate(shapes.items()):
        g = _gen(dev, seed, 20 + j)
        if cfg.weight_dtype == E4M3:
            q = torch.empty((n_slabs, n, k), dtype=torch.uint8, device=dev)
            s = torch.empty((n_slabs, n), dtype=torch.float32, device=dev)
            for e in range(n_slabs):
                q[e], s[e] = quantize_e4m3_rows(_normal((n, k), var, g, dev))
            out[name] = q
            out["s_" + name[2:]] = s
        else:
            wdt = torch.float32 if cfg.weight_dtype == F32 else torch.bfloat16
            t = torch.empty((n_slabs, n, k), dtype=wdt, device=dev)
            for e in range(n_slabs):  # one slab at a time keeps the fp32 temporary small
                t[e] = _normal((n, k), var, g, dev, wdt)
            out[name] = t
    return out


def desc_dict(cfg: LayerConfig, S: Optional[int] = None) -> dict:
    """Field values of the C ABI's moe_desc for this workload."""
    return dict(num_tokens=cfg.S if S is None else S, d_model=cfg.d, num_experts=cfg.E, top_k=cfg.K,
                d_ff=cfg.h, score_fn=cfg.score_fn, renormalize=cfg.renormalize, num_groups=cfg.num_groups,
                topk_groups=cfg.topk_groups, num_shared=cfg.num_shared, activation=cfg.activation,
                act_dtype=cfg.act_dtype, weight_dtype=cfg.weight_dtype, capacity=cfg.capacity,
                act_quant=cfg.act_quant, reroute=cfg.reroute, temperature=cfg.temperature)

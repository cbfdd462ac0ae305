"""Calibrate the router-offset scale c of the fp8_skew_capacity workload.

The workload asks for per-expert router offsets that make the max/mean
expert load about 4 (the top of the 3-5 range quoted in chapter 11, 11.2.3 of
jsqmd.com "第11章 MoE模型推理").  Offsets are c * z_e with z_e ~ N(0, 1)
drawn from the seeded generator; this script bisects c on the CPU oracle's
routing of the full-size workload and prints it.  The printed value is
stored as SKEW_OFFSET_SCALE in the synthetic-input module.

Run: python tests/golden/calibrate_skew.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from mixture_experts_layer_bias_b200 import synthetic as syn  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


def ratio_for(c, base_logits, z, K):
    logits = (base_logits.astype(np.float64) + c * z[None, :]).astype(np.float32)
    idx, _ = O.select_experts(logits, K)
    counts = O.expert_counts(idx, z.shape[0])
    return O.load_stats(counts, K, logits.shape[0])["max_over_mean"]


def main(target=4.0):
    cfg = syn.scaled(syn.CONFIGS["fp8_skew_capacity"], skew_offset_scale=1.0)
    x = syn.make_inputs(cfg, "cpu", seed=0, x_only=True)["x"].float().numpy()
    # router weights and unit offsets exactly as make_inputs draws them
    import torch
    g = syn._gen(torch.device("cpu"), 0, 2)
    w_r = syn._normal((cfg.E, cfg.d), 1.0 / cfg.d, g, torch.device("cpu"), torch.bfloat16).float().numpy()
    z = syn._normal((cfg.E,), 1.0, syn._gen(torch.device("cpu"), 0, 4), torch.device("cpu")).numpy()
    base = O.router_logits(x, w_r)
    lo, hi = 0.0, 4.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if ratio_for(mid, base, z, cfg.K) < target:
            lo = mid
        else:
            hi = mid
    c = round(0.5 * (lo + hi), 3)
    print(f"c = {c:.3f}  max/mean = {ratio_for(c, base, z, cfg.K):.3f}")


if __name__ == "__main__":
    main()

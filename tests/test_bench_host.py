"""Host-side checks of bench.py's bookkeeping (no GPU): the committed DRAM
traffic record belongs to the current GEMM sources, and the launch counts and
algorithmic work figures follow the workloads' shapes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_bias_b200 import synthetic as syn  # noqa: E402


def test_traffic_record_matches_current_gemm_sources():
    """bench.py reports the ncu DRAM bytes only while the GEMM sources are the
    ones they were captured on; the committed record must be current."""
    assert bench.ffn_traffic(bench.FFN_TRAFFIC_CAPTURE["workload"]) == bench.FFN_TRAFFIC_CAPTURE["bytes"]
    assert bench.ffn_traffic("dsv3_grouped") is None


def test_traffic_not_reported_for_other_kernels(monkeypatch):
    for choice in ("pair", "wt", "hybrid", "pairtok"):
        monkeypatch.setenv("MOE_B200_GEMM", choice)
        assert bench.ffn_traffic("mixtral_prefill") is None
    monkeypatch.setenv("MOE_B200_GEMM", "single")
    assert bench.ffn_traffic("mixtral_prefill") is not None


def test_traffic_record_is_near_the_algorithmic_bytes():
    cfg = syn.CONFIGS["mixtral_prefill"]
    rows = cfg.S * cfg.K
    algo = 3 * cfg.E * cfg.d * cfg.h * 2 + rows * (cfg.d + 2 * cfg.h + cfg.d) * 2
    assert 1.0 <= bench.FFN_TRAFFIC_CAPTURE["bytes"] / algo <= 1.2


@pytest.mark.parametrize("name,expected", [
    ("mixtral_prefill", 1 + 5 + 2 + 1),              # fused route, permutation, two GEMMs, combine
    ("dsv3_grouped", 2 + 5 + 2 + 1),                 # router GEMM + top-k
    ("fp8_skew_capacity", 2 + 5 + 2 + 3 + 1),        # E = 64: router GEMM + top-k; three E4M3 decodes
    ("mixtral_prefill_w8a8", 1 + 5 + 2 + 1 + 1),     # + quantisation of the hidden rows
    ("fp8_skew_capacity_reroute", 2 + 5 + 2 + 3 + 5 + 1),  # + ranks (3), assignment, gates
])
def test_kernels_per_layer_call(name, expected):
    cfg = syn.CONFIGS.get(name) or syn.VARIANTS[name]
    assert bench.kernels_per_step(cfg) == expected


def test_expert_flops():
    cfg = syn.CONFIGS["mixtral_prefill"]
    # 6 d h per routed row for SwiGLU: 2.886 TFLOP for the Mixtral-shaped prefill layer
    assert abs(bench.expert_flops(cfg, cfg.S * cfg.K) - 2.886e12) / 2.886e12 < 1e-3
    g = syn.CONFIGS["tiny_f32"]
    assert bench.expert_flops(g, 1) == 4 * g.d * g.h

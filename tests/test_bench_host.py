"""Host-side checks of bench.py's bookkeeping (no GPU): the DRAM traffic
record is reported only for the GEMM sources it was captured on, and the
launch counts and algorithmic work figures follow the workloads' shapes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_bias_b200 import synthetic as syn  # noqa: E402


def test_traffic_record_follows_the_gemm_sources(monkeypatch):
    """bench.py reports the ncu DRAM bytes only while the GEMM sources are the
    ones they were captured on, and only for the captured workload."""
    rec = dict(bench.GEMM_TRAFFIC_CAPTURE)
    monkeypatch.setitem(bench.GEMM_TRAFFIC_CAPTURE, "bytes", 3.5e9)
    monkeypatch.setitem(bench.GEMM_TRAFFIC_CAPTURE, "sha1", bench.gemm_sources_sha1())
    assert bench.gemm_traffic(rec["workload"]) == 3.5e9
    assert bench.gemm_traffic("dsv3_grouped") is None
    monkeypatch.setitem(bench.GEMM_TRAFFIC_CAPTURE, "sha1", "0" * 40)
    assert bench.gemm_traffic(rec["workload"]) is None


def test_committed_traffic_record_is_current_or_absent():
    rec = bench.GEMM_TRAFFIC_CAPTURE
    if rec["bytes"] is not None:
        assert rec["sha1"] == bench.gemm_sources_sha1(), "re-capture the GEMM traffic or clear the record"
        cfg = syn.CONFIGS[rec["workload"]]
        assert 1.0 <= rec["bytes"] / bench.gemm_algorithmic_bytes(cfg) <= 1.3


@pytest.mark.parametrize("name,S,expected", [
    ("mixtral_prefill", None, 1 + 4 + 1 + 2 + 1),           # route, chunked permutation + groups, gather, GEMMs, combine
    ("dsv3_grouped", None, 2 + 4 + 1 + 2 + 1),              # router GEMM + top-k
    ("fp8_skew_capacity", None, 2 + 4 + 1 + 2 + 1 + 1),     # E = 64: router GEMM + top-k; codes of the hidden rows
    ("mixtral_prefill_w8a8", None, 1 + 4 + 1 + 2 + 1 + 1),  # + quantisation of the hidden rows
    ("fp8_skew_capacity_reroute", None, 2 + 4 + 1 + 2 + 1 + 7 + 1),  # + ranks (3), picks, epochs, apply, gates
    ("mixtral_decode_e4m3", 1, 1 + 1 + 1 + 2 + 2 + 1 + 1),  # coded gather, split-K finalizes, hidden codes
    ("mixtral_decode", 1, 1 + 1 + 2 + 2 + 1),               # one-CTA permutation with the gather, split-K finalizes
    ("mixtral_decode", 8, 1 + 1 + 2 + 2 + 1),               # 8 x 2 rows of 8 KB: gathered by the permutation
    ("mixtral_decode", 32, 1 + 1 + 1 + 2 + 2 + 1),          # 512 KB of rows: the gather kernel
    ("tiny_f32", None, 1 + 1 + 2 + 1),                      # fp32: no split-K; 64 x 2 rows of 512 B: folded gather
])
def test_kernels_per_layer_call(name, S, expected):
    cfg = syn.CONFIGS.get(name) or syn.VARIANTS[name]
    assert bench.kernels_per_step(cfg, S) == expected


def test_expert_flops_and_bytes():
    cfg = syn.CONFIGS["mixtral_prefill"]
    # 6 d h per routed row for SwiGLU: 2.886 TFLOP for the Mixtral-shaped prefill layer
    assert abs(bench.expert_flops(cfg, cfg.S * cfg.K) - 2.886e12) / 2.886e12 < 1e-3
    g = syn.CONFIGS["tiny_f32"]
    assert bench.expert_flops(g, 1) == 4 * g.d * g.h
    # weights 2.818 GB + rows 8192 x (d + 2h + d) x 2 B
    assert bench.gemm_algorithmic_bytes(cfg) == 3 * 8 * 4096 * 14336 * 2 + 8192 * (2 * 4096 + 2 * 14336) * 2


def test_only_the_tiny_layer_is_flushed():
    assert bench.layer_bytes(syn.CONFIGS["tiny_f32"]) < bench.L2_BYTES
    for name in ("mixtral_prefill", "dsv3_grouped", "fp8_skew_capacity"):
        assert bench.layer_bytes(syn.CONFIGS[name]) > bench.L2_BYTES
    assert bench.layer_bytes(syn.scaled(syn.CONFIGS["mixtral_decode"], S=1)) > bench.L2_BYTES


def test_every_extra_workload_has_a_cpu_sample():
    for name in bench.EXTRA_WORKLOADS + (bench.WORKLOAD,):
        assert name in bench.CPU_SAMPLES
        bench.get_cfg(name)

"""Benchmark of the MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-decode] [--no-cpu] [--no-workloads]

Headline workload: the Mixtral-shaped prefill layer (S=4096 tokens, d=4096,
E=8 experts, top-2 softmax renormalised, SwiGLU experts h=14336, bf16
weights and activations, fp32 accumulation), synthetic seeded inputs
resident in HBM.  A step is one layer forward (route -> permute -> grouped
FFN -> combine) through the library's C ABI.  The timed steps call
moe_layer_forward_timed, which is moe_layer_forward plus CUDA event records
between its stages on the launching stream, so the per-stage and per-GEMM
times (and the roofline of the grouped GEMM kernel) come from the same timed
layer calls as the headline number.  Expert weights (2.8 GB) exceed the 126
MB L2, so no flush is needed between steps (the tiny workload, which fits in
L2, flushes it with a 256 MB write between steps, outside the timed stages).

Multi-GPU (torchrun): every rank runs an independent replica on its own S
tokens (the layer has no exchange step on one node's data-parallel path);
timing is the max over ranks, value = all ranks' tokens / that time.

Also reported: the end-to-end number with host buffers (pinned host ->
device copy of x, layer, device -> host copy of y inside the timed region),
the decode sweep S in {1, 8, 32, 128} against the HBM roofline, the load
report of the routing (moe_load_stats), the CPU oracle timed on bounded
samples (rank 0 only), and -- under "workloads" -- the same record for every
other workload: tiny fp32, DeepSeek-shaped grouped, skewed FP8 with capacity,
the two W8A8 variants and the re-routing variant.

--impl reference times the CPU oracle as it stands (the only reference this
layer has) on a bounded token sample per step and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from mixture_experts_layer_bias_b200 import ops  # noqa: E402
from mixture_experts_layer_bias_b200 import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s (prefill & decode); % of TC peak or HBM roofline"
WORKLOAD = "mixtral_prefill"
EXTRA_WORKLOADS = ("tiny_f32", "dsv3_grouped", "fp8_skew_capacity", "mixtral_prefill_w8a8",
                   "fp8_skew_capacity_w8a8", "fp8_skew_capacity_reroute")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 FMA rate of the CUDA cores (148 SMs x 128 lanes x 2 FLOP x 1.965 GHz):
# the bound of the fp32 workload's SIMT kernels
F32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
L2_BYTES = 126 << 20
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) of the grouped GEMM kernel's launches (up + down
# projection) in one Mixtral-shaped prefill layer call, from an ncu capture of
# those two launches.  Valid only for the GEMM sources it was taken on: the
# `traffic` field is null whenever their hash differs (bytes None: no capture
# of the current sources yet).
GEMM_TRAFFIC_CAPTURE = {
    "workload": "mixtral_prefill",
    # dram__bytes_read.sum + dram__bytes_write.sum of the up and down GEMM launches of one layer call,
    # one-pass ncu capture of the full-size workload (None: not captured on the current GEMM sources)
    "bytes": 3669152512,  # 1946752512 + 228090368 (up) + 1432097536 + 62212096 (down)
    "sources": ("common.cuh", "gemm_common.cuh", "gemm_sm100.cu"),
    "sha1": "112b954715e693cb4ff154f8fa636d82bd54d4db",
}


def gemm_sources_sha1() -> str:
    h = hashlib.sha1()
    for f in GEMM_TRAFFIC_CAPTURE["sources"]:
        with open(os.path.join(ROOT, "mixture_experts_layer_bias_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def gemm_traffic(workload: str):
    """The committed DRAM bytes of the GEMM launches, or None when the capture
    does not belong to this workload or to the current GEMM sources."""
    rec = GEMM_TRAFFIC_CAPTURE
    if workload != rec["workload"] or rec["bytes"] is None:
        return None
    return rec["bytes"] if gemm_sources_sha1() == rec["sha1"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def get_cfg(name: str) -> syn.LayerConfig:
    return syn.CONFIGS.get(name) or syn.VARIANTS[name]


def workload_desc(cfg):
    return (f"{cfg.name}: S={cfg.S} d={cfg.d} E={cfg.E}{'+1 shared' if cfg.num_shared else ''} K={cfg.K} "
            f"h={cfg.h} {'SwiGLU' if cfg.activation == syn.SWIGLU else 'GeLU'} "
            f"{'bf16' if cfg.act_dtype == syn.BF16 else 'fp32'} act, "
            f"{ {0: 'fp32', 1: 'bf16', 2: 'e4m3'}[cfg.weight_dtype]} weights"
            f"{', capacity ' + str(cfg.capacity) if cfg.capacity else ''}"
            f"{', over-capacity re-routing' if cfg.reroute else ''}"
            f"{', W8A8 (e4m3 activation rows, per-row scales)' if cfg.act_quant else ''}")


def coded_a_rows(cfg):
    """The expert GEMMs read E4M3 codes of their A rows: W8A8, or E4M3 weights
    with bf16 activations (two-term codes; d and h multiples of 16)."""
    return bool(cfg.act_quant) or (cfg.weight_dtype == syn.E4M3 and cfg.act_dtype == syn.BF16
                                   and cfg.d % 16 == 0 and cfg.h % 16 == 0)


def kernels_per_step(cfg, S=None):
    """Launches of this library's kernels in one moe_layer_forward call."""
    S = cfg.S if S is None else S
    small = S * cfg.K <= 4096               # one-CTA permutation for small batches
    elem = 4 if cfg.act_dtype == syn.F32 else 2
    logits_first = cfg.E > 32 or (S > 512 and cfg.E * cfg.d * elem > 64 * 1024)
    n = 2 if logits_first else 1           # logits GEMM + top-k, or the routing kernel computing the logits
    n += 1 if small else 4                 # permutation (+ group table): one kernel, or count, scan, scatter, groups
    coded = coded_a_rows(cfg)
    if coded or not (small and S * cfg.K * cfg.d * elem <= 256 * 1024):
        n += 1                             # row gather (writing E4M3 codes); tiny bf16 batches: inside the permutation
    n += 2                                 # up and down GEMM
    rows = S * cfg.K + cfg.num_shared * S + (cfg.E * cfg.capacity if cfg.capacity else 0)
    if cfg.act_dtype == syn.BF16 and rows <= 4096:
        n += 2                             # split-K finalize of both GEMMs
    if coded:
        n += 1                             # per-row E4M3 codes of the hidden rows
    elif cfg.weight_dtype == syn.E4M3:
        n += 3                             # E4M3 -> bf16 decode of the three stacks (d or h not a multiple of 16)
    if cfg.reroute:
        n += (1 if small else 3) + 4       # ranks, re-route picks, epochs and apply, gates
    n += 1                                 # combine
    return n


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (identity outside a process group)."""
    import torch.distributed as td
    if not (td.is_available() and td.is_initialized()) or td.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, max_ms: float, world: int) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank / (max_ms * 1e-3)


def expert_flops(cfg, rows):
    per_row = (6 if cfg.activation == syn.SWIGLU else 4) * cfg.d * cfg.h
    return rows * per_row


def gemm_algorithmic_bytes(cfg, S=None):
    """Bytes the two expert GEMMs must move: every expert's weights once, the
    permuted rows in, the hidden rows out and in, the expert rows out."""
    S = cfg.S if S is None else S
    rows = S * cfg.K + cfg.num_shared * S
    wbytes = {syn.F32: 4, syn.BF16: 2, syn.E4M3: 1}[cfg.weight_dtype]
    abytes = 4 if cfg.act_dtype == syn.F32 else 2
    if cfg.act_quant:
        abytes = 1  # the GEMMs read 8-bit rows
    n_up = 2 if cfg.activation == syn.SWIGLU else 1
    return ((cfg.E + cfg.num_shared) * (n_up + 1) * cfg.d * cfg.h * wbytes
            + rows * (cfg.d + 2 * cfg.h + cfg.d) * abytes)


def layer_bytes(cfg, S=None):
    """Expert weights plus the token rows in and out of one layer call."""
    S = cfg.S if S is None else S
    wbytes = {syn.F32: 4, syn.BF16: 2, syn.E4M3: 1}[cfg.weight_dtype]
    abytes = 4 if cfg.act_dtype == syn.F32 else 2
    n_up = 2 if cfg.activation == syn.SWIGLU else 1
    return (cfg.E + cfg.num_shared) * (n_up + 1) * cfg.d * cfg.h * wbytes + 2 * S * cfg.d * abytes


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        # raw samples: MOE_B200_CLOCKS_DIR if set, else the system temp directory
        out_dir = os.environ.get("MOE_B200_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"moe_b200_clocks_rank{device_index}.csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={gid}", "--query-gpu=" + ",".join(self.FIELDS),
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# stage intervals of moe_layer_forward_timed's events (include/moe.h)
STAGES = {"route": (0, 1), "permute": (1, 2), "ffn_prep": (2, 3), "up_gemm": (3, 4), "hidden_prep": (4, 5),
          "down_gemm": (5, 6), "combine": (6, 7)}


class LayerRun:
    """Buffers of one workload's layer calls and the timed loop."""

    def __init__(self, cfg, device, S=None, seed=0, inp=None):
        self.cfg = cfg
        self.S = cfg.S if S is None else S
        self.device = device
        self.inp = syn.make_inputs(cfg, device, seed=seed) if inp is None else inp
        self.desc = ops.make_desc(**syn.desc_dict(cfg, self.S))
        self.ws = torch.empty(ops.moe_workspace_size(self.desc), dtype=torch.uint8, device=device)
        ops.moe_workspace_init(self.ws)
        adt = torch.bfloat16 if cfg.act_dtype == syn.BF16 else torch.float32
        self.y = torch.empty((self.S, cfg.d), dtype=adt, device=device)
        self.idx = torch.empty((self.S, cfg.K), dtype=torch.int32, device=device)
        self.gw = torch.empty((self.S, cfg.K), dtype=torch.float32, device=device)
        self.counts = torch.empty((cfg.E,), dtype=torch.int32, device=device)
        self.w = ops.make_weights(self.inp)
        self.flush_buf = None
        if layer_bytes(cfg, self.S) < L2_BYTES:
            # the whole layer fits in L2: overwrite it between timed steps
            self.flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call(self, events=None, stream=None):
        if events is None:
            ops.moe_layer_forward(self.desc, self.w, self.inp["x"], self.y, self.idx, self.gw, self.counts, self.ws,
                                  stream)
        else:
            ops.moe_layer_forward_timed(self.desc, self.w, self.inp["x"], self.y, self.idx, self.gw, self.counts,
                                        self.ws, events, stream)

    def flush(self):
        if self.flush_buf is not None:
            self.flush_buf.fill_(1)

    def timed(self, steps, warmup, dist=False):
        """`warmup` untimed calls, then `steps` timed calls with stage events.
        Returns (total ms over ranks, per-stage mean ms dict)."""
        st = torch.cuda.current_stream()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ops.MOE_NUM_STAGE_EVENTS)] for _ in range(steps)]
        for row in evs:
            for e in row:
                e.record(st)  # creates the events before they are handed to the library
        for _ in range(warmup):
            self.flush()
            self.call()
        torch.cuda.synchronize()
        if dist:
            import torch.distributed as td
            td.barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush()
            self.call(evs[i])
        torch.cuda.synchronize()
        if dist:
            td.barrier()
        per_step = [evs[i][0].elapsed_time(evs[i][7]) for i in range(steps)]
        if self.flush_buf is None:
            total = evs[0][0].elapsed_time(evs[-1][7])   # back-to-back steps: first start to last end
        else:
            total = sum(per_step)                       # the flushes between steps are not timed
        stages = {n: statistics.mean(evs[i][b].elapsed_time(evs[i][c]) for i in range(steps))
                  for n, (b, c) in STAGES.items()}
        stages["step_median"] = statistics.median(per_step)
        return max_over_ranks(total, self.device), stages

    def load_report(self):
        stats = torch.empty(ops.MOE_NUM_LOAD_STATS, dtype=torch.float64, device=self.device)
        ops.moe_load_stats(self.desc, self.counts, stats)
        return {k: round(v, 4) for k, v in zip(ops.LOAD_STAT_NAMES, stats.cpu().tolist())}

    def status(self):
        code, flags, counters = ops.moe_get_status(self.ws)
        if flags:
            raise RuntimeError(f"{self.cfg.name}: device status flags {flags} {counters}")
        return counters


def roofline_for(cfg, S, stages, peaks, workload_name):
    """Roofline of the dominant kernel: the grouped expert GEMM
    (grouped_gemm_tc_kernel, two launches per layer call -- up SwiGLU and
    down projection -- timed by the events around them in the timed calls);
    the fp32 workload's SIMT GEMM (gemm_f32_kernel) against the CUDA cores'
    FP32 rate."""
    rows = S * cfg.K + cfg.num_shared * S
    flops = expert_flops(cfg, rows)
    gemm_ms = stages["up_gemm"] + stages["down_gemm"]
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    algo = gemm_algorithmic_bytes(cfg, S)
    hbm_frac = algo / (gemm_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]
    if cfg.act_dtype == syn.F32:
        return {"bound": "alu", "achieved": round(achieved, 3), "peak": round(F32_SIMT_TFLOPS, 1), "unit": "TFLOP/s",
                "frac": round(achieved / F32_SIMT_TFLOPS, 4), "traffic": None, "algorithmic_bytes": algo,
                "kernel": "gemm_f32_kernel (up GeLU + down launches), per layer call",
                "gemm_ms_per_step": round(gemm_ms, 4),
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x 1.965 GHz",
                "note": "latency-bound: 16.8 MFLOP per call runs in a few microseconds per launch"}
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    kind = "bf16 burst"
    if cfg.weight_dtype == syn.E4M3 and not cfg.act_quant and coded_a_rows(cfg):
        # two E4M3 MMAs (one per activation term) per product: the fp8 peak / 2, i.e. the bf16 peak
        kind = "bf16 burst (two-term E4M3 activations: two E4M3 MMAs per product, half the nominal e4m3 rate)"
    elif cfg.act_quant:
        # E4M3 x E4M3: the measured bf16 peak times the nominal fp8 : bf16 ratio (4.5 : 2.25)
        peak, sustained = 2 * peak, 2 * sustained
        kind = "bf16 burst x 2 (nominal e4m3 : bf16 ratio)"
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "frac_of_sustained_peak": round(achieved / sustained, 4),
            "hbm_frac_of_gemm_bytes": round(hbm_frac, 4),
            "traffic": gemm_traffic(workload_name), "algorithmic_bytes": algo,
            "kernel": "grouped_gemm_tc_kernel (up SwiGLU + down launches), event-timed inside the timed layer calls",
            "gemm_ms_per_step": round(gemm_ms, 4),
            "peak_source": f"{peaks['source']} {kind}"}


def decode_sweep(base_inp, device, peaks, reps=20, dcfg0=None):
    """Decode-regime calls S in {1, 8, 32, 128} on the prefill weights (or
    dcfg0's) with the decode router offsets, captured in a CUDA graph; reports
    us per call (median of five batches of `reps` replays), tokens/s and the
    HBM fraction of the expert weights touched
    (their stored bytes: 2 per bf16 weight, 1 per E4M3 code plus the fp32
    channel scales)."""
    out = {}
    dcfg0 = dcfg0 or syn.CONFIGS["mixtral_decode"]
    for S in syn.DECODE_SIZES:
        cfg = syn.scaled(dcfg0, S=S)
        dinp = syn.make_inputs(cfg, device, seed=0, x_only=True)
        inp = dict(base_inp)
        inp["x"] = dinp["x"]
        inp["router_bias"] = syn.router_offsets(cfg, seed=0).to(device)
        run = LayerRun(cfg, device, S=S, inp=inp)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for _ in range(3):
                run.call(stream=s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            run.call(stream=s)
        # untimed replays first (tens of ms), so that the clocks have left any idle state
        for _ in range(100):
            g.replay()
        torch.cuda.synchronize()
        # five batches of `reps` replays; the median batch's time per call
        batches = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            batches.append(e0.elapsed_time(e1) * 1e3 / reps)
        us = statistics.median(batches)
        touched = int((run.counts > 0).sum().item())
        if cfg.weight_dtype == syn.E4M3:
            wbytes = touched * (3 * cfg.d * cfg.h + (2 * cfg.h + cfg.d) * 4)
        else:
            wbytes = touched * 3 * cfg.d * cfg.h * 2
        gbs = wbytes / (us * 1e-6) / 1e9
        out[str(S)] = {"us_per_call": round(us, 2), "tokens_per_s": round(S / (us * 1e-6), 1),
                       "experts_touched": touched, "weight_bytes": wbytes, "hbm_gbs": round(gbs, 1),
                       "hbm_frac": round(gbs / peaks["hbm_gbs"], 3),
                       "gpu_launches_per_call": kernels_per_step(cfg, S)}
        run.status()
        del g
    return out


def time_bias_update(cfg, device, S, window=1000, reps=50):
    """Mean time of one sliding-window selection-bias update (us)."""
    desc = ops.make_desc(**syn.desc_dict(cfg, S))
    state = torch.empty(ops.moe_bias_state_size(desc, window), dtype=torch.uint8, device=device)
    ops.moe_bias_state_init(state)
    bias = torch.zeros(cfg.E, dtype=torch.float32, device=device)
    idx = torch.randint(0, cfg.E, (S, cfg.K), dtype=torch.int32, device=device)
    for _ in range(3):
        ops.moe_update_sel_bias(desc, idx, window, 0.001, state, bias)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ops.moe_update_sel_bias(desc, idx, window, 0.001, state, bias)
    e1.record()
    torch.cuda.synchronize()
    return round(e0.elapsed_time(e1) * 1e3 / reps, 2)


def time_routing(run, peaks, reps=20, nbuf=5):
    """The routing call alone (moe_route: logits, scoring, top-K), `reps`
    calls captured in a CUDA graph over `nbuf` token buffers together larger
    than L2; us per call (median of seven replays) and the HBM fraction of
    its algorithmic bytes (x, W_r, the ids and gates written)."""
    cfg, S, dev = run.cfg, run.S, run.device
    xs = [run.inp["x"]] + [syn.make_inputs(cfg, dev, seed=100 + i, x_only=True)["x"] for i in range(nbuf - 1)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(3):
            ops.moe_route(run.desc, run.w, xs[0], None, run.idx, run.gw, run.ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(reps):
            ops.moe_route(run.desc, run.w, xs[i % nbuf], None, run.idx, run.gw, run.ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(7):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / reps)
    del g
    us = statistics.median(times)
    b = 2 if cfg.act_dtype == syn.BF16 else 4
    nbytes = S * cfg.d * b + cfg.E * cfg.d * b + S * cfg.K * 8
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"us_per_call": round(us, 2), "bytes": nbytes, "hbm_gbs": round(gbs, 1),
            "hbm_frac": round(gbs / peaks["hbm_gbs"], 3),
            "note": f"{reps} calls in a CUDA graph over {nbuf} token buffers ({nbuf * S * cfg.d * b / 1e6:.0f} MB)"}


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline (rank 0, bounded samples)
# ---------------------------------------------------------------------------

def _oracle_modules():
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np

    from oracle import moe_oracle as O
    from parity import SCORE, OracleExperts, np64, oracle_layer
    return np, O, SCORE, OracleExperts, np64, oracle_layer


def _blas_threads():
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])


def oracle_routing_permutation_rate(cfg, inp):
    """Tokens/s of the oracle's router logits, selection and permutation over
    all S tokens of the workload (float64 router, float32 keys)."""
    np, O, SCORE, _, np64, _ = _oracle_modules()
    x = np64(inp["x"])
    wr = np64(inp["w_router"])
    rb = None if inp.get("router_bias") is None else np64(inp["router_bias"])
    sb = None if inp.get("sel_bias") is None else inp["sel_bias"].cpu().numpy().astype(np.float32)
    t0 = time.perf_counter()
    logits = O.router_logits(x, wr, rb)
    idx, _ = O.select_experts(logits, cfg.K, SCORE[cfg.score_fn], bool(cfg.renormalize), sb, cfg.num_groups,
                              cfg.topk_groups, cfg.temperature or 1.0)
    O.expert_permutation(idx, cfg.E, cfg.capacity)
    dt = time.perf_counter() - t0
    return cfg.S / dt, dt


def oracle_layer_rate(cfg, inp, n_tokens):
    """Tokens/s of the whole oracle layer (routing + the tokens' experts in
    float64) on the first n_tokens tokens."""
    np, _, _, _, _, oracle_layer = _oracle_modules()
    toks = np.arange(n_tokens)
    t0 = time.perf_counter()
    oracle_layer(inp, cfg, toks)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def cpu_baseline(cfg, inp, n_tokens, one_core_tokens):
    """The CPU oracle as it stands: the layer on a bounded token sample (all
    host threads BLAS uses, then one core), and routing + permutation on the
    whole workload."""
    from threadpoolctl import threadpool_limits
    rate, dt = oracle_layer_rate(cfg, inp, n_tokens)
    threads = _blas_threads()
    rp_rate, rp_dt = oracle_routing_permutation_rate(cfg, inp)
    torch_threads = torch.get_num_threads()
    with threadpool_limits(limits=1):
        torch.set_num_threads(1)
        try:
            rate1, dt1 = oracle_layer_rate(cfg, inp, one_core_tokens)
            rp1, rp_dt1 = oracle_routing_permutation_rate(cfg, inp) if cfg.S <= 8192 else (None, None)
        finally:
            torch.set_num_threads(torch_threads)
    return {"value": round(rate, 3), "unit": "tokens/s", "cores": threads, "nproc": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n_tokens} tokens of {cfg.name}: routing + their experts' FFN in float64 ({dt:.1f} s)",
            "one_core": {"value": round(rate1, 3), "unit": "tokens/s",
                         "sample": f"{one_core_tokens} tokens, 1 BLAS thread ({dt1:.1f} s)"},
            "routing_permutation": {"value": round(rp_rate, 1), "unit": "tokens/s", "cores": threads,
                                    "sample": f"all {cfg.S} tokens ({rp_dt:.2f} s)",
                                    "one_core_value": None if rp1 is None else round(rp1, 1)}}


# sample sizes of the oracle baseline per workload: (layer tokens, 1-core layer tokens)
CPU_SAMPLES = {"mixtral_prefill": (32, 8), "tiny_f32": (64, 64), "dsv3_grouped": (4, 1),
               "fp8_skew_capacity": (16, 4), "mixtral_prefill_w8a8": (2, 1), "fp8_skew_capacity_w8a8": (8, 2),
               "fp8_skew_capacity_reroute": (16, 4), "mixtral_decode": (1, 1)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    name = WORKLOAD if args.workload.startswith("profile_small") else args.workload
    cfg = get_cfg(name)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = syn.make_inputs(cfg, dev, seed=0)
    n_tok = 8
    import numpy as np
    _, _, _, _, _, oracle_layer = _oracle_modules()
    for i in range(args.warmup):
        oracle_layer(inp, cfg, np.arange(i * n_tok, (i + 1) * n_tok) % cfg.S)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_layer(inp, cfg, np.arange(i * n_tok, (i + 1) * n_tok) % cfg.S)
    dt = time.perf_counter() - t0
    value = n_tok * args.steps / dt
    threads = _blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(cfg), "global_batch": cfg.S,
                                            "seq_len": cfg.S, "parallelism": "none (CPU oracle)"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads, "nproc": os.cpu_count(),
                             "kind": "oracle", "sample": f"{n_tok} tokens per step of {cfg.name}"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def e2e_run(run, steps, warmup, world, dist):
    """The same metric end to end through moe_layer_forward with host
    buffers: every step copies its input from pinned host memory and its
    output back.  As in a serving loop, step i+1's upload and step i-1's
    download overlap step i's layer (two copy streams, double-buffered device
    buffers); the layer calls stay serialised on one stream because they
    share the workspace."""
    cfg, S, device = run.cfg, run.S, run.device
    x_host = [run.inp["x"].cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty((S, cfg.d), dtype=x_host[0].dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(run.inp["x"]) for _ in range(2)]
    y_dev = [torch.empty((S, cfg.d), dtype=run.inp["x"].dtype, device=device) for _ in range(2)]
    comp = torch.cuda.current_stream()
    up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        computed[b].record(comp)
        downloaded[b].record(comp)

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(up_s):
            up_s.wait_event(computed[b])       # x_dev[b] no longer read by the layer two steps back
            x_dev[b].copy_(x_host[b], non_blocking=True)
            uploaded[b].record(up_s)
        comp.wait_event(uploaded[b])
        comp.wait_event(downloaded[b])          # y_dev[b] already copied out
        ops.moe_layer_forward(run.desc, run.w, x_dev[b], y_dev[b], None, None, None, run.ws, comp)
        computed[b].record(comp)
        with torch.cuda.stream(down_s):
            down_s.wait_event(computed[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            downloaded[b].record(down_s)

    for i in range(warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        import torch.distributed as td
        td.barrier()
    t0 = time.perf_counter()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    for i in range(steps):
        e2e_step(i)
    for b in range(2):
        comp.wait_event(downloaded[b])
    stop.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), device)
    return {"value": round(whole_job_rate(S * steps, ms, world), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": x_host[0].numel() * x_host[0].element_size(),
            "d2h_bytes_per_step": y_host[0].numel() * y_host[0].element_size(),
            "copies": "overlapped with the neighbouring steps' layers (2 copy streams)",
            "wall_ms": round((time.perf_counter() - t0) * 1e3, 3)}


def workload_record(name, device, peaks, steps, warmup, with_cpu):
    """One extra workload: timed layer calls, roofline, load report, oracle."""
    cfg = get_cfg(name)
    run = LayerRun(cfg, device)
    total_ms, stages = run.timed(steps, warmup)
    counters = run.status()
    rec = {"workload": workload_desc(cfg), "value": round(whole_job_rate(cfg.S * steps, total_ms, 1), 1),
           "unit": "tokens/s", "ms_per_step": round(total_ms / steps, 4), "steps": steps, "warmup": warmup,
           "l2": "flushed (256 MB write) between steps, outside the timed stages" if run.flush_buf is not None
                 else "no flush: the expert weights read every step exceed the 126 MB L2",
           "roofline": roofline_for(cfg, cfg.S, stages, peaks, name),
           "stages_ms": {k: round(v, 4) for k, v in stages.items()},
           "load": run.load_report(), "counters": counters,
           "gpu_launches": kernels_per_step(cfg) * steps}
    if with_cpu:
        n, n1 = CPU_SAMPLES.get(name, (8, 2))
        rec["cpu_baseline"] = cpu_baseline(cfg, run.inp, n, n1)
    del run
    gc.collect()
    torch.cuda.empty_cache()
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the records of the other workloads")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=sorted(syn.CONFIGS) + sorted(syn.VARIANTS)
                    + ["profile_small", "profile_small_w8a8", "profile_small_dsv3"],
                    help="profile_small*: smaller cases of the same kernels (0.4-2.9 GB of weights) for ncu "
                         "captures: Mixtral-shaped S=2048, h=4096 (bf16 or W8A8); DeepSeek-shaped S=1024 with "
                         "32 routed experts in 4 groups (top-2 groups, biased selection: uneven loads around "
                         "256 rows) + the shared one")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if dist:
        import datetime

        import torch.distributed as td
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    peaks = load_peaks()
    if args.workload == "profile_small":
        cfg = syn.scaled(syn.CONFIGS[WORKLOAD], S=2048, h=4096)
    elif args.workload == "profile_small_w8a8":
        cfg = syn.scaled(syn.VARIANTS["mixtral_prefill_w8a8"], S=2048, h=4096)
    elif args.workload == "profile_small_dsv3":
        cfg = syn.scaled(syn.CONFIGS["dsv3_grouped"], S=1024, E=32, num_groups=4, topk_groups=2)
    else:
        cfg = get_cfg(args.workload)
    S = cfg.S
    run = LayerRun(cfg, device)

    # timed region: K layer forwards through the public call, with stage events
    clocks = ClockSampler(local)
    total_ms, stages = run.timed(args.steps, args.warmup, dist)
    clk = clocks.stop()
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(S * args.steps, total_ms, world)
    counters = run.status()
    roofline = roofline_for(cfg, S, stages, peaks, args.workload)
    load = run.load_report()

    e2e = e2e_run(run, args.steps, args.warmup, world, dist)
    bias_us = time_bias_update(cfg, device, S)
    routing = time_routing(run, peaks)
    dec = dec8 = None
    if not args.no_decode and args.workload == WORKLOAD:
        # right after the power-capped prefill loop the clocks are still held down for a
        # moment; the decode sweep measures the steady decode regime after a short pause
        time.sleep(3.0)
        dec = decode_sweep(run.inp, device, peaks)
    inp = run.inp
    del run
    gc.collect()
    torch.cuda.empty_cache()
    if not args.no_decode and args.workload == WORKLOAD:
        # the same decode sizes on E4M3 expert weights (two-term E4M3 activations)
        c8 = syn.VARIANTS["mixtral_decode_e4m3"]
        inp8 = syn.make_inputs(c8, device, seed=0)
        dec8 = decode_sweep(inp8, device, peaks, dcfg0=c8)
        del inp8
        gc.collect()
        torch.cuda.empty_cache()
    workloads = None
    if not args.no_workloads and args.workload == WORKLOAD:
        workloads = {}
        for name in EXTRA_WORKLOADS:
            workloads[name] = workload_record(name, device, peaks, max(5, args.steps // 2), args.warmup,
                                              with_cpu=(not args.no_cpu and world == 1 and rank == 0))
    if dist:
        td.barrier()
        td.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu and world == 1:
        n, n1 = CPU_SAMPLES.get(cfg.name, (8, 2))
        cpu = cpu_baseline(cfg, inp, n, n1)
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if cfg.act_quant else "bf16",
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "global_batch": world * S, "seq_len": S,
                       "parallelism": f"replicas x{world}",
                       "l2": "no flush: the expert weights read every step exceed the 126 MB L2"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_step(cfg) * args.steps, "clocks": clk,
            "stages_ms": {k: round(v, 4) for k, v in stages.items()},
            "load": load, "decode_sweep": dec, "decode_sweep_e4m3": dec8, "bias_update_us": bias_us,
            "routing": routing, "counters": counters,
            "workloads": workloads}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

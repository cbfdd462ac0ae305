"""Helpers of the GPU parity tests: run the library through its C ABI and the
oracle on the same seeded inputs, and compare."""
from __future__ import annotations


import numpy as np
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

SCORE = {0: "softmax", 1: "sigmoid"}

# tolerances from the parity contract
F32_MAXABS_REL = 1e-4   # max-abs error <= 1e-4 * max|ref|
BF16_REL_L2 = 1e-2
FP8_REL_L2 = 3e-2
MARGIN = 1e-4           # tokens with a K-th vs (K+1)-th key gap below this are excluded end to end


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs_rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def new_ws(desc, device="cuda"):
    n = ops.moe_workspace_size(desc)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    ops.moe_workspace_init(ws)
    return ws


def assert_status_clean(ws, ignore=0):
    code, flags, counters = ops.moe_get_status(ws)
    assert (flags & ~ignore) == 0, (flags, counters)
    return counters


class OracleExperts:
    """expert_fn(e, rows) of the oracle over the synthetic weights (converted
    to float64 one slab at a time)."""

    def __init__(self, inp: dict, cfg: syn.LayerConfig):
        self.inp, self.cfg = inp, cfg
        self._cache = {}

    def _slab(self, name, e):
        key = (name, e)
        if key not in self._cache:
            t = self.inp[name][e]
            if self.cfg.weight_dtype == syn.E4M3 and name in ("w_gate", "w_up", "w_down"):
                arr = O.e4m3_bits_to_f64(t.cpu().numpy())
            else:
                arr = np64(t)
            if len(self._cache) > 6:
                self._cache.clear()
            self._cache[key] = arr
        return self._cache[key]

    def __call__(self, e, rows):
        cfg = self.cfg
        if cfg.act_quant:
            codes = [self.inp[n][e].cpu().numpy() for n in ("w_gate", "w_up", "w_down")]
            return O.expert_swiglu_w8a8(rows, *codes, np64(self.inp["s_gate"][e]), np64(self.inp["s_up"][e]),
                                        np64(self.inp["s_down"][e]), round_hidden_bf16=True)
        if cfg.activation == syn.GELU:
            return O.expert_gelu(rows, self._slab("w1", e), np64(self.inp["b1"][e]), self._slab("w2", e),
                                 np64(self.inp["b2"][e]))
        sc = {}
        if cfg.weight_dtype == syn.E4M3:
            sc = dict(s_gate=np64(self.inp["s_gate"][e]), s_up=np64(self.inp["s_up"][e]),
                      s_down=np64(self.inp["s_down"][e]))
        return O.expert_swiglu(rows, self._slab("w_gate", e), self._slab("w_up", e), self._slab("w_down", e),
                               round_hidden_bf16=cfg.act_dtype == syn.BF16, **sc)


def oracle_routing(inp: dict, cfg: syn.LayerConfig, tokens=None):
    """Oracle router logits, selection, gates and margins for the given
    tokens (all by default).  With re-routing the assignment depends on the
    whole batch, so every token is routed and the given ones returned."""
    if cfg.reroute and tokens is not None:
        x, idx, w, margin = oracle_routing(inp, cfg)
        tokens = np.asarray(tokens)
        return x[tokens], idx[tokens], w[tokens], margin[tokens]
    x = np64(inp["x"]) if tokens is None else np64(inp["x"][tokens])
    rb = None if inp.get("router_bias") is None else np64(inp["router_bias"])
    logits = O.router_logits(x, np64(inp["w_router"]), rb)
    sb = None if inp.get("sel_bias") is None else inp["sel_bias"].cpu().numpy().astype(np.float32)
    tau = cfg.temperature or 1.0
    idx, w = O.select_experts(logits, cfg.K, SCORE[cfg.score_fn], bool(cfg.renormalize), sb, cfg.num_groups,
                              cfg.topk_groups, tau)
    margin = O.selection_margin(logits, cfg.K, SCORE[cfg.score_fn], sb, cfg.num_groups, cfg.topk_groups, tau)
    if cfg.reroute:
        idx, w = oracle_reroute(logits, idx, cfg, sb)
    return x, idx, w, margin


def oracle_reroute(logits, idx, cfg: syn.LayerConfig, sel_bias=None):
    """Over-capacity re-routing of the oracle's selection, gates recomputed."""
    scores, keys, cand = O.selection_keys(logits, SCORE[cfg.score_fn], sel_bias, cfg.num_groups, cfg.topk_groups,
                                          cfg.temperature or 1.0)
    new, _ = O.reroute_over_capacity(idx, keys, cand, cfg.capacity)
    return new, O.gate_weights(scores, new, SCORE[cfg.score_fn], bool(cfg.renormalize))


def oracle_layer(inp: dict, cfg: syn.LayerConfig, tokens=None):
    """Oracle layer output for the given tokens, with its routing."""
    x, idx, w, margin = oracle_routing(inp, cfg, tokens)
    fn = OracleExperts(inp, cfg)
    shared = (lambda rows: fn(cfg.E, rows)) if cfg.num_shared else None
    y = O.moe_layer(x, idx, w, fn, cfg.E, shared_fn=shared)
    return y, idx, w, margin


def run_layer(inp: dict, cfg: syn.LayerConfig, S=None):
    """The whole layer through moe_layer_forward."""
    S = cfg.S if S is None else S
    desc = ops.make_desc(**syn.desc_dict(cfg, S))
    weights = ops.make_weights(inp)
    ws = new_ws(desc)
    adt = torch.float32 if cfg.act_dtype == syn.F32 else torch.bfloat16
    y = torch.empty((S, cfg.d), dtype=adt, device="cuda")
    idx = torch.empty((S, cfg.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, cfg.K), dtype=torch.float32, device="cuda")
    counts = torch.empty((cfg.E,), dtype=torch.int32, device="cuda")
    ops.moe_layer_forward(desc, weights, inp["x"], y, idx, gw, counts, ws)
    torch.cuda.synchronize()
    return dict(y=y, idx=idx, w=gw, counts=counts, ws=ws, desc=desc)


def compare_layer(gpu: dict, inp: dict, cfg: syn.LayerConfig, tokens=None, tol=None):
    """Compare GPU layer output rows (tokens) with the oracle, excluding
    tokens whose selection margin is below MARGIN.  Returns a report."""
    if tokens is None:
        tokens = np.arange(cfg.S)
    tokens = np.asarray(tokens)
    y_ref, idx_ref, w_ref, margin = oracle_layer(inp, cfg, tokens)
    keep = margin >= MARGIN
    y_gpu = np64(gpu["y"])[tokens]
    idx_gpu = gpu["idx"].cpu().numpy()[tokens]
    route_ok = (idx_gpu[keep] == idx_ref[keep]).all()
    rep = dict(n=len(tokens), excluded=int((~keep).sum()))
    if cfg.act_dtype == syn.F32:
        rep["max_abs_rel"] = max_abs_rel(y_gpu[keep], y_ref[keep])
        rep["ok"] = bool(route_ok and rep["max_abs_rel"] <= (tol or F32_MAXABS_REL))
    else:
        rep["rel_l2"] = rel_l2(y_gpu[keep], y_ref[keep])
        lim = tol or (FP8_REL_L2 if cfg.weight_dtype == syn.E4M3 else BF16_REL_L2)
        rep["ok"] = bool(route_ok and rep["rel_l2"] <= lim)
    rep["route_ok"] = bool(route_ok)
    return rep


def skewed_logits(rng, S, E, spread=1.5):
    """Random float32 logits with per-expert offsets (uneven loads)."""
    return (rng.normal(size=(S, E)) + spread * rng.normal(size=E)[None, :]).astype(np.float32)


def ffn_case(cfg, seed=0):
    """Route with the oracle, permute with the oracle, run moe_grouped_ffn and
    compare every written row with the oracle expert on that row."""
    inp = syn.make_inputs(cfg, "cuda", seed=seed)
    x, ridx, rw, _ = oracle_routing(inp, cfg)
    P = O.expert_permutation(ridx, cfg.E, cfg.capacity)
    R = P["num_rows"]
    desc = ops.make_desc(**syn.desc_dict(cfg))
    ws = new_ws(desc)
    tor = P["token_of_row"]
    used = np.nonzero(tor >= 0)[0]
    xp = torch.zeros((R, cfg.d), dtype=inp["x"].dtype, device="cuda")
    xp[torch.tensor(used, device="cuda")] = inp["x"][torch.tensor(tor[used], device="cuda", dtype=torch.long)]
    offs = P["offsets"] if not cfg.capacity else np.concatenate([P["offsets"], P["ovf_offsets"]])
    Rt = R + cfg.num_shared * cfg.S
    yp = torch.zeros((Rt, cfg.d), dtype=inp["x"].dtype, device="cuda")
    ops.moe_grouped_ffn(desc, ops.make_weights(inp), xp, torch.tensor(offs, dtype=torch.int32, device="cuda"),
                        inp["x"], yp, ws)
    torch.cuda.synchronize()
    assert_status_clean(ws)
    fn = OracleExperts(inp, cfg)
    ref = np.zeros((Rt, cfg.d))
    flat = ridx.reshape(-1)
    for e in range(cfg.E):
        rows = P["row_of_slot"][flat == e]
        if len(rows):
            ref[rows] = fn(e, x[tor[rows]])
    if cfg.num_shared:
        ref[R:] = fn(cfg.E, x)
    rows_all = np.concatenate([used, np.arange(R, Rt)])
    return np64(yp)[rows_all], ref[rows_all]

"""ctypes binding of the C ABI in include/moe.h (argument marshalling only).

Every function takes torch tensors (or None) for device buffers, passes their
data pointers and the current CUDA stream to the library, and raises
``MoeError`` on a non-OK status.  All computation happens in the library's
kernels; nothing here falls back to another implementation: if the shared
library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
_lib = None

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_STATUS = range(6)
MOE_STATUS_NONFINITE_LOGIT, MOE_STATUS_BAD_EXPERT_ID, MOE_STATUS_TIMEOUT, MOE_STATUS_BAD_GROUP = 1, 2, 4, 8
MOE_STATUS_DEBUG_CHECK = 0x10
MOE_NUM_COUNTERS = 8
COUNTER_NAMES = ("nonfinite", "bad_id", "timeout", "overflow_rows", "rerouted")

DESC_FIELDS = ("num_tokens", "d_model", "num_experts", "top_k", "d_ff", "score_fn", "renormalize", "num_groups",
               "topk_groups", "num_shared", "activation", "act_dtype", "weight_dtype", "capacity", "act_quant",
               "reroute", "temperature")
DESC_FLOAT_FIELDS = ("temperature",)
WEIGHT_FIELDS = ("w_router", "router_bias", "sel_bias", "w1", "b1", "w2", "b2", "w_gate", "w_up", "w_down",
                 "s_gate", "s_up", "s_down")

EXPORTED = ("moe_routed_rows", "moe_workspace_size", "moe_workspace_init", "moe_route", "moe_permute",
            "moe_permute_static", "moe_grouped_ffn", "moe_combine", "moe_layer_forward", "moe_layer_forward_timed",
            "moe_load_stats", "moe_bias_state_size", "moe_bias_state_init", "moe_update_sel_bias",
            "moe_quantize_rows_e4m3", "moe_split_rows_e4m3", "moe_reroute", "moe_get_status", "moe_strerror")

MOE_NUM_STAGE_EVENTS = 8
MOE_NUM_LOAD_STATS = 6
LOAD_STAT_NAMES = ("max_over_mean", "std", "mean", "max", "overflow_rows", "dropped")


class MoeDesc(ctypes.Structure):
    _fields_ = [(f, ctypes.c_float if f in DESC_FLOAT_FIELDS else ctypes.c_int32) for f in DESC_FIELDS]


class MoeWeights(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in WEIGHT_FIELDS]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (status {code})")


def lib():
    """Load libmoe_b200.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m mixture_experts_layer_bias_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    pd, pw = ctypes.POINTER(MoeDesc), ctypes.POINTER(MoeWeights)
    sig = {
        "moe_routed_rows": (ctypes.c_int64, [pd]),
        "moe_workspace_size": (I, [pd, ctypes.POINTER(ctypes.c_size_t)]),
        "moe_workspace_init": (I, [P, SZ, P]),
        "moe_route": (I, [pd, pw, P, P, P, P, P, SZ, P]),
        "moe_permute": (I, [pd, P, P, P, P, P, P, P, P, SZ, P]),
        "moe_permute_static": (I, [pd, P, P, P, P, P, P, P, P]),
        "moe_grouped_ffn": (I, [pd, pw, P, P, P, P, P, SZ, P]),
        "moe_combine": (I, [pd, P, P, P, P, P, SZ, P]),
        "moe_layer_forward": (I, [pd, pw, P, P, P, P, P, P, SZ, P]),
        "moe_layer_forward_timed": (I, [pd, pw, P, P, P, P, P, P, SZ, P, ctypes.POINTER(ctypes.c_void_p)]),
        "moe_load_stats": (I, [pd, P, P, P]),
        "moe_bias_state_size": (I, [pd, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
        "moe_bias_state_init": (I, [P, SZ, P]),
        "moe_update_sel_bias": (I, [pd, P, ctypes.c_int32, ctypes.c_float, P, SZ, P, P, P]),
        "moe_quantize_rows_e4m3": (I, [P, ctypes.c_int64, ctypes.c_int32, P, P, P]),
        "moe_split_rows_e4m3": (I, [P, ctypes.c_int64, ctypes.c_int32, P, P, P]),
        "moe_reroute": (I, [pd, P, P, P, P, P, SZ, P]),
        "moe_get_status": (I, [P, P, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_int32)]),
        "moe_strerror": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def make_desc(**fields) -> MoeDesc:
    d = MoeDesc()
    defaults = dict(score_fn=0, renormalize=1, num_groups=1, topk_groups=1, num_shared=0, activation=1,
                    act_dtype=1, weight_dtype=1, capacity=0, act_quant=0, reroute=0, temperature=0.0)
    defaults.update(fields)
    for f in DESC_FIELDS:
        setattr(d, f, float(defaults[f]) if f in DESC_FLOAT_FIELDS else int(defaults[f]))
    return d


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def make_weights(tensors: dict) -> MoeWeights:
    """Weights struct from a dict of tensors (missing names -> NULL).  The
    caller keeps the tensors alive."""
    w = MoeWeights()
    for f in WEIGHT_FIELDS:
        setattr(w, f, _ptr(tensors.get(f)))
    return w


def _stream(stream) -> Optional[int]:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(ws):
    return _ptr(ws), (ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0)


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


def moe_routed_rows(desc: MoeDesc) -> int:
    r = lib().moe_routed_rows(ctypes.byref(desc))
    if r < 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_routed_rows")
    return int(r)


def moe_workspace_size(desc: MoeDesc) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(desc), ctypes.byref(n)), "moe_workspace_size")
    return int(n.value)


def moe_workspace_init(ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_workspace_init(p, n, _stream(stream)), "moe_workspace_init")


def moe_route(desc, weights, x, logits_in, topk_idx, topk_w, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_route(ctypes.byref(desc), ctypes.byref(weights), _ptr(x), _ptr(logits_in), _ptr(topk_idx),
                           _ptr(topk_w), p, n, _stream(stream)), "moe_route")


def moe_permute(desc, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_permute(ctypes.byref(desc), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                             _ptr(row_of_slot), _ptr(token_of_row), _ptr(x_perm), p, n, _stream(stream)),
           "moe_permute")


def moe_permute_static(desc, x, topk_idx, counts, offsets, row_of_slot, token_of_row, x_perm, stream=None):
    """moe_permute without a workspace: its scratch is a fixed 256 KB device
    array inside the library (for callers that cannot allocate)."""
    _check(lib().moe_permute_static(ctypes.byref(desc), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                    _ptr(row_of_slot), _ptr(token_of_row), _ptr(x_perm), _stream(stream)),
           "moe_permute_static")


def moe_grouped_ffn(desc, weights, x_perm, offsets, x, y_perm, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_grouped_ffn(ctypes.byref(desc), ctypes.byref(weights), _ptr(x_perm), _ptr(offsets), _ptr(x),
                                 _ptr(y_perm), p, n, _stream(stream)), "moe_grouped_ffn")


def moe_combine(desc, y_perm, row_of_slot, topk_w, y, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_combine(ctypes.byref(desc), _ptr(y_perm), _ptr(row_of_slot), _ptr(topk_w), _ptr(y), p, n,
                             _stream(stream)), "moe_combine")


def moe_layer_forward(desc, weights, x, y, topk_idx, topk_w, counts, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_layer_forward(ctypes.byref(desc), ctypes.byref(weights), _ptr(x), _ptr(y), _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(counts), p, n, _stream(stream)), "moe_layer_forward")


def moe_layer_forward_timed(desc, weights, x, y, topk_idx, topk_w, counts, ws, events, stream=None):
    """moe_layer_forward recording the stage events: `events` is a list of
    MOE_NUM_STAGE_EVENTS torch.cuda.Event (or None) already created on this
    device (record each once, or query it, before the first call)."""
    p, n = _ws(ws)
    handles = (ctypes.c_void_p * MOE_NUM_STAGE_EVENTS)()
    for i, ev in enumerate(events):
        handles[i] = None if ev is None else ev.cuda_event
    _check(lib().moe_layer_forward_timed(ctypes.byref(desc), ctypes.byref(weights), _ptr(x), _ptr(y), _ptr(topk_idx),
                                         _ptr(topk_w), _ptr(counts), p, n, _stream(stream), handles),
           "moe_layer_forward_timed")


def moe_load_stats(desc, counts, stats, stream=None):
    """Load report of the counts [E] into stats (float64 [6], device): see
    LOAD_STAT_NAMES for the order."""
    _check(lib().moe_load_stats(ctypes.byref(desc), _ptr(counts), _ptr(stats), _stream(stream)), "moe_load_stats")


def moe_bias_state_size(desc, window_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_bias_state_size(ctypes.byref(desc), int(window_tokens), ctypes.byref(n)), "moe_bias_state_size")
    return int(n.value)


def moe_bias_state_init(state, stream=None):
    p, n = _ws(state)
    _check(lib().moe_bias_state_init(p, n, _stream(stream)), "moe_bias_state_init")


def moe_update_sel_bias(desc, topk_idx, window_tokens, gamma, state, sel_bias, window_counts=None, stream=None):
    p, n = _ws(state)
    _check(lib().moe_update_sel_bias(ctypes.byref(desc), _ptr(topk_idx), int(window_tokens), float(gamma), p, n,
                                     _ptr(sel_bias), _ptr(window_counts), _stream(stream)), "moe_update_sel_bias")


def moe_reroute(desc, topk_idx, topk_w, counts, row_of_slot, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_reroute(ctypes.byref(desc), _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(row_of_slot), p, n,
                             _stream(stream)), "moe_reroute")


def moe_quantize_rows_e4m3(x, q, s, stream=None):
    """Per-row E4M3 codes q [rows][d] (uint8) and scales s [rows] (fp32) of
    the bf16 rows x [rows][d]."""
    rows, d = int(x.shape[0]), int(x.shape[1])
    _check(lib().moe_quantize_rows_e4m3(_ptr(x), rows, d, _ptr(q), _ptr(s), _stream(stream)),
           "moe_quantize_rows_e4m3")


def moe_split_rows_e4m3(x, q, s, stream=None):
    """Two-term E4M3 codes q [rows][2d] (uint8: first terms, then second
    terms) and power-of-two scales s [rows] (fp32) of the bf16 rows x
    [rows][d]."""
    rows, d = int(x.shape[0]), int(x.shape[1])
    _check(lib().moe_split_rows_e4m3(_ptr(x), rows, d, _ptr(q), _ptr(s), _stream(stream)), "moe_split_rows_e4m3")


def moe_get_status(ws, stream=None):
    """(status code, flags, counters dict) of the workspace's status block."""
    flags = ctypes.c_uint32(0)
    cnt = (ctypes.c_int32 * MOE_NUM_COUNTERS)()
    code = lib().moe_get_status(_ptr(ws), _stream(stream), ctypes.byref(flags), cnt)
    if code not in (MOE_OK, MOE_ERR_DEVICE_STATUS):
        raise MoeError(code, "moe_get_status")
    return code, int(flags.value), {name: int(cnt[i]) for i, name in enumerate(COUNTER_NAMES)}

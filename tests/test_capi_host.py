"""Host-side checks of the C ABI: the library loads, exports every entry
point the header declares, sizes workspaces, and rejects bad arguments before
touching CUDA.  No GPU needed: none of these calls reaches a CUDA API."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_bias_b200 import build as B
from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    B.build()
    return ops.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = header_functions()
    assert len(names) >= 10
    lib = ops.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ops.EXPORTED)


def test_strerror():
    assert ops.strerror(0) == "ok"
    for code in range(1, 6):
        assert len(ops.strerror(code)) > 3
    assert ops.strerror(99) == "unknown status"


def _desc(name, **over):
    cfg = syn.CONFIGS[name] if name in syn.CONFIGS else syn.VARIANTS[name]
    return ops.make_desc(**dict(syn.desc_dict(cfg), **over))


@pytest.mark.parametrize("name", list(syn.CONFIGS))
def test_workspace_size_and_rows(name):
    cfg = syn.CONFIGS[name]
    d = _desc(name)
    R = ops.moe_routed_rows(d)
    if cfg.capacity:
        assert R == cfg.E * cfg.capacity + cfg.S * cfg.K
    else:
        assert R == cfg.S * cfg.K
    n = ops.moe_workspace_size(d)
    ab = 4 if cfg.act_dtype == 0 else 2
    Rt = R + cfg.num_shared * cfg.S
    # at least the permuted rows, hidden and expert outputs
    assert n >= (R * cfg.d + Rt * cfg.h + Rt * cfg.d) * ab
    assert n % 256 == 0


def test_capacity_value_of_skew_workload():
    cfg = syn.CONFIGS["fp8_skew_capacity"]
    assert cfg.capacity == syn.capacity_for(cfg.S, cfg.K, cfg.E) == 2560


BAD = [
    dict(top_k=0), dict(top_k=9), dict(num_experts=0), dict(num_experts=300), dict(d_model=100),
    dict(d_ff=0), dict(score_fn=5), dict(num_groups=3), dict(num_groups=2, topk_groups=3),
    dict(num_groups=4, topk_groups=1, top_k=3), dict(num_shared=2), dict(capacity=-1), dict(num_tokens=-1),
    dict(renormalize=2), dict(activation=7), dict(act_dtype=5), dict(act_quant=2), dict(act_quant=-1),
    dict(reroute=2), dict(reroute=1),  # re-routing needs a capacity (mixtral_prefill has none)
    dict(temperature=-0.5), dict(temperature=float("nan")), dict(temperature=float("inf")),
]


@pytest.mark.parametrize("over", BAD)
def test_invalid_desc_rejected(over):
    d = _desc("mixtral_prefill", **over)
    n = ctypes.c_size_t(0)
    assert ops.lib().moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == ops.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(act_dtype=0), dict(weight_dtype=0),
                                  dict(weight_dtype=2, activation=0),
                                  dict(act_quant=1),                                  # W8A8 needs E4M3 weights
                                  dict(act_quant=1, weight_dtype=2, d_model=4104),    # d not a multiple of 16
                                  dict(act_quant=1, weight_dtype=2, d_ff=14344),      # h not a multiple of 16
                                  dict(score_fn=1, temperature=0.5)])                 # temperature: softmax only
def test_unsupported_combination(over):
    d = _desc("mixtral_prefill", **over)
    n = ctypes.c_size_t(0)
    assert ops.lib().moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == ops.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("tau", [0.0, 1.0, 0.5, 2.0, 0.7])
def test_temperature_accepted(tau):
    n = ctypes.c_size_t(0)
    assert ops.lib().moe_workspace_size(ctypes.byref(_desc("mixtral_prefill", temperature=tau)),
                                        ctypes.byref(n)) == ops.MOE_OK
    # a sigmoid router takes only tau = 1 (or 0, its spelling)
    if tau in (0.0, 1.0):
        assert ops.lib().moe_workspace_size(ctypes.byref(_desc("dsv3_grouped", temperature=tau)),
                                            ctypes.byref(n)) == ops.MOE_OK


def test_group_size_must_be_power_of_two():
    d = _desc("dsv3_grouped", num_experts=96, num_groups=2)  # groups of 48
    n = ctypes.c_size_t(0)
    assert ops.lib().moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == ops.MOE_ERR_INVALID_ARG


def test_calls_reject_missing_workspace_and_pointers():
    L = ops.lib()
    d = _desc("tiny_f32")
    w = ops.MoeWeights()
    p = ctypes.c_void_p(0x1000)
    # no workspace
    assert L.moe_route(ctypes.byref(d), ctypes.byref(w), p, None, p, p, None, 0, None) == ops.MOE_ERR_WORKSPACE
    # workspace too small (pointer value only: nothing is dereferenced on the host)
    ws = ctypes.c_void_p(0x100000)
    assert L.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), p, p, None, None, None, ws, 256,
                               None) == ops.MOE_ERR_WORKSPACE
    # misaligned workspace
    n = ops.moe_workspace_size(d)
    assert L.moe_combine(ctypes.byref(d), p, p, p, p, ctypes.c_void_p(0x100010), n, None) == ops.MOE_ERR_WORKSPACE
    # missing outputs / weights
    assert L.moe_route(ctypes.byref(d), ctypes.byref(w), p, None, None, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(d), ctypes.byref(w), p, None, p, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), p, p, None, None, None, ws, n,
                               None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_permute(ctypes.byref(d), p, p, None, p, p, p, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    # x without x_perm
    assert L.moe_permute(ctypes.byref(d), p, p, p, p, p, p, None, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    # misaligned activations
    assert L.moe_combine(ctypes.byref(d), ctypes.c_void_p(0x1004), p, p, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_get_status(None, None, None, None) == ops.MOE_ERR_WORKSPACE
    assert L.moe_workspace_init(None, 0, None) == ops.MOE_ERR_WORKSPACE


def test_empty_batch_is_a_no_op():
    """S = 0 is valid: the calls return OK without launching anything."""
    L = ops.lib()
    d = _desc("tiny_f32", num_tokens=0)
    n = ops.moe_workspace_size(d)
    ws = ctypes.c_void_p(0x100000)
    w = ops.MoeWeights()
    p = ctypes.c_void_p(0x1000)
    assert L.moe_route(ctypes.byref(d), ctypes.byref(w), None, None, p, p, ws, n, None) == ops.MOE_OK
    assert L.moe_combine(ctypes.byref(d), p, p, p, p, ws, n, None) == ops.MOE_OK
    assert L.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, None, None, ws, n,
                               None) == ops.MOE_OK
    assert ops.moe_routed_rows(d) == 0


def test_bias_state_size_and_argument_errors():
    L = ops.lib()
    d = _desc("dsv3_grouped")
    n = ops.moe_bias_state_size(d, 1000)
    assert n >= 256 + 256 * 4 + 1000 * 8 * 4 and n % 256 == 0
    size = ctypes.c_size_t(0)
    assert L.moe_bias_state_size(ctypes.byref(d), 0, ctypes.byref(size)) == ops.MOE_ERR_INVALID_ARG
    p = ctypes.c_void_p(0x1000)
    st = ctypes.c_void_p(0x200000)
    # state missing / too small / misaligned
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, 0.1, None, n, p, None, None) == ops.MOE_ERR_WORKSPACE
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, 0.1, st, n - 256, p, None, None) == ops.MOE_ERR_WORKSPACE
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, 0.1, ctypes.c_void_p(0x200010), n, p, None,
                                 None) == ops.MOE_ERR_WORKSPACE
    # bias missing, negative or NaN step
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, 0.1, st, n, None, None, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, -0.1, st, n, p, None, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_update_sel_bias(ctypes.byref(d), p, 1000, float("nan"), st, n, p, None,
                                 None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_bias_state_init(None, 0, None) == ops.MOE_ERR_WORKSPACE


@pytest.mark.parametrize("name", [n for n, c in syn.VARIANTS.items() if c.act_quant])
def test_w8a8_workspace_holds_codes_and_scales(name):
    """W8A8 holds one E4M3 code per activation element and a scale per row;
    the same layer on bf16 activations holds two codes per element (two-term
    codes) and the same scales."""
    cfg = syn.VARIANTS[name]
    d8 = _desc(name)
    d16 = ops.make_desc(**dict(syn.desc_dict(cfg), act_quant=0))
    R = ops.moe_routed_rows(d8)
    Rt = R + cfg.num_shared * cfg.S
    n8, n16 = ops.moe_workspace_size(d8), ops.moe_workspace_size(d16)
    codes = R * cfg.d + Rt * cfg.h + (R + Rt) * 4
    assert n8 >= codes
    assert R * cfg.d + Rt * cfg.h <= n16 - n8 <= R * cfg.d + Rt * cfg.h + 8 * 4096


@pytest.mark.parametrize("name", ["moe_quantize_rows_e4m3", "moe_split_rows_e4m3"])
def test_quantize_rows_argument_errors(name):
    fn = getattr(ops.lib(), name)
    p = ctypes.c_void_p(0x1000)
    assert fn(p, 0, 32, p, p, None) == ops.MOE_OK       # nothing to do
    assert fn(p, -1, 32, p, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 24, p, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 0, p, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(None, 4, 32, p, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 32, None, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 32, p, None, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(ctypes.c_void_p(0x1008), 4, 32, p, p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 32, ctypes.c_void_p(0x1004), p, None) == ops.MOE_ERR_INVALID_ARG
    assert fn(p, 4, 32, p, ctypes.c_void_p(0x1002), None) == ops.MOE_ERR_INVALID_ARG


def test_reroute_workspace_and_argument_errors():
    L = ops.lib()
    d = _desc("fp8_skew_capacity_reroute")
    d0 = _desc("fp8_skew_capacity")
    cfg = syn.VARIANTS["fp8_skew_capacity_reroute"]
    # keys + gate sources of every expert, the excess list and the changed flags
    assert ops.moe_workspace_size(d) - ops.moe_workspace_size(d0) >= cfg.S * cfg.E * 8 + cfg.S * cfg.K * 4
    n = ops.moe_workspace_size(d)
    p = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)
    assert L.moe_reroute(ctypes.byref(d0), p, p, p, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG  # reroute = 0
    assert L.moe_reroute(ctypes.byref(d), None, p, p, p, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_reroute(ctypes.byref(d), p, p, p, None, ws, n, None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_reroute(ctypes.byref(d), p, p, p, p, ws, n - 256, None) == ops.MOE_ERR_WORKSPACE
    assert L.moe_reroute(ctypes.byref(d), p, p, p, p, None, n, None) == ops.MOE_ERR_WORKSPACE


def test_header_is_plain_c(tmp_path):
    """include/moe.h is a C header: a C99 translation unit that includes it and
    takes the address of every entry point compiles without warnings."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = header_functions()
    src = tmp_path / "use_header.c"
    body = "\n".join(f"  p[{i}] = (fn)&{n};" for i, n in enumerate(names))
    src.write_text('#include "moe.h"\ntypedef void (*fn)(void);\nvoid touch(fn *p) {\n' + body + '\n}\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-c", str(src), "-I",
                        os.path.join(ROOT, "include"), "-o", str(tmp_path / "use_header.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_argument_counts_match_the_header():
    """Every ctypes prototype in ops.py has as many arguments as the C
    prototype in include/moe.h."""
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = dict(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S))
    L = ops.lib()
    assert set(protos) == set(ops.EXPORTED)
    for name, args in protos.items():
        args = args.strip()
        n = 0 if args in ("", "void") else args.count(",") + 1
        assert len(getattr(L, name).argtypes) == n, name


def _struct_fields(text, name):
    bodies = dict((n, b) for b, n in re.findall(r"typedef struct \{([^{}]*)\}\s*(\w+)\s*;", text))
    body = bodies[name]
    return [m.group(1) for m in re.finditer(r"\**\s*([a-z_0-9]+)\s*;", body)]


def test_struct_layouts_match_the_header():
    """moe_desc and moe_weights as ctypes structures list the header's fields
    in the header's order with the header's member types (int32 and float
    members of the descriptor, pointers of the weights)."""
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moe.h")).read(), flags=re.S)
    assert _struct_fields(text, "moe_desc") == list(ops.DESC_FIELDS)
    assert _struct_fields(text, "moe_weights") == list(ops.WEIGHT_FIELDS)
    body = dict((n, b) for b, n in re.findall(r"typedef struct \{([^{}]*)\}\s*(\w+)\s*;", text))["moe_desc"]
    types = dict((m.group(2), m.group(1)) for m in re.finditer(r"(int32_t|float)\s+([a-z_0-9]+)\s*;", body))
    for name, ctype in ops.MoeDesc._fields_:
        assert types[name] == ("float" if ctype is ctypes.c_float else "int32_t"), name
    assert ctypes.sizeof(ops.MoeDesc) == 4 * len(ops.DESC_FIELDS)
    assert ctypes.sizeof(ops.MoeWeights) == 8 * len(ops.WEIGHT_FIELDS)


def test_product_path_never_touches_the_oracle():
    """The library and its binding import, read and call nothing under
    oracle/ (only tests, the smoke check and the benchmark's CPU legs may)."""
    pkg = os.path.join(ROOT, "mixture_experts_layer_bias_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                where = os.path.join(dirpath, f)
                assert "moe_oracle" not in text and "oracle/" not in text, where
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), where


def test_missing_library_fails_loudly():
    """No CPU fallback: without the built library the first call raises."""
    import subprocess
    import sys
    missing = os.path.join(ROOT, "no_such_library.so")
    code = ("from mixture_experts_layer_bias_b200 import ops\n"
            f"ops._LIB_PATH = {missing!r}\n"
            "try:\n    ops.lib()\nexcept RuntimeError as e:\n    print('raised', e)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert "raised" in r.stdout, (r.stdout, r.stderr)


def test_e4m3_workspace_two_term_codes_instead_of_decoded_weights():
    """E4M3 weights with bf16 activations: the GEMMs read the stored weight
    codes, so the workspace holds no bf16 copy of the weights.  The token
    rows' two-term codes (2 bytes per element) take the place of the bf16
    copy of the permuted rows, and the hidden rows get their codes beside the
    bf16 hidden rows, with one fp32 scale per row.  With d or h not a
    multiple of 16 the layer decodes the weights into the workspace first."""
    size = lambda c: ops.moe_workspace_size(ops.make_desc(**syn.desc_dict(c)))
    for S in (64, 8192, 16384):
        c8 = syn.scaled(syn.CONFIGS["fp8_skew_capacity"], S=S)
        c16 = syn.scaled(c8, weight_dtype=syn.BF16)
        R = ops.moe_routed_rows(ops.make_desc(**syn.desc_dict(c8)))
        extra = 2 * R * c8.h + 4 * 2 * R                                  # hidden codes, scales
        assert extra <= size(c8) - size(c16) <= extra + 8 * 4096, S       # alignment slack only
    c8 = syn.scaled(syn.CONFIGS["fp8_skew_capacity"], S=1024)
    odd8 = syn.scaled(c8, d=2056)
    odd16 = syn.scaled(c8, d=2056, weight_dtype=syn.BF16)
    n_dec = 3 * (odd8.E + odd8.num_shared) * odd8.h * odd8.d * 2
    assert size(odd8) - size(odd16) >= n_dec

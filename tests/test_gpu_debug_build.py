"""The guard build (libmoe_b200_debug.so, compiled with MOE_DEBUG).

It checks the permutation's invariants after every permutation and the range
of every row the combine reads.  On valid inputs it must agree with the oracle
and leave the status block clean; a combine given a row beyond the permuted
buffer must report MOE_STATUS_DEBUG_CHECK and skip that row (the check comes
before the read, so nothing outside the buffer is touched).  The guard build
is loaded in a child process of its own.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np
import torch
from mixture_experts_layer_bias_b200 import ops, synthetic as syn
from mixture_experts_layer_bias_b200.build import DEBUG_LIB
ops._LIB_PATH = DEBUG_LIB
from parity import run_layer, compare_layer, new_ws
res = {{}}
cases = {{
    "decode": syn.scaled(syn.CONFIGS["mixtral_decode"], S=4, d=512, h=512),
    "prefill": syn.scaled(syn.CONFIGS["mixtral_prefill"], S=300, d=256, h=256),
    "capacity": syn.scaled(syn.CONFIGS["fp8_skew_capacity"], S=700, d=256, h=128),
    "grouped": syn.scaled(syn.CONFIGS["dsv3_grouped"], S=96, d=256, h=128),
}}
for name, cfg in cases.items():
    inp = syn.make_inputs(cfg, "cuda", seed=3)
    gpu = run_layer(inp, cfg)
    rep = compare_layer(gpu, inp, cfg)
    code, flags, cnt = ops.moe_get_status(gpu["ws"])
    res[name] = dict(ok=rep["ok"], code=code, flags=flags)
# combine with one row beyond the permuted rows
cfg = syn.scaled(syn.CONFIGS["mixtral_prefill"], S=8, d=256, h=256)
desc = ops.make_desc(**syn.desc_dict(cfg))
R = ops.moe_routed_rows(desc)
ws = new_ws(desc)
y_perm = torch.randn((R, cfg.d), device="cuda").to(torch.bfloat16)
ros = torch.arange(cfg.S * cfg.K, dtype=torch.int32, device="cuda")
ros[5] = R + 7
gw = torch.full((cfg.S, cfg.K), 0.5, dtype=torch.float32, device="cuda")
y = torch.empty((cfg.S, cfg.d), dtype=torch.bfloat16, device="cuda")
ops.moe_combine(desc, y_perm, ros, gw, y, ws)
torch.cuda.synchronize()
code, flags, cnt = ops.moe_get_status(ws)
yp = y_perm.float().cpu().numpy()
ref = np.zeros((cfg.S, cfg.d))
for t in range(cfg.S):
    for k in range(cfg.K):
        s = t * cfg.K + k
        if s != 5:
            ref[t] += 0.5 * yp[s]
err = float(np.abs(y.float().cpu().numpy() - ref).max() / np.abs(ref).max())
res["bad_row"] = dict(code=code, flags=flags, rel_err=err)
print("RESULT " + json.dumps(res))
"""


def test_guard_build_agrees_and_reports():
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    for name in ("decode", "prefill", "capacity", "grouped"):
        assert res[name]["ok"], (name, res[name])
        assert res[name]["flags"] == 0 and res[name]["code"] == 0, (name, res[name])
    bad = res["bad_row"]
    assert bad["flags"] & 0x10, bad            # MOE_STATUS_DEBUG_CHECK
    assert bad["code"] == 5, bad               # MOE_ERR_DEVICE_STATUS
    assert bad["rel_err"] < 1e-2, bad          # the bad row skipped, the others summed

"""Failure detection on the GPU without a GPU fault.

Every wait inside the tensor-core GEMM is bounded in time.  A test hook,
present only in the test build of the library (libmoe_b200_testhooks.so,
moe_test_stall_gemms(1)), makes the next GEMM launch run with a producer that
never delivers a tile -- a flag nothing sets -- so the MMA warp's wait must
give up, raise MOE_STATUS_TIMEOUT in the status block and let the kernel
exit.  The host reads the status, and the same CUDA context must then run a
correct layer.  The test build is loaded in a child process of its own.
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
import torch
from mixture_experts_layer_bias_b200 import ops, synthetic as syn
from mixture_experts_layer_bias_b200.build import TEST_HOOKS_LIB
ops._LIB_PATH = TEST_HOOKS_LIB
ops.lib().moe_test_stall_gemms(1)
from parity import run_layer, compare_layer
if {e4m3!r}:   # E4M3 weights: the f8f6f4 kernel with two activation terms per stage
    cfg = syn.scaled(syn.VARIANTS["mixtral_decode_e4m3"], S=4, d=256, h=384)
else:
    cfg = syn.scaled(syn.CONFIGS["mixtral_prefill"], S=64, d=256, h=256)
inp = syn.make_inputs(cfg, "cuda", seed=0)
first = run_layer(inp, cfg)                     # its first GEMM launch stalls
code1, flags1, cnt1 = ops.moe_get_status(first["ws"])
second = run_layer(inp, cfg)                    # the hook is spent: a normal layer
rep = compare_layer(second, inp, cfg)
code2, flags2, cnt2 = ops.moe_get_status(second["ws"])
err = torch.cuda.synchronize() or "ok"
print("RESULT " + json.dumps(dict(code1=code1, flags1=flags1, timeouts=cnt1["timeout"], code2=code2,
                                  flags2=flags2, ok=rep["ok"], err=err)))
"""


@pytest.mark.parametrize("e4m3", [False, True])
def test_bounded_wait_gives_up_and_context_survives(e4m3):
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), e4m3=e4m3)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["flags1"] & 0x4, res          # MOE_STATUS_TIMEOUT
    assert res["timeouts"] > 0, res
    assert res["code1"] == 5, res            # MOE_ERR_DEVICE_STATUS
    assert res["flags2"] == 0 and res["code2"] == 0, res
    assert res["ok"], res

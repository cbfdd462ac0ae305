"""Sliding-window load and selection-bias update (aux-loss-free routing,
ybb.press 2.3) on the GPU against the oracle: window counts and the float32
bias must match bit for bit over a sequence of batches (partial fill, wrap
around the ring, a batch longer than the window, ids outside [0, E))."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _desc(S, E, K):
    return ops.make_desc(num_tokens=S, d_model=64, num_experts=E, top_k=K, d_ff=64)


@pytest.mark.parametrize("E,K,W", [(64, 8, 1000), (8, 2, 37), (256, 8, 64)])
def test_bias_update_matches_oracle(E, K, W):
    rng = np.random.default_rng(E + K + W)
    state = torch.empty(ops.moe_bias_state_size(_desc(1, E, K), W), dtype=torch.uint8, device="cuda")
    ops.moe_bias_state_init(state)
    bias_gpu = torch.zeros(E, dtype=torch.float32, device="cuda")
    counts_gpu = torch.empty(E, dtype=torch.int32, device="cuda")
    ref = O.WindowBias(E, K, W)
    bias_ref = np.zeros(E, np.float32)
    offs = rng.normal(size=E) * 1.2
    for S in (3, W // 2, 1, W - 1, 2 * W + 5, 7, W, 5):
        logits = (rng.normal(size=(S, E)) + offs).astype(np.float32)
        idx, _ = O.select_experts(logits, K)
        if S == 7:
            idx[0, 0] = E + 3  # not counted
            idx[1, 1] = -2
        ops.moe_update_sel_bias(_desc(S, E, K), torch.tensor(idx, dtype=torch.int32, device="cuda"), W, 0.0125,
                                state, bias_gpu, counts_gpu)
        bias_ref, c_ref = ref.update(idx, bias_ref, 0.0125)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(counts_gpu.cpu().numpy(), c_ref)
        np.testing.assert_array_equal(bias_gpu.cpu().numpy(), bias_ref)


def test_bias_update_steers_gpu_routing():
    """GPU routing with the GPU-updated selection bias evens out a skewed load."""
    rng = np.random.default_rng(3)
    E, K, S, W = 16, 2, 512, 1000
    offs = (rng.normal(size=E) * 1.5).astype(np.float32)
    d = _desc(S, E, K)
    ws = torch.empty(ops.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    ops.moe_workspace_init(ws)
    state = torch.empty(ops.moe_bias_state_size(d, W), dtype=torch.uint8, device="cuda")
    ops.moe_bias_state_init(state)
    bias = torch.zeros(E, dtype=torch.float32, device="cuda")
    idx = torch.empty((S, K), dtype=torch.int32, device="cuda")
    gw = torch.empty((S, K), dtype=torch.float32, device="cuda")
    ratios = []
    for _ in range(60):
        logits = torch.tensor((rng.normal(size=(S, E)) + offs).astype(np.float32), device="cuda")
        ops.moe_route(d, ops.make_weights({"sel_bias": bias}), None, logits, idx, gw, ws)
        counts = torch.bincount(idx.reshape(-1).long(), minlength=E).cpu().numpy()
        ratios.append(O.load_stats(counts, K, S)["max_over_mean"])
        ops.moe_update_sel_bias(d, idx, W, 0.05, state, bias)
    assert ratios[0] > 2.0 and np.mean(ratios[-10:]) < 0.6 * ratios[0], ratios

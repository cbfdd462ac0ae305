"""moe_permute_static: the workspace-free permutation for callers that cannot
allocate device memory (fixed memory budgets, allocator callbacks, loops that
must avoid cudaFree's synchronisation).

It must give exactly what moe_permute gives (integer maps and gathered rows,
compared bit for bit, the bar of every permutation test here), on two calls
in a row -- the second smaller than the first, so stale scratch from the
first call would show.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _inputs(S, E, K, cap, seed):
    rng = np.random.default_rng(seed)
    logits = (rng.normal(size=(S, E)) + 2.0 * rng.normal(size=E)[None, :]).astype(np.float32)
    ridx, _ = O.select_experts(logits, K)
    desc = ops.make_desc(num_tokens=S, d_model=256, num_experts=E, top_k=K, d_ff=64, capacity=cap)
    x = torch.randn((S, 256), device="cuda").to(torch.bfloat16)
    return desc, x, torch.tensor(ridx, dtype=torch.int32, device="cuda")


def _outputs(desc):
    S, E, K = desc.num_tokens, desc.num_experts, desc.top_k
    R = ops.moe_routed_rows(desc)
    return dict(counts=torch.full((E,), -3, dtype=torch.int32, device="cuda"),
                offsets=torch.full((2 * (E + 1),), -3, dtype=torch.int32, device="cuda"),
                ros=torch.full((S * K,), -3, dtype=torch.int32, device="cuda"),
                tor=torch.full((R,), -3, dtype=torch.int32, device="cuda"),
                xp=torch.zeros((R, desc.d_model), dtype=torch.bfloat16, device="cuda"))


def test_permute_static_matches_permute_on_two_calls():
    cases = [(6000, 64, 8, 0, 1), (1500, 16, 4, syn.capacity_for(1500, 4, 16), 2)]
    for S, E, K, cap, seed in cases:
        desc, x, idx = _inputs(S, E, K, cap, seed)
        ref = _outputs(desc)
        ws = torch.empty(ops.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
        ops.moe_workspace_init(ws)
        ops.moe_permute(desc, x, idx, ref["counts"], ref["offsets"], ref["ros"], ref["tor"], ref["xp"], ws)
        got = _outputs(desc)
        ops.moe_permute_static(desc, x, idx, got["counts"], got["offsets"], got["ros"], got["tor"], got["xp"])
        torch.cuda.synchronize()
        n_off = 2 * (E + 1) if cap else E + 1
        assert torch.equal(got["counts"], ref["counts"])
        assert torch.equal(got["offsets"][:n_off], ref["offsets"][:n_off])
        assert torch.equal(got["ros"], ref["ros"])
        assert torch.equal(got["tor"], ref["tor"])
        used = ref["tor"] >= 0
        assert torch.equal(got["xp"][used], ref["xp"][used])


def test_permute_static_rejects_sizes_beyond_its_scratch():
    # 256 experts x ceil(S / 128) chunks > 65536 entries once S > 32768 tokens at K = 8
    desc = ops.make_desc(num_tokens=40000, d_model=256, num_experts=256, top_k=8, d_ff=64)
    t = torch.empty(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.MoeError) as e:
        ops.moe_permute_static(desc, None, t, t, t, t, t, None)
    assert e.value.code == ops.MOE_ERR_WORKSPACE

"""moe_permute_static: the workspace-free permutation, for callers that cannot
allocate device memory (a runtime whose device-memory budget is fixed at
start-up, code running inside an allocator or other callback where a nested
cudaMalloc/cudaFree is not allowed, a loop that must not risk the device-wide
synchronisation cudaFree can cause).

Its maps must equal the oracle's expert_permutation (bit for bit, the bar of
every permutation test here), its gathered rows must be bit copies of the
token rows, and it must give exactly what moe_permute gives -- on two calls
in a row, the second smaller than the first, so stale scratch from the first
call would show.  The cases cover the chunked path (S*K > 4096), the one-CTA
path of small batches (S*K <= 4096), capacity with overflow rows, and the
maps-only form (x = NULL).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_bias_b200 import ops
from mixture_experts_layer_bias_b200 import synthetic as syn
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

D = 256


def _case(S, E, K, cap, seed):
    rng = np.random.default_rng(seed)
    logits = (rng.normal(size=(S, E)) + 2.0 * rng.normal(size=E)[None, :]).astype(np.float32)
    ridx, _ = O.select_experts(logits, K)
    desc = ops.make_desc(num_tokens=S, d_model=D, num_experts=E, top_k=K, d_ff=64, capacity=cap)
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((S, D), device="cuda", generator=g).to(torch.bfloat16)
    return desc, ridx, x, torch.tensor(ridx, dtype=torch.int32, device="cuda")


def _outputs(desc):
    S, E, K = desc.num_tokens, desc.num_experts, desc.top_k
    R = ops.moe_routed_rows(desc)
    return dict(counts=torch.full((E,), -3, dtype=torch.int32, device="cuda"),
                offsets=torch.full((2 * (E + 1),), -3, dtype=torch.int32, device="cuda"),
                ros=torch.full((S * K,), -3, dtype=torch.int32, device="cuda"),
                tor=torch.full((R,), -3, dtype=torch.int32, device="cuda"),
                xp=torch.zeros((R, desc.d_model), dtype=torch.bfloat16, device="cuda"))


def _static(desc, x, idx, out, with_rows=True):
    ops.moe_permute_static(desc, x if with_rows else None, idx, out["counts"], out["offsets"], out["ros"],
                           out["tor"], out["xp"] if with_rows else None)


def _check_against_oracle(desc, ridx, x, out, with_rows=True):
    E, cap = desc.num_experts, desc.capacity
    P = O.expert_permutation(ridx, E, cap)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), P["counts"])
    offs = out["offsets"].cpu().numpy()
    np.testing.assert_array_equal(offs[: E + 1], P["offsets"])
    if cap:
        np.testing.assert_array_equal(offs[E + 1:], P["ovf_offsets"])
    np.testing.assert_array_equal(out["ros"].cpu().numpy(), P["row_of_slot"])
    np.testing.assert_array_equal(out["tor"].cpu().numpy(), P["token_of_row"])
    if with_rows:
        used = np.nonzero(P["token_of_row"] >= 0)[0]
        src = torch.tensor(P["token_of_row"][used], device="cuda", dtype=torch.long)
        assert torch.equal(out["xp"][torch.tensor(used, device="cuda")], x[src])
    return P


# (S, E, K, capacity, seed, gather rows): chunked path, capacity + overflow,
# small-batch one-CTA path, maps only
CASES = [(6000, 64, 8, 0, 1, True), (1500, 16, 4, syn.capacity_for(1500, 4, 16), 2, True),
         (700, 8, 2, 0, 3, True), (300, 32, 4, syn.capacity_for(300, 4, 32), 4, False)]


@pytest.mark.parametrize("first,second", [(0, 1), (1, 2), (0, 3)])
def test_permute_static_matches_oracle_and_permute_on_two_calls(first, second):
    for ci in (first, second):  # two calls in a row, the second smaller
        S, E, K, cap, seed, rows = CASES[ci]
        desc, ridx, x, idx = _case(S, E, K, cap, seed)
        got = _outputs(desc)
        _static(desc, x, idx, got, rows)
        torch.cuda.synchronize()
        P = _check_against_oracle(desc, ridx, x, got, rows)
        # and exactly what moe_permute (with a workspace) gives
        ref = _outputs(desc)
        ws = torch.empty(ops.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
        ops.moe_workspace_init(ws)
        ops.moe_permute(desc, x if rows else None, idx, ref["counts"], ref["offsets"], ref["ros"], ref["tor"],
                        ref["xp"] if rows else None, ws)
        torch.cuda.synchronize()
        n_off = 2 * (E + 1) if cap else E + 1
        assert torch.equal(got["counts"], ref["counts"])
        assert torch.equal(got["offsets"][:n_off], ref["offsets"][:n_off])
        assert torch.equal(got["ros"], ref["ros"])
        assert torch.equal(got["tor"], ref["tor"])
        if rows:
            used = torch.tensor(P["token_of_row"] >= 0, device="cuda")
            assert torch.equal(got["xp"][used], ref["xp"][used])


def test_permute_static_allocates_nothing():
    """After the kernels have been loaded once, further calls change neither
    torch's allocator nor the device's free memory."""
    prepared = []
    for ci in (0, 2):
        S, E, K, cap, seed, rows = CASES[ci]
        desc, ridx, x, idx = _case(S, E, K, cap, seed)
        out = _outputs(desc)
        _static(desc, x, idx, out, rows)  # first call on this device: loads kernels, looks up the scratch
        prepared.append((desc, ridx, x, idx, out, rows))
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for desc, ridx, x, idx, out, rows in prepared:
        for v in out.values():
            v.fill_(-3)
        _static(desc, x, idx, out, rows)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    for desc, ridx, x, idx, out, rows in prepared:
        _check_against_oracle(desc, ridx, x, out, rows)


def test_permute_static_rejects_sizes_beyond_its_scratch():
    # 256 experts x ceil(S / 128) chunks > 65536 entries once S > 32768 tokens at K = 8
    desc = ops.make_desc(num_tokens=40000, d_model=256, num_experts=256, top_k=8, d_ff=64)
    t = torch.empty(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.MoeError) as e:
        ops.moe_permute_static(desc, None, t, t, t, t, t, None)
    assert e.value.code == ops.MOE_ERR_WORKSPACE

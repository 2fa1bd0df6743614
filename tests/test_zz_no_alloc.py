"""The allocation-free permute entry point (moe_permute_static_ws), through the C-ABI on a GPU.

It serves callers that cannot supply device scratch memory (a fixed interface without a workspace
argument and no allocator of their own, or no cudaMalloc allowed at run time). It must give exactly
what moe_permute gives with a caller-provided workspace, call after call, since every call reuses the
library's one static scratch array. This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _inputs(T, d, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    x = synth.normal_bf16(seed, 0, 0, T * d, 1.0)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(T, d).cuda()
    return xd, torch.from_numpy(idx).cuda()


def _outputs(T, d, E, k):
    R = T * k
    return dict(counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
                perm_src=torch.full((R,), -7, dtype=torch.int32, device="cuda"),
                inv_perm=torch.full((R,), -7, dtype=torch.int32, device="cuda"),
                x_perm=torch.zeros(R, d, dtype=torch.bfloat16, device="cuda"))


def test_static_scratch_permute_matches_workspace_permute_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mixture_experts_ffn_11_b200 import _native as N

    N.get_device_error()
    # two calls in a row with different shapes; the second reuses the scratch the first left behind
    for T, d, E, k, seed in ((4096, 64, 32, 4, 11), (9000, 32, 128, 8, 12)):
        x, idx = _inputs(T, d, E, k, seed)
        ref = _outputs(T, d, E, k)
        ws = torch.empty(N.permute_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
        N.permute(x, idx, E, ref["counts"], ref["offsets"], ref["perm_src"], ref["inv_perm"], ref["x_perm"], ws)
        got = _outputs(T, d, E, k)
        N.permute_static_ws(x, idx, E, got["counts"], got["offsets"], got["perm_src"], got["inv_perm"],
                            got["x_perm"])
        torch.cuda.synchronize()
        assert N.get_device_error() == 0
        for name in ("counts", "offsets", "perm_src", "inv_perm"):
            assert torch.equal(got[name], ref[name]), name  # integer results: bit for bit
        assert torch.equal(got["x_perm"].view(torch.int16), ref["x_perm"].view(torch.int16))
        # and directly against the oracle's stable grouping
        want = oracle.permute(idx.cpu().numpy(), E)
        for name, w in zip(("counts", "offsets", "perm_src", "inv_perm"), want):
            assert (got[name].cpu().numpy() == w).all(), f"{name} differs from the oracle"
        xs = x.view(torch.int16).cpu().numpy()
        assert (got["x_perm"].view(torch.int16).cpu().numpy() == xs[want[2]]).all()


def test_static_scratch_permute_at_its_exact_limit():
    """E = 1024 and T*k = 262,144 need exactly the 1 MiB array: accepted and identical to moe_permute; one
    more 1024-assignment block is rejected before any launch."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mixture_experts_ffn_11_b200 import _native as N

    N.get_device_error()
    T, d, E, k = 32_768, 16, 1024, 8
    assert N.permute_workspace_size(T, E, k) == N.PERMUTE_STATIC_WS_BYTES
    x, idx = _inputs(T, d, E, k, 13)
    ref = _outputs(T, d, E, k)
    ws = torch.empty(N.permute_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    N.permute(x, idx, E, ref["counts"], ref["offsets"], ref["perm_src"], ref["inv_perm"], ref["x_perm"], ws)
    got = _outputs(T, d, E, k)
    N.permute_static_ws(x, idx, E, got["counts"], got["offsets"], got["perm_src"], got["inv_perm"], got["x_perm"])
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    for name in ("counts", "offsets", "perm_src", "inv_perm", "x_perm"):
        a, b = got[name], ref[name]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), name
    T2 = T + 128  # 1024 more assignments: 257 blocks
    assert N.permute_workspace_size(T2, E, k) > N.PERMUTE_STATIC_WS_BYTES
    idx2 = torch.zeros(T2, k, dtype=torch.int32, device="cuda")
    out = _outputs(T2, 8, E, k)
    with pytest.raises(N.MoEError) as err:
        N.permute_static_ws(None, idx2, E, out["counts"], out["offsets"], out["perm_src"], out["inv_perm"], None)
    assert err.value.status == N.MOE_ERR_WORKSPACE
    assert (out["counts"] == -7).all()


def test_static_scratch_permute_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mixture_experts_ffn_11_b200 import _native as N

    T, E, k = 70_000, 1024, 4  # 280,000 assignments: 274 blocks of 1024 x 1024 experts x 4 B > 1 MiB
    assert N.permute_workspace_size(T, E, k) > N.PERMUTE_STATIC_WS_BYTES
    idx = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    out = _outputs(T, 8, E, k)
    with pytest.raises(N.MoEError) as err:
        N.permute_static_ws(None, idx, E, out["counts"], out["offsets"], out["perm_src"], out["inv_perm"], None)
    assert err.value.status == N.MOE_ERR_WORKSPACE
    assert (out["counts"] == -7).all()  # nothing was launched

"""The grouped GEMMs' failure path on a B200: a pipeline wait that never ends must end the kernel cleanly.

Every wait inside the GEMM kernels is bounded. The test hook moe_test_set_wait shortens the limit to 1 ms and
makes the MMA-issuing warp wait on a barrier that nothing arrives on (no fault, no trap, no endless loop): the
kernel must return, report MOE_DEVERR_WAIT_TIMEOUT in the device error word, and leave the context usable, so that
the next, normal call matches the oracle and leaves the error word clear. Both the single-CTA kernel and the CTA
pair kernels (whose two CTAs must leave together) are covered.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_host_f32, check_close, to_dev_bf16

pytestmark = pytest.mark.gpu

N = pytest.importorskip("mixture_experts_ffn_11_b200._native")

COUNTS, D, F = [300, 0, 129, 45, 7], 256, 136


@pytest.fixture(scope="module")
def problem():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    torch.cuda.set_device(0)
    N.get_device_error()
    rng = np.random.default_rng(6)
    E = len(COUNTS)
    idx = np.concatenate([np.full(c, e) for e, c in enumerate(COUNTS)]).astype(np.int32)
    rng.shuffle(idx)
    idx = idx.reshape(-1, 1)
    T = idx.shape[0]
    x = synth.normal_bf16(11, 0, 0, T * D, 1.0).reshape(T, D)
    gu = synth.normal_bf16(11, 2, 0, E * 2 * F * D, 0.05).reshape(E, 2 * F, D)
    dn = synth.normal_bf16(11, 3, 0, E * D * F, 0.05).reshape(E, D, F)
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, np.ones((T, 1)), np.arange(T))
    R = T
    p = dict(counts=torch.empty(E, dtype=torch.int32, device="cuda"),
             offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
             perm_src=torch.empty(R, dtype=torch.int32, device="cuda"),
             inv_perm=torch.empty(R, dtype=torch.int32, device="cuda"),
             x_perm=torch.empty(R, D, dtype=torch.bfloat16, device="cuda"),
             ws=torch.empty(max(N.permute_workspace_size(T, E, 1), 256), dtype=torch.uint8, device="cuda"))
    N.permute(to_dev_bf16(x), torch.from_numpy(idx).cuda(), E, p["counts"], p["offsets"], p["perm_src"],
              p["inv_perm"], p["x_perm"], p["ws"])
    p.update(gu=to_dev_bf16(gu), dn=to_dev_bf16(dn), T=T, ref=ref)
    yield p
    N.test_set_wait(0, False)
    N.set_gemm_kernel("auto")


def _layer(p, h, y_perm):
    N.grouped_gemm_gateup(p["x_perm"], p["gu"], p["offsets"], h)
    N.grouped_gemm_down(h, p["dn"], p["offsets"], y_perm)


@pytest.mark.parametrize("family", ["single", "pair", "wide", "swap"])
def test_wait_timeout_ends_kernel_and_context_stays_usable(problem, family):
    p = problem
    T = p["T"]
    h = torch.zeros(T, F, dtype=torch.bfloat16, device="cuda")
    y_perm = torch.zeros(T, D, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    with N.gemm_kernel(family):
        N.test_set_wait(1_000_000, stall=True)
        try:
            _layer(p, h, y_perm)  # both launches return: their waits give up after 1 ms
            err = N.get_device_error()  # synchronises
        finally:
            N.test_set_wait(0, stall=False)
        assert err & 0x1, f"{family}: timeout not reported (error word {err:#x})"
        assert N.get_device_error() == 0  # read-and-clear
        # the context is usable and the next call is right
        _layer(p, h, y_perm)
        N.unpermute_combine(y_perm, p["inv_perm"], torch.ones(T, 1, dtype=torch.float32, device="cuda"), None, y)
        torch.cuda.synchronize()
    assert N.get_device_error() == 0
    check_close(bf16_to_host_f32(y), p["ref"], f"after timeout ({family})")

"""MoEFFN's host-side decisions on the CPU, without a device: when the shared expert is folded into the routed MXFP4
GEMMs, and how many kernels one forward() launches (the count the bench reports as gpu_launches; the launch lists
in profiles/ were taken from the same shapes)."""
import pytest

import synth


@pytest.fixture(scope="module")
def MoEFFN():
    from mixture_experts_ffn_11_b200 import MoEFFN as cls

    return cls


def _host_layer(cls, wl, fused=False):
    """A layer object with the attributes the host logic reads, built without allocating device weights."""
    lay = object.__new__(cls)
    lay.E, lay.d, lay.f, lay.k = wl.E, wl.d, wl.f, wl.k
    lay.weights, lay.fused, lay.shared_f = wl.weights, fused, wl.shared_f
    lay.fold_shared = wl.weights == "mxfp4" and wl.shared_f == wl.f and wl.shared_f > 0
    return lay


def test_decode_mxfp4_folds_the_shared_expert(MoEFFN):
    wl = synth.workload("decode-256e-shared-mxfp4")
    lay = _host_layer(MoEFFN, wl)
    assert lay._fold(wl.T)  # R + T = 576 rows, at most 8 per group over E + 1 = 257 groups
    # router logits + top-k (E > 128), 4 permute kernels, gate|up, down, combine, and the copy of the shared rows
    assert lay.kernel_launches(wl.T) == 2 + 4 + 3 + 1


def test_fold_stops_where_the_routed_experts_would_leave_the_decode_kernel(MoEFFN):
    wl = synth.workload("decode-256e-shared-mxfp4")
    lay = _host_layer(MoEFFN, wl)
    E, k = wl.E, wl.k
    t_max = 8 * (E + 1) // (k + 1)  # T (k + 1) <= 8 (E + 1)
    assert lay._fold(t_max) and not lay._fold(t_max + 1)
    assert not lay._fold(0)
    # unfolded: the shared expert's own gate|up and down
    assert lay.kernel_launches(t_max + 1) == 2 + 4 + 3 + 2


def test_no_fold_past_the_group_limit(MoEFFN):
    from mixture_experts_ffn_11_b200 import _native as N

    wl = synth.Workload(**{**synth.workload("decode-256e-shared-mxfp4").__dict__, "E": N.MAX_GEMM_GROUPS})
    assert not _host_layer(MoEFFN, wl)._fold(64)  # E + 1 groups would pass the grouped GEMMs' limit
    wl = synth.Workload(**{**wl.__dict__, "E": N.MAX_GEMM_GROUPS - 1})
    assert _host_layer(MoEFFN, wl)._fold(64)


def test_bf16_and_narrower_shared_experts_are_not_folded(MoEFFN):
    bf = _host_layer(MoEFFN, synth.workload("decode-256e-shared"))
    assert not bf.fold_shared and not bf._fold(64)
    assert bf.kernel_launches(64) == 2 + 4 + 3 + 2
    narrow = synth.Workload(**{**synth.workload("decode-256e-shared-mxfp4").__dict__, "shared_f": 1024})
    assert not _host_layer(MoEFFN, narrow)._fold(64)


def test_prefill_launch_counts(MoEFFN):
    wl = synth.workload("gpt-oss-20b-prefill")
    lay = _host_layer(MoEFFN, wl)
    # tensor-core router with fused top-k (E <= 128, T >= 2048), 4 permute kernels, gate|up, down, combine
    assert lay.kernel_launches(wl.T) == 1 + 4 + 3
    # a training forward keeps the pre-activations in the same gate|up launch at >= 128 rows per expert
    assert lay.kernel_launches(wl.T, train=True) == 1 + 4 + 3
    assert lay.kernel_launches(0) == 0

"""The C-ABI library on the CPU: it loads, exports every entry point include/moe.h declares, and rejects
bad arguments before touching a device (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def native():
    from mixture_experts_ffn_11_b200 import _native

    return _native


def test_header_declares_the_five_calls():
    fns = _header_functions()
    for name in ("moe_route_topk", "moe_permute", "moe_grouped_gemm_gateup", "moe_grouped_gemm_down",
                 "moe_unpermute_combine"):
        assert name in fns


def test_every_declared_symbol_is_exported(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in _header_functions():
        assert hasattr(lib, name), name
    assert set(_header_functions()) == set(native.EXPORTS)


def test_static_scratch_size_matches_header(native):
    """The binding's copy of MOE_PERMUTE_STATIC_WS_BYTES is the header's value, and the array holds exactly
    the workspace of 262,144 assignments over 1024 experts (256 segments x 1024 experts x 4 B)."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    m = re.search(r"#define\s+MOE_PERMUTE_STATIC_WS_BYTES\s+\(1u\s*<<\s*(\d+)\)", src)
    assert m, "MOE_PERMUTE_STATIC_WS_BYTES not found in include/moe.h"
    assert native.PERMUTE_STATIC_WS_BYTES == 1 << int(m.group(1))
    assert native.permute_workspace_size(262_144, 1024, 1) == native.PERMUTE_STATIC_WS_BYTES
    assert native.permute_workspace_size(262_144 + 1, 1024, 1) > native.PERMUTE_STATIC_WS_BYTES


def test_workspace_size(native):
    ws = native.permute_workspace_size
    assert ws(0, 8, 2) == 0
    assert ws(64, 8, 2) == 256  # one 1024-assignment segment x 8 experts x 4 B, rounded to 256
    assert ws(16384, 128, 8) == 128 * 128 * 4
    assert ws(4096, 32, 4) % 256 == 0
    gws = native.grouped_gemm_gateup_gather_workspace_size
    assert gws(32, 16384, 2880) == 0  # >= 128 rows per group: the gather rides in the GEMM's operand load
    assert gws(32, 32 * 128 - 1, 64) == ((32 * 128 - 1) * 64 * 2 + 255) // 256 * 256  # a grouped copy
    assert gws(256, 512, 7168) == 512 * 7168 * 2
    assert gws(4, 3, 8) == 256


def test_invalid_arguments_rejected_before_any_launch(native):
    lib = native.lib()
    null = None
    # k > E
    assert lib.moe_route_topk(null, null, null, 4, 8, 2, 3, 0, null, null, null, null) == native.MOE_ERR_INVALID_ARG
    # unknown routing mode
    assert lib.moe_topk_from_logits(null, 4, 8, 2, 7, null, null, null) == native.MOE_ERR_INVALID_ARG
    # d not a multiple of 8
    assert lib.moe_grouped_gemm_gateup(16, 16, 16, 1, 8, 12, 8, 16, null) == native.MOE_ERR_INVALID_ARG
    # misaligned pointer
    assert lib.moe_grouped_gemm_down(16, 16 + 2, 16, 1, 8, 8, 8, 16, null) == native.MOE_ERR_INVALID_ARG
    # too many groups (the limit is 1024)
    assert lib.moe_grouped_gemm_down(16, 16, 16, 4096, 8, 8, 8, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup(16, 16, 16, native.MAX_GEMM_GROUPS + 1, 8, 8, 8, 16, null) == \
        native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup_mxfp4(16, 16, 16, 16, native.MAX_GEMM_GROUPS + 1, 8, 64, 64, 16, null) == \
        native.MOE_ERR_INVALID_ARG
    # k > 32 in combine
    assert lib.moe_unpermute_combine(16, 16, 16, null, 4, 8, 33, 16, null) == native.MOE_ERR_INVALID_ARG
    # split router: no pieces; E out of range for the split
    assert lib.moe_route_topk_split(16, 16, null, null, 4, 8, 8, 2, 0, 16, 16, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_router_split_weights(16, 0, 8, 16, null) == native.MOE_ERR_INVALID_ARG
    # MXFP4: K not a multiple of 32; f not a multiple of 32; null scales; misaligned codes
    assert lib.moe_mxfp4_quantize(16, 1, 8, 48, 16, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup_mxfp4(16, 16, 16, 16, 1, 8, 64, 40, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_down_mxfp4(16, 16, null, 16, 1, 8, 64, 64, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_down_mxfp4(16, 24, 16, 16, 1, 8, 64, 64, 16, null) == native.MOE_ERR_INVALID_ARG
    # gathering gate|up: no row_src; T = 0 with rows to compute; workspace missing on the small-group path
    assert lib.moe_grouped_gemm_gateup_gather(16, null, 8, 16, 16, 1, 8, 8, 8, 16, null, 0, null) == \
        native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup_gather(16, 16, 0, 16, 16, 1, 8, 8, 8, 16, null, 0, null) == \
        native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup_gather(16, 16, 8, 16, 16, 1, 8, 8, 8, 16, null, 0, null) == \
        native.MOE_ERR_WORKSPACE
    # down + combine: M != T*k; workspace missing
    assert lib.moe_grouped_gemm_down_combine(16, 16, 16, 1, 8, 8, 8, 16, 16, 16, null, 3, 2, 16, 16, null, 0,
                                             null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_down_combine(16, 16, 16, 1, 8, 8, 8, 16, 16, 16, null, 4, 2, 16, 16, null, 0,
                                             null) == native.MOE_ERR_WORKSPACE
    # gate|up keeping its pre-activations: no gu buffer; misaligned gu
    assert lib.moe_grouped_gemm_gateup_save(16, 16, 16, 1, 8, 8, 8, 16, null, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_gateup_save(16, 16, 16, 1, 8, 8, 8, 16, 24, null) == native.MOE_ERR_INVALID_ARG
    # row gather: d not a multiple of 8; misaligned output
    assert lib.moe_gather_rows(16, 16, 4, 12, 4, 16, null) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(16, 16, 4, 8, 4, 24, null) == native.MOE_ERR_INVALID_ARG
    # missing workspace
    st = lib.moe_permute(null, 16, 64, 0, 8, 2, 16, 16, 16, 16, null, null, 0, null)
    assert st == native.MOE_ERR_WORKSPACE
    assert b"workspace" in lib.moe_last_error_string()


def test_no_device_reports_an_error_not_a_crash(native):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = native.lib()
    st = lib.moe_topk_from_logits(16, 4, 8, 2, 0, 16, 16, None)
    assert st in (native.MOE_ERR_CUDA, native.MOE_ERR_UNSUPPORTED)

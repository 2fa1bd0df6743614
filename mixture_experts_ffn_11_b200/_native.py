"""ctypes binding of libmoe.so, the C-ABI declared in include/moe.h.

Argument marshalling only: every function here checks dtypes/devices/shapes of torch tensors, passes
their device pointers and the current CUDA stream to the library, and turns a non-zero status into an
exception. All computation happens in the library's CUDA kernels. There is no fallback: if the library
is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE"}
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
DEVERR = {0x1: "wait timeout", 0x2: "expert id out of range", 0x4: "group offsets out of range",
          0x8: "permutation entry out of range"}
ROUTE_MODES = {"topk_softmax": 0, "softmax_topk_renorm": 1, "sigmoid_topk_norm": 2}

# every entry point of include/moe.h
EXPORTS = ("moe_route_topk", "moe_router_split_weights", "moe_route_topk_split", "moe_topk_from_logits", "moe_permute_workspace_size", "moe_permute",
           "moe_permute_static_ws",
           "moe_grouped_gemm_gateup", "moe_grouped_gemm_gateup_gather_workspace_size",
           "moe_grouped_gemm_gateup_gather", "moe_gather_rows", "moe_grouped_gemm_down",
           "moe_grouped_gemm_down_combine_workspace_size", "moe_grouped_gemm_down_combine", "moe_mxfp4_quantize", "moe_grouped_gemm_gateup_mxfp4",
           "moe_grouped_gemm_down_mxfp4", "moe_unpermute_combine", "moe_grouped_gemm_gateup_preact",
           "moe_grouped_gemm_gateup_save",
           "moe_swiglu_backward", "moe_permute_backward", "moe_transpose_weights",
           "moe_grouped_weight_grad_workspace_size", "moe_grouped_weight_grad", "moe_router_backward_workspace_size",
           "moe_router_backward", "moe_set_gemm_kernel", "moe_test_set_wait", "moe_get_device_error",
           "moe_last_error_string")
GEMM_KERNELS = {"auto": 0, "single": 1, "pair": 2, "wide": 3, "swap": 4}


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python mixture_experts_ffn_11_b200/build.py` "
                          "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "moe_route_topk": [vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp],
        "moe_router_split_weights": [vp, ci, ci, vp, vp],
        "moe_route_topk_split": [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp],
        "moe_topk_from_logits": [vp, ci, ci, ci, ci, vp, vp, vp],
        "moe_permute_workspace_size": [ci, ci, ci],
        "moe_permute": [vp, vp, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_permute_static_ws": [vp, vp, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp],
        "moe_grouped_gemm_gateup": [vp, vp, vp, ci, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_gateup_gather_workspace_size": [ci, ci, ci],
        "moe_grouped_gemm_gateup_gather": [vp, vp, ci, vp, vp, ci, ci, ci, ci, vp, vp, sz, vp],
        "moe_gather_rows": [vp, vp, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_down": [vp, vp, vp, ci, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_down_combine_workspace_size": [ci, ci],
        "moe_grouped_gemm_down_combine": [vp, vp, vp, ci, ci, ci, ci, vp, vp, vp, vp, ci, ci, vp, vp, vp, sz, vp],
        "moe_mxfp4_quantize": [vp, ci, ci, ci, vp, vp, vp],
        "moe_grouped_gemm_gateup_mxfp4": [vp, vp, vp, vp, ci, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_down_mxfp4": [vp, vp, vp, vp, ci, ci, ci, ci, vp, vp],
        "moe_unpermute_combine": [vp, vp, vp, vp, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_gateup_preact": [vp, vp, vp, ci, ci, ci, ci, vp, vp],
        "moe_grouped_gemm_gateup_save": [vp, vp, vp, ci, ci, ci, ci, vp, vp, vp],
        "moe_swiglu_backward": [vp, vp, ci, ci, vp, vp],
        "moe_permute_backward": [vp, vp, vp, vp, ci, ci, ci, vp, vp, vp],
        "moe_transpose_weights": [vp, ci, ci, ci, vp, vp],
        "moe_grouped_weight_grad_workspace_size": [ci, ci, ci, ci],
        "moe_grouped_weight_grad": [vp, vp, vp, ci, ci, ci, ci, vp, vp, sz, vp],
        "moe_router_backward_workspace_size": [ci, ci, ci, ci],
        "moe_router_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, sz, vp],
        "moe_set_gemm_kernel": [ci],
        "moe_test_set_wait": [ctypes.c_ulonglong, ci],
        "moe_get_device_error": [ctypes.POINTER(ctypes.c_uint), vp],
        "moe_last_error_string": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ci
    lib.moe_permute_workspace_size.restype = sz
    lib.moe_grouped_weight_grad_workspace_size.restype = sz
    lib.moe_grouped_gemm_gateup_gather_workspace_size.restype = sz
    lib.moe_grouped_gemm_down_combine_workspace_size.restype = sz
    lib.moe_router_backward_workspace_size.restype = sz
    lib.moe_last_error_string.restype = ctypes.c_char_p
    return lib


_lib = load_library()


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what, (_lib.moe_last_error_string() or b"").decode())


def _stream(stream):
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _p(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, shape=None, name="tensor"):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: want a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: want shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def route_topk(x, w_router, bias, k, mode, logits, topk_idx, topk_w, stream=None):
    T, d = x.shape
    E = w_router.shape[0]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(w_router, torch.float32, (E, d), "w_router")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(logits, torch.float32, (T, E), "logits")
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    _check(_lib.moe_route_topk(_p(x), _p(w_router), _p(bias), T, d, E, k, ROUTE_MODES[mode], _p(logits),
                               _p(topk_idx), _p(topk_w), _stream(stream)), "moe_route_topk")


def router_split_weights(w_router, w_pieces, stream=None):
    """w_pieces [3, E, d] bf16 <- the hi / mid / lo split of w_router [E, d] fp32 (once per weight update)."""
    E, d = w_router.shape
    _need(w_router, torch.float32, (E, d), "w_router")
    _need(w_pieces, torch.bfloat16, (3, E, d), "w_pieces")
    _check(_lib.moe_router_split_weights(_p(w_router), E, d, _p(w_pieces), _stream(stream)),
           "moe_router_split_weights")


def route_topk_split(x, w_router, w_pieces, bias, k, mode, logits, topk_idx, topk_w, stream=None):
    """route_topk with the pieces written by router_split_weights for this w_router."""
    T, d = x.shape
    E = w_router.shape[0]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(w_router, torch.float32, (E, d), "w_router")
    _need(w_pieces, torch.bfloat16, (3, E, d), "w_pieces")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _need(logits, torch.float32, (T, E), "logits")
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    _check(_lib.moe_route_topk_split(_p(x), _p(w_router), _p(w_pieces), _p(bias), T, d, E, k, ROUTE_MODES[mode],
                                     _p(logits), _p(topk_idx), _p(topk_w), _stream(stream)), "moe_route_topk_split")


def topk_from_logits(logits, k, mode, topk_idx, topk_w, stream=None):
    T, E = logits.shape
    _need(logits, torch.float32, (T, E), "logits")
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    _check(_lib.moe_topk_from_logits(_p(logits), T, E, k, ROUTE_MODES[mode], _p(topk_idx), _p(topk_w),
                                     _stream(stream)), "moe_topk_from_logits")


def permute_workspace_size(T: int, E: int, k: int) -> int:
    return int(_lib.moe_permute_workspace_size(T, E, k))


def permute(x, topk_idx, E, counts, offsets, perm_src, inv_perm, x_perm, ws, stream=None):
    T, k = topk_idx.shape
    R = T * k
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(counts, torch.int32, (E,), "counts")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(perm_src, torch.int32, (R,), "perm_src")
    _need(inv_perm, torch.int32, (R,), "inv_perm")
    d = 0
    if x is not None:
        d = x.shape[1]
        _need(x, torch.bfloat16, (T, d), "x")
        _need(x_perm, torch.bfloat16, (R, d), "x_perm")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.moe_permute(_p(x), _p(topk_idx), T, d, E, k, _p(counts), _p(offsets), _p(perm_src),
                            _p(inv_perm), _p(x_perm), _p(ws), ws_bytes, _stream(stream)), "moe_permute")


PERMUTE_STATIC_WS_BYTES = 1 << 20  # MOE_PERMUTE_STATIC_WS_BYTES in include/moe.h
MAX_GEMM_GROUPS = 1024  # the grouped GEMMs' limit on G (include/moe.h)


def permute_static_ws(x, topk_idx, E, counts, offsets, perm_src, inv_perm, x_perm, stream=None):
    """moe_permute without a workspace argument: the library uses its own static scratch array (for
    callers that cannot supply device scratch memory; see include/moe.h for the limits)."""
    T, k = topk_idx.shape
    R = T * k
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(counts, torch.int32, (E,), "counts")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(perm_src, torch.int32, (R,), "perm_src")
    _need(inv_perm, torch.int32, (R,), "inv_perm")
    d = 0
    if x is not None:
        d = x.shape[1]
        _need(x, torch.bfloat16, (T, d), "x")
        _need(x_perm, torch.bfloat16, (R, d), "x_perm")
    _check(_lib.moe_permute_static_ws(_p(x), _p(topk_idx), T, d, E, k, _p(counts), _p(offsets), _p(perm_src),
                                      _p(inv_perm), _p(x_perm), _stream(stream)), "moe_permute_static_ws")


def grouped_gemm_gateup(a, w_gateup, group_offsets, h, stream=None):
    M, d = a.shape
    G, two_f, d2 = w_gateup.shape
    f = two_f // 2
    _need(a, torch.bfloat16, (M, d), "a")
    _need(w_gateup, torch.bfloat16, (G, 2 * f, d), "w_gateup")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(h, torch.bfloat16, (M, f), "h")
    _check(_lib.moe_grouped_gemm_gateup(_p(a), _p(w_gateup), _p(group_offsets), G, M, d, f, _p(h),
                                        _stream(stream)), "moe_grouped_gemm_gateup")


def grouped_gemm_gateup_gather_workspace_size(G: int, M: int, d: int) -> int:
    return int(_lib.moe_grouped_gemm_gateup_gather_workspace_size(G, M, d))


def grouped_gemm_gateup_gather(x, row_src, w_gateup, group_offsets, h, ws=None, stream=None):
    """h for A rows x[row_src[r]] (moe_grouped_gemm_gateup_gather); ws: a uint8 tensor of at least
    grouped_gemm_gateup_gather_workspace_size(G, M, d) bytes, or None when that is 0."""
    T, d = x.shape
    M = row_src.shape[0]
    G, two_f, d2 = w_gateup.shape
    f = two_f // 2
    _need(x, torch.bfloat16, (T, d), "x")
    _need(row_src, torch.int32, (M,), "row_src")
    _need(w_gateup, torch.bfloat16, (G, 2 * f, d), "w_gateup")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(h, torch.bfloat16, (M, f), "h")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.moe_grouped_gemm_gateup_gather(_p(x), _p(row_src), T, _p(w_gateup), _p(group_offsets), G, M, d, f,
                                               _p(h), _p(ws), ws_bytes, _stream(stream)),
           "moe_grouped_gemm_gateup_gather")


def gather_rows(x, row_src, out, stream=None):
    """out[r] = x[row_src[r]] (moe_gather_rows)."""
    T, d = x.shape
    R = row_src.shape[0]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(row_src, torch.int32, (R,), "row_src")
    _need(out, torch.bfloat16, (R, d), "out")
    _check(_lib.moe_gather_rows(_p(x), _p(row_src), T, d, R, _p(out), _stream(stream)), "moe_gather_rows")


def grouped_gemm_down(h, w_down, group_offsets, y, stream=None):
    M, f = h.shape
    G, d, f2 = w_down.shape
    _need(h, torch.bfloat16, (M, f), "h")
    _need(w_down, torch.bfloat16, (G, d, f), "w_down")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(y, torch.bfloat16, (M, d), "y")
    _check(_lib.moe_grouped_gemm_down(_p(h), _p(w_down), _p(group_offsets), G, M, d, f, _p(y), _stream(stream)),
           "moe_grouped_gemm_down")


def grouped_gemm_down_combine_workspace_size(T: int, d: int) -> int:
    return int(_lib.moe_grouped_gemm_down_combine_workspace_size(T, d))


def grouped_gemm_down_combine(h, w_down, group_offsets, perm_src, inv_perm, topk_w, shared, y_perm, y, ws,
                              stream=None):
    """y_perm = down(h) and y = combine(y_perm) in one call (moe_grouped_gemm_down_combine); ws: a uint8 tensor of
    at least grouped_gemm_down_combine_workspace_size(T, d) bytes."""
    M, f = h.shape
    G, d, f2 = w_down.shape
    T, k = topk_w.shape
    _need(h, torch.bfloat16, (M, f), "h")
    _need(w_down, torch.bfloat16, (G, d, f), "w_down")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(perm_src, torch.int32, (M,), "perm_src")
    _need(inv_perm, torch.int32, (M,), "inv_perm")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    if shared is not None:
        _need(shared, torch.bfloat16, (T, d), "shared")
    _need(y_perm, torch.bfloat16, (M, d), "y_perm")
    _need(y, torch.bfloat16, (T, d), "y")
    _need(ws, torch.uint8, None, "ws")
    _check(_lib.moe_grouped_gemm_down_combine(_p(h), _p(w_down), _p(group_offsets), G, M, d, f, _p(perm_src),
                                              _p(inv_perm), _p(topk_w), _p(shared), T, k, _p(y_perm), _p(y), _p(ws),
                                              ws.numel(), _stream(stream)), "moe_grouped_gemm_down_combine")


def mxfp4_quantize(w, q, s, stream=None):
    """Encode bf16 weights w [G, N, K] as MXFP4 codes q [G, N, K/2] (uint8) and scales s [G, K/32, N] (uint8)."""
    G, N, K = w.shape
    _need(w, torch.bfloat16, (G, N, K), "w")
    _need(q, torch.uint8, (G, N, K // 2), "q")
    _need(s, torch.uint8, (G, K // 32, N), "s")
    _check(_lib.moe_mxfp4_quantize(_p(w), G, N, K, _p(q), _p(s), _stream(stream)), "moe_mxfp4_quantize")


def grouped_gemm_gateup_mxfp4(a, wq_gateup, ws_gateup, group_offsets, h, stream=None):
    M, d = a.shape
    G, two_f, _ = wq_gateup.shape
    f = two_f // 2
    _need(a, torch.bfloat16, (M, d), "a")
    _need(wq_gateup, torch.uint8, (G, 2 * f, d // 2), "wq_gateup")
    _need(ws_gateup, torch.uint8, (G, d // 32, 2 * f), "ws_gateup")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(h, torch.bfloat16, (M, f), "h")
    _check(_lib.moe_grouped_gemm_gateup_mxfp4(_p(a), _p(wq_gateup), _p(ws_gateup), _p(group_offsets), G, M, d, f,
                                              _p(h), _stream(stream)), "moe_grouped_gemm_gateup_mxfp4")


def grouped_gemm_down_mxfp4(h, wq_down, ws_down, group_offsets, y, stream=None):
    M, f = h.shape
    G, d, _ = wq_down.shape
    _need(h, torch.bfloat16, (M, f), "h")
    _need(wq_down, torch.uint8, (G, d, f // 2), "wq_down")
    _need(ws_down, torch.uint8, (G, f // 32, d), "ws_down")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(y, torch.bfloat16, (M, d), "y")
    _check(_lib.moe_grouped_gemm_down_mxfp4(_p(h), _p(wq_down), _p(ws_down), _p(group_offsets), G, M, d, f, _p(y),
                                            _stream(stream)), "moe_grouped_gemm_down_mxfp4")


def unpermute_combine(y_perm, inv_perm, topk_w, shared, y, stream=None):
    T, k = topk_w.shape
    d = y.shape[1]
    _need(y_perm, torch.bfloat16, (T * k, d), "y_perm")
    _need(inv_perm, torch.int32, (T * k,), "inv_perm")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    if shared is not None:
        _need(shared, torch.bfloat16, (T, d), "shared")
    _need(y, torch.bfloat16, (T, d), "y")
    _check(_lib.moe_unpermute_combine(_p(y_perm), _p(inv_perm), _p(topk_w), _p(shared), T, d, k, _p(y),
                                      _stream(stream)), "moe_unpermute_combine")


# ---- backward ----

def grouped_gemm_gateup_preact(a, w_gateup, group_offsets, gu, stream=None):
    """gu [M, 2f] <- the gate (columns [0, f)) and up (columns [f, 2f)) pre-activations of the grouped projection."""
    M, d = a.shape
    G, two_f, _ = w_gateup.shape
    f = two_f // 2
    _need(a, torch.bfloat16, (M, d), "a")
    _need(w_gateup, torch.bfloat16, (G, 2 * f, d), "w_gateup")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(gu, torch.bfloat16, (M, 2 * f), "gu")
    _check(_lib.moe_grouped_gemm_gateup_preact(_p(a), _p(w_gateup), _p(group_offsets), G, M, d, f, _p(gu),
                                               _stream(stream)), "moe_grouped_gemm_gateup_preact")


def grouped_gemm_gateup_save(a, w_gateup, group_offsets, h, gu, stream=None):
    """h [M, f] as grouped_gemm_gateup and gu [M, 2f] as grouped_gemm_gateup_preact, from one pass where possible."""
    M, d = a.shape
    G, two_f, _ = w_gateup.shape
    f = two_f // 2
    _need(a, torch.bfloat16, (M, d), "a")
    _need(w_gateup, torch.bfloat16, (G, 2 * f, d), "w_gateup")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(h, torch.bfloat16, (M, f), "h")
    _need(gu, torch.bfloat16, (M, 2 * f), "gu")
    _check(_lib.moe_grouped_gemm_gateup_save(_p(a), _p(w_gateup), _p(group_offsets), G, M, d, f, _p(h), _p(gu),
                                             _stream(stream)), "moe_grouped_gemm_gateup_save")


def swiglu_backward(dh, gu, dgu, stream=None):
    M, f = dh.shape
    _need(dh, torch.bfloat16, (M, f), "dh")
    _need(gu, torch.bfloat16, (M, 2 * f), "gu")
    _need(dgu, torch.bfloat16, (M, 2 * f), "dgu")
    _check(_lib.moe_swiglu_backward(_p(dh), _p(gu), M, f, _p(dgu), _stream(stream)), "moe_swiglu_backward")


def permute_backward(dy, inv_perm, topk_w, y_perm, dy_perm, dw, stream=None):
    T, d = dy.shape
    k = topk_w.shape[1]
    _need(dy, torch.bfloat16, (T, d), "dy")
    _need(inv_perm, torch.int32, (T * k,), "inv_perm")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    _need(y_perm, torch.bfloat16, (T * k, d), "y_perm")
    _need(dy_perm, torch.bfloat16, (T * k, d), "dy_perm")
    _need(dw, torch.float32, (T, k), "dw")
    _check(_lib.moe_permute_backward(_p(dy), _p(inv_perm), _p(topk_w), _p(y_perm), T, d, k, _p(dy_perm), _p(dw),
                                     _stream(stream)), "moe_permute_backward")


def transpose_weights(w, wt, stream=None):
    """wt [G, C, R] <- per-group transpose of w [G, R, C] (bf16)."""
    G, R, C = w.shape
    _need(w, torch.bfloat16, (G, R, C), "w")
    _need(wt, torch.bfloat16, (G, C, R), "wt")
    _check(_lib.moe_transpose_weights(_p(w), G, R, C, _p(wt), _stream(stream)), "moe_transpose_weights")


def grouped_weight_grad_workspace_size(M: int, G: int, P: int, Q: int) -> int:
    return int(_lib.moe_grouped_weight_grad_workspace_size(M, G, P, Q))


def grouped_weight_grad(a, b, group_offsets, dw, ws, stream=None):
    """dw [G, P, Q] fp32 <- for each group g: sum over its rows of a[r]^T b[r] (a [M, P], b [M, Q] bf16)."""
    M, P = a.shape
    Q = b.shape[1]
    G = group_offsets.shape[0] - 1
    _need(a, torch.bfloat16, (M, P), "a")
    _need(b, torch.bfloat16, (M, Q), "b")
    _need(group_offsets, torch.int32, (G + 1,), "group_offsets")
    _need(dw, torch.float32, (G, P, Q), "dw")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.moe_grouped_weight_grad(_p(a), _p(b), _p(group_offsets), G, M, P, Q, _p(dw), _p(ws), ws_bytes,
                                        _stream(stream)), "moe_grouped_weight_grad")


def router_backward_workspace_size(T: int, d: int, E: int, k: int) -> int:
    return int(_lib.moe_router_backward_workspace_size(T, d, E, k))


def router_backward(x, w_router, logits, topk_idx, topk_w, dw, perm_src, inv_perm, expert_offsets, mode, dx,
                    dw_router, dbias=None, dx_addend=None, ws=None, stream=None):
    T, d = x.shape
    E = w_router.shape[0]
    k = topk_idx.shape[1]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(w_router, torch.float32, (E, d), "w_router")
    _need(logits, torch.float32, (T, E), "logits")
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    _need(dw, torch.float32, (T, k), "dw")
    _need(perm_src, torch.int32, (T * k,), "perm_src")
    _need(inv_perm, torch.int32, (T * k,), "inv_perm")
    _need(expert_offsets, torch.int32, (E + 1,), "expert_offsets")
    _need(dx, torch.bfloat16, (T, d), "dx")
    _need(dw_router, torch.float32, (E, d), "dw_router")
    if dbias is not None:
        _need(dbias, torch.float32, (E,), "dbias")
    if dx_addend is not None:
        _need(dx_addend, torch.bfloat16, (T, d), "dx_addend")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.moe_router_backward(_p(x), _p(w_router), _p(logits), _p(topk_idx), _p(topk_w), _p(dw), _p(perm_src),
                                    _p(inv_perm), _p(expert_offsets), T, d, E, k, ROUTE_MODES[mode], _p(dx_addend),
                                    _p(dx), _p(dw_router), _p(dbias), _p(ws), ws_bytes, _stream(stream)),
           "moe_router_backward")


def set_gemm_kernel(name: str) -> None:
    """Force one bf16 grouped-GEMM kernel family ("single", "pair", "wide", "swap") for every later call in the
    process, or restore the library's own choice ("auto"). A measurement and test hook."""
    if name not in GEMM_KERNELS:
        raise ValueError(f"unknown GEMM kernel family {name!r}")
    _check(_lib.moe_set_gemm_kernel(GEMM_KERNELS[name]), "moe_set_gemm_kernel")


class gemm_kernel:
    """Context manager: `with gemm_kernel("swap"): ...` forces a family inside the block, then restores "auto"."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        set_gemm_kernel(self.name)
        return self

    def __exit__(self, *exc):
        set_gemm_kernel("auto")
        return False


def test_set_wait(limit_ns: int = 0, stall: bool = False) -> None:
    """Test hook: the bounded waits' limit on the current device (0 = the default 2 s) and, with stall, a wait
    that nothing ends in every bf16 grouped GEMM, so its timeout path runs."""
    _check(_lib.moe_test_set_wait(int(limit_ns), 1 if stall else 0), "moe_test_set_wait")


def get_device_error(stream=None) -> int:
    """Synchronise the stream and read-and-clear the device error word (0 = no anomaly)."""
    v = ctypes.c_uint(0)
    st = _lib.moe_get_device_error(ctypes.byref(v), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        _check(st, "moe_get_device_error")
    return int(v.value)

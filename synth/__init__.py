"""Seeded synthetic inputs for the sparse MoE feed-forward layer.

This module is the only code shared by the CPU oracle and the CUDA path. It
draws numbers and nothing else: it holds none of the layer's arithmetic
(no routing, no sorting, no projections). The generator is defined in
``gen.c`` and implemented twice, for the host (``gen.c``) and for the GPU
(``gen_cuda.cu``), bit-identically.

Workloads follow the shapes of the models named in the blog post
"Mixture of Experts (MoEs) in Transformers" (section "From Dense to Sparse":
gpt-oss-20b with 32 experts and 4 active; the adoption list naming
Mixtral-8x7B) plus a tiny case, a Zipf-skewed 128-expert case and a
256-expert decode case with a shared expert. No trained weights or datasets
are involved; everything is drawn from the generator.

Tensor ids within one seed: 0 x, 1 router weight, 2 gate|up weight,
3 down weight, 4 router-bias permutation, 5 shared gate|up, 6 shared down,
7 upstream gradient dy (for the backward pass).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "_gen.so")
_CUDA_SO = os.path.join(_HERE, "_gen_cuda.so")

TID_X, TID_WR, TID_WGU, TID_WD, TID_BIAS_PERM, TID_WGU_SHARED, TID_WD_SHARED, TID_DY = range(8)

X_SIGMA = 1.0
W_SIGMA = 0.02


def build_host(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", src, "-o", _HOST_SO])
    return _HOST_SO


def build_cuda(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen_cuda.cu")
    if force or not os.path.exists(_CUDA_SO) or os.path.getmtime(_CUDA_SO) < os.path.getmtime(src):
        subprocess.check_call([
            "nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC",
            "-gencode", "arch=compute_100a,code=sm_100a", src, "-o", _CUDA_SO,
        ])
    return _CUDA_SO


_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        lib = ctypes.CDLL(build_host())
        u64, dbl, vp, ci = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, u64, dbl, vp, ci]
        lib.synth_normal_f32.argtypes = [u64, u64, u64, u64, dbl, vp, ci]
        lib.synth_uniform_u64.argtypes = [u64, u64, u64, u64, vp]
        lib.synth_stream_key.argtypes = [u64, u64]
        lib.synth_stream_key.restype = u64
        _host = lib
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(_CUDA_SO):
            raise RuntimeError(f"{_CUDA_SO} is missing: build it with synth.build_cuda()")
        lib = ctypes.CDLL(_CUDA_SO)
        u64, dbl, vp = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        for name in ("synth_normal_bf16_device", "synth_normal_f32_device"):
            getattr(lib, name).argtypes = [u64, u64, u64, u64, dbl, vp, vp]
            getattr(lib, name).restype = ctypes.c_int
        _cuda = lib
    return _cuda


def host_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def normal_bf16(seed: int, tensor_id: int, first: int, count: int, sigma: float) -> np.ndarray:
    """Elements [first, first+count) of a bf16 tensor, as raw uint16 bits."""
    out = np.empty(count, dtype=np.uint16)
    if count:
        _host_lib().synth_normal_bf16(seed, tensor_id, first, count, sigma, out.ctypes.data, host_threads())
    return out


def normal_f32(seed: int, tensor_id: int, first: int, count: int, sigma: float) -> np.ndarray:
    out = np.empty(count, dtype=np.float32)
    if count:
        _host_lib().synth_normal_f32(seed, tensor_id, first, count, sigma, out.ctypes.data, host_threads())
    return out


def uniform_u64(seed: int, tensor_id: int, first: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    if count:
        _host_lib().synth_uniform_u64(seed, tensor_id, first, count, out.ctypes.data)
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bits (finite inputs)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


@dataclass(frozen=True)
class Workload:
    """One MoE layer shape and its input recipe.

    route: "topk_softmax" (softmax over the k selected logits),
    "softmax_topk_renorm" (softmax over all E, keep top-k, divide by their sum),
    "sigmoid_topk_norm" (sigmoid scores of the selected experts, divided by their sum).
    Selection is always on the logits.
    """
    name: str
    T: int
    d: int
    f: int
    E: int
    k: int
    route: str = "topk_softmax"
    zipf_s: float = 0.0  # > 0: per-expert router bias so popularity follows Zipf(s)
    shared_f: int = 0  # > 0: one always-on shared SwiGLU expert of this width
    seed: int = 0
    weights: str = "bf16"  # storage of the expert weights: "bf16", or "mxfp4" (encoded from the bf16 draws)
    note: str = field(default="", compare=False)

    @property
    def R(self) -> int:
        return self.T * self.k

    def flops(self) -> float:
        """6*T*k*d*f (+6*T*d*f_shared): two multiply-adds per weight element touched per routed row."""
        return 6.0 * self.T * self.k * self.d * self.f + 6.0 * self.T * self.d * self.shared_f


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 512, 8, 2, note="tiny layer, parity only"),
    "gpt-oss-20b-prefill": Workload("gpt-oss-20b-prefill", 4096, 2880, 2880, 32, 4,
                                    note="gpt-oss-20b-shaped prefill"),
    "mixtral-8x7b-prefill": Workload("mixtral-8x7b-prefill", 8192, 4096, 14336, 8, 2,
                                     route="softmax_topk_renorm", note="Mixtral-8x7B-shaped prefill"),
    "zipf-128e": Workload("zipf-128e", 16384, 2048, 768, 128, 8, zipf_s=1.2,
                          note="128 small experts, Zipf(1.2) skewed load"),
    "decode-256e-shared": Workload("decode-256e-shared", 64, 7168, 2048, 256, 8, route="sigmoid_topk_norm",
                                   shared_f=2048, note="256-expert decode with one shared expert"),
    "decode-256e-shared-mxfp4": Workload("decode-256e-shared-mxfp4", 64, 7168, 2048, 256, 8,
                                         route="sigmoid_topk_norm", shared_f=2048, weights="mxfp4",
                                         note="the 256-expert decode layer with MXFP4 expert weights"),
}


def workload(name: str, **over) -> Workload:
    w = WORKLOADS[name]
    if over:
        w = Workload(**{**w.__dict__, **over})
    return w


def zipf_bias(w: Workload) -> np.ndarray | None:
    """Per-expert router bias b_e = ln p_{pi(e)}, p_r proportional to r^-s (r = 1..E), pi a seeded permutation.

    The bias is an input of the router, added to every token's logit of expert e.
    """
    if w.zipf_s <= 0:
        return None
    E = w.E
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-w.zipf_s)
    p /= p.sum()
    # Fisher-Yates with draws from the bias-permutation stream.
    perm = np.arange(E)
    draws = uniform_u64(w.seed, TID_BIAS_PERM, 0, E)
    for i in range(E - 1, 0, -1):
        j = int(draws[i] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return np.log(p[perm]).astype(np.float32)


# ---- host tensors (numpy) -------------------------------------------------------------------------

def x_host(w: Workload) -> np.ndarray:
    return normal_bf16(w.seed, TID_X, 0, w.T * w.d, X_SIGMA).reshape(w.T, w.d)


def dy_host(w: Workload) -> np.ndarray:
    """Upstream gradient d loss / d y for the backward pass: [T, d] bf16 bits, N(0, 1)."""
    return normal_bf16(w.seed, TID_DY, 0, w.T * w.d, X_SIGMA).reshape(w.T, w.d)


def w_router_host(w: Workload) -> np.ndarray:
    return normal_f32(w.seed, TID_WR, 0, w.E * w.d, W_SIGMA).reshape(w.E, w.d)


def w_gateup_expert_host(w: Workload, e: int) -> np.ndarray:
    n = 2 * w.f * w.d
    return normal_bf16(w.seed, TID_WGU, e * n, n, W_SIGMA).reshape(2 * w.f, w.d)


def w_down_expert_host(w: Workload, e: int) -> np.ndarray:
    n = w.d * w.f
    return normal_bf16(w.seed, TID_WD, e * n, n, W_SIGMA).reshape(w.d, w.f)


def w_gateup_host(w: Workload) -> np.ndarray:
    return normal_bf16(w.seed, TID_WGU, 0, w.E * 2 * w.f * w.d, W_SIGMA).reshape(w.E, 2 * w.f, w.d)


def w_down_host(w: Workload) -> np.ndarray:
    return normal_bf16(w.seed, TID_WD, 0, w.E * w.d * w.f, W_SIGMA).reshape(w.E, w.d, w.f)


def shared_host(w: Workload):
    if not w.shared_f:
        return None, None
    gu = normal_bf16(w.seed, TID_WGU_SHARED, 0, 2 * w.shared_f * w.d, W_SIGMA).reshape(2 * w.shared_f, w.d)
    dn = normal_bf16(w.seed, TID_WD_SHARED, 0, w.d * w.shared_f, W_SIGMA).reshape(w.d, w.shared_f)
    return gu, dn


# ---- device tensors (torch, filled by the GPU generator) -------------------------------------------

def fill_device(t, seed: int, tensor_id: int, first: int, sigma: float, stream=None) -> None:
    """Fill a contiguous CUDA tensor (torch.bfloat16 or torch.float32) with generator elements [first, ...)."""
    import torch

    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("fill_device wants a contiguous CUDA tensor")
    lib = _cuda_lib()
    s = (stream or torch.cuda.current_stream(t.device)).cuda_stream
    with torch.cuda.device(t.device):
        if t.dtype == torch.bfloat16:
            rc = lib.synth_normal_bf16_device(seed, tensor_id, first, t.numel(), sigma, t.data_ptr(), s)
        elif t.dtype == torch.float32:
            rc = lib.synth_normal_f32_device(seed, tensor_id, first, t.numel(), sigma, t.data_ptr(), s)
        else:
            raise ValueError(f"unsupported dtype {t.dtype}")
    if rc != 0:
        raise RuntimeError(f"synth device fill failed ({rc})")


def device_inputs(w: Workload, device="cuda", with_x: bool = True) -> dict:
    """All inputs of a workload, resident on the GPU (torch tensors)."""
    import torch

    dev = torch.device(device)
    out = {}
    if with_x:
        out["x"] = torch.empty(w.T, w.d, dtype=torch.bfloat16, device=dev)
        fill_device(out["x"], w.seed, TID_X, 0, X_SIGMA)
    out["w_router"] = torch.empty(w.E, w.d, dtype=torch.float32, device=dev)
    fill_device(out["w_router"], w.seed, TID_WR, 0, W_SIGMA)
    out["w_gateup"] = torch.empty(w.E, 2 * w.f, w.d, dtype=torch.bfloat16, device=dev)
    fill_device(out["w_gateup"], w.seed, TID_WGU, 0, W_SIGMA)
    out["w_down"] = torch.empty(w.E, w.d, w.f, dtype=torch.bfloat16, device=dev)
    fill_device(out["w_down"], w.seed, TID_WD, 0, W_SIGMA)
    b = zipf_bias(w)
    out["bias"] = torch.from_numpy(b).to(dev) if b is not None else None
    if w.shared_f:
        out["w_gateup_shared"] = torch.empty(2 * w.shared_f, w.d, dtype=torch.bfloat16, device=dev)
        fill_device(out["w_gateup_shared"], w.seed, TID_WGU_SHARED, 0, W_SIGMA)
        out["w_down_shared"] = torch.empty(w.d, w.shared_f, dtype=torch.bfloat16, device=dev)
        fill_device(out["w_down_shared"], w.seed, TID_WD_SHARED, 0, W_SIGMA)
    else:
        out["w_gateup_shared"] = out["w_down_shared"] = None
    return out

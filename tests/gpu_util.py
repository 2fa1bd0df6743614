"""Helpers shared by the GPU tests: host<->device moves of bf16 bit patterns and the parity bar."""
from __future__ import annotations

import numpy as np
import torch

import synth

# Parity bar of the layer output: per element |gpu - ref| <= 1e-2 * max|ref| + 1e-2 * |ref|, and the
# relative Frobenius error over the compared rows <= 5e-3.
ELEM_ABS, ELEM_REL, FRO_MAX = 1e-2, 1e-2, 5e-3


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_host_f32(t: torch.Tensor) -> np.ndarray:
    return synth.bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_close(gpu: np.ndarray, ref: np.ndarray, what: str) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite GPU output"
    err = np.abs(gpu - ref)
    bound = ELEM_ABS * np.abs(ref).max() + ELEM_REL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements outside the bound; "
                           f"worst excess {float((err - bound).max()):.3g}, max err {float(err.max()):.3g}")
    fro = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))
    assert fro <= FRO_MAX, f"{what}: relative Frobenius error {fro:.3e} > {FRO_MAX}"
    return fro

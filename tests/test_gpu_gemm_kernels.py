"""Every bf16 grouped-GEMM kernel family, forced through the C-ABI hook, on ragged groups (B200).

The families (single CTA, CTA pair, two-accumulator pair, weights-as-M "swap" pair) tile the same sums
differently; each output element is the same fp32 accumulation of bf16 products over K in 16-wide steps, so
their h and y_perm must agree bit for bit, and the layer output of each must meet the parity bar against the
oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_host_f32, check_close, to_dev_bf16

pytestmark = pytest.mark.gpu

N = pytest.importorskip("mixture_experts_ffn_11_b200._native")

FAMILIES = ("single", "pair", "wide", "swap")

CASES = [
    # (name, rows per expert, d, f)
    ("empty_single_tail_full", [0, 1, 127, 128, 129, 257, 0], 200, 72),
    ("many_small", [3] * 40 + [0] * 24, 64, 96),
    # token tiles of the swap kernel: every remainder of 16, balanced splits of 257..1000 rows, an empty last group
    ("swap_token_tiles", [1, 15, 16, 17, 31, 33, 255, 256, 257, 447, 569, 1000, 0], 200, 136),
    # weight blocks: gate|up f = 136 (a 128-column block and an 8-column one), down d = 200 (one part-filled block)
    ("swap_partial_weight_blocks", [300, 0, 700, 45], 264, 360),
    # gpt-oss-like sizes: d = f = 2880 (the last 128-column block half full, down's last 256 block a quarter full)
    ("gpt_oss_like", [447, 569, 512, 0, 511], 2880, 2880),
    # K tails: K = 4160 (65 K blocks: the last ring stage holds one), down K = 136
    ("k_tail_in_last_stage", [0, 300, 1, 257], 4160, 136),
    # one big group, many token tiles
    ("one_expert_takes_all", [0, 0, 2000, 0], 256, 512),
]


def _inputs(counts, d, f, seed=3):
    rng = np.random.default_rng(2)
    E = len(counts)
    idx = np.concatenate([np.full(c, e) for e, c in enumerate(counts)]).astype(np.int32)
    rng.shuffle(idx)
    idx = idx.reshape(-1, 1)
    T = idx.shape[0]
    x = synth.normal_bf16(seed, 0, 0, T * d, 1.0).reshape(T, d)
    gu = synth.normal_bf16(seed, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    dn = synth.normal_bf16(seed, 3, 0, E * d * f, 0.05).reshape(E, d, f)
    return idx, x, gu, dn


def _run(family, idx, x_bits, gu_bits, dn_bits):
    T, d = x_bits.shape
    E, two_f, _ = gu_bits.shape
    f = two_f // 2
    k = idx.shape[1]
    R = T * k
    dev = "cuda"
    p = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
             offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
             perm_src=torch.empty(R, dtype=torch.int32, device=dev),
             inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
             x_perm=torch.empty(R, d, dtype=torch.bfloat16, device=dev),
             ws=torch.empty(max(N.permute_workspace_size(T, E, k), 256), dtype=torch.uint8, device=dev))
    N.permute(to_dev_bf16(x_bits), torch.from_numpy(idx).cuda(), E, p["counts"], p["offsets"], p["perm_src"],
              p["inv_perm"], p["x_perm"], p["ws"])
    h = torch.full((R, f), float("nan"), dtype=torch.bfloat16, device=dev)
    y_perm = torch.full((R, d), float("nan"), dtype=torch.bfloat16, device=dev)
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    with N.gemm_kernel(family):
        N.grouped_gemm_gateup(p["x_perm"], to_dev_bf16(gu_bits), p["offsets"], h)
        N.grouped_gemm_down(h, to_dev_bf16(dn_bits), p["offsets"], y_perm)
    N.unpermute_combine(y_perm, p["inv_perm"], torch.ones(T, k, dtype=torch.float32, device=dev), None, y)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0, family
    return h, y_perm, y


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    torch.cuda.set_device(0)
    N.get_device_error()
    yield
    N.set_gemm_kernel("auto")


@pytest.mark.parametrize("name,counts,d,f", CASES, ids=[c[0] for c in CASES])
def test_kernel_families_agree_bitwise_and_match_oracle(name, counts, d, f):
    idx, x, gu, dn = _inputs(counts, d, f)
    T = idx.shape[0]
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, np.ones((T, 1)), np.arange(T))
    outs = {}
    for fam in FAMILIES:
        h, yp, y = _run(fam, idx, x, gu, dn)
        assert not torch.isnan(h.float()).any(), f"{name}/{fam}: rows of h left unwritten"
        assert not torch.isnan(yp.float()).any(), f"{name}/{fam}: rows of y_perm left unwritten"
        check_close(bf16_to_host_f32(y), ref, f"{name}/{fam}")
        outs[fam] = (h.view(torch.int16), yp.view(torch.int16))
    for fam in FAMILIES[1:]:
        assert torch.equal(outs[fam][0], outs["single"][0]), f"{name}: h of {fam} differs from single"
        assert torch.equal(outs[fam][1], outs["single"][1]), f"{name}: y_perm of {fam} differs from single"


def test_unknown_family_rejected():
    with pytest.raises(ValueError):
        N.set_gemm_kernel("nope")
    assert N.lib().moe_set_gemm_kernel(99) == N.MOE_ERR_INVALID_ARG


def test_swiglu_saturation_matches_oracle():
    """Gate pre-activations far into both tails (|g| from 16 to 4096): silu(g) tends to g above and to 0 below,
    where e^-g overflows fp32. With W_down = identity (d = f) the layer output is h itself, so every h value is
    compared with the oracle's fp64 silu(g) * u, in every kernel family."""
    rng = np.random.default_rng(7)
    counts = [150, 0, 170]
    E, d = len(counts), 256
    f = d
    idx = np.concatenate([np.full(c, e) for e, c in enumerate(counts)]).astype(np.int32)
    rng.shuffle(idx)
    idx = idx.reshape(-1, 1)
    T = idx.shape[0]
    xf = synth.bf16_bits_to_f32(synth.normal_bf16(12, 0, 0, T * d, 1.0)).reshape(T, d)
    xf[:, 0] = rng.choice([-64.0, -8.0, -4.0, -2.0, 2.0, 4.0, 8.0, 64.0], size=T)
    guf = synth.bf16_bits_to_f32(synth.normal_bf16(12, 2, 0, E * 2 * f * d, 0.05)).reshape(E, 2 * f, d)
    guf[:, :f, 0] = rng.choice([-64.0, -32.0, -8.0, 8.0, 32.0, 64.0], size=(E, f))  # gate rows: g ~ c * x0
    dnf = np.broadcast_to(np.eye(d, dtype=np.float32), (E, d, f)).copy()
    x, gu, dn = (synth.f32_to_bf16_bits(a) for a in (xf, guf, dnf))
    g = xf @ guf[0, :f].T
    assert (g > 100).any() and (g < -100).any() and np.abs(g).max() >= 4000
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, np.ones((T, 1)), np.arange(T))
    for fam in FAMILIES:
        _, _, y = _run(fam, idx, x, gu, dn)
        check_close(bf16_to_host_f32(y), ref, f"saturated SwiGLU ({fam})")

"""Parity of the CUDA path (through the C-ABI) with the CPU oracle, on a B200.

Inputs come from the seeded generator; expected values come only from the oracle. Integer results
(routing indices, counts, offsets, permutation, gathered rows) must match bit for bit; the layer output
must meet the bar in gpu_util (per element and relative Frobenius).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_bits_of, bf16_to_host_f32, check_close, to_dev_bf16

pytestmark = pytest.mark.gpu

N = pytest.importorskip("mixture_experts_ffn_11_b200._native")
from mixture_experts_ffn_11_b200 import MoEFFN  # noqa: E402

NEAR_TIE = 1e-5
CONFIGS = ["tiny", "gpt-oss-20b-prefill", "mixtral-8x7b-prefill", "zipf-128e", "decode-256e-shared"]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    synth.build_cuda()
    torch.cuda.set_device(0)
    N.get_device_error()  # clear
    yield
    torch.cuda.synchronize()


_refs = {}


def layer_ref(name):
    if name not in _refs:
        _refs[name] = oracle.LayerReference(synth.workload(name))
    return _refs[name]


# ---- generator -------------------------------------------------------------------------------------

def test_device_generator_matches_host_bitwise():
    for tid, first, count, sigma in ((0, 0, 100_003, 1.0), (2, 77_777, 50_000, 0.02), (3, 1 << 33, 4096, 0.02)):
        t = torch.empty(count, dtype=torch.bfloat16, device="cuda")
        synth.fill_device(t, 0, tid, first, sigma)
        assert (bf16_bits_of(t) == synth.normal_bf16(0, tid, first, count, sigma)).all()
    t = torch.empty(10_000, dtype=torch.float32, device="cuda")
    synth.fill_device(t, 5, 1, 123, 0.02)
    assert (t.cpu().numpy() == synth.normal_f32(5, 1, 123, 10_000, 0.02)).all()


# ---- routing ---------------------------------------------------------------------------------------

def _gpu_route(wl, x, w_router, bias):
    T, E, k = wl.T, wl.E, wl.k
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    N.route_topk(x, w_router, bias, k, wl.route, logits, idx, w)
    return logits, idx, w


@pytest.mark.parametrize("name", CONFIGS)
def test_router_matches_oracle(name):
    wl = synth.workload(name)
    ref = layer_ref(name)
    x = to_dev_bf16(ref.x)
    wr = torch.from_numpy(ref.w_router).cuda()
    bias = torch.from_numpy(ref.bias).cuda() if ref.bias is not None else None
    logits, idx, w = _gpu_route(wl, x, wr, bias)
    assert N.get_device_error() == 0
    lg = logits.cpu().numpy().astype(np.float64)
    scale = np.abs(ref.logits64).max()
    assert np.abs(lg - ref.logits64).max() <= 1e-5 * max(scale, 1.0)
    ties = set(ref.near_ties(NEAR_TIE).tolist())
    keep = np.array([t for t in range(wl.T) if t not in ties], dtype=np.int64)
    gi = idx.cpu().numpy()
    assert (gi[keep] == ref.idx[keep]).all(), "routing indices differ outside near-ties"
    np.testing.assert_allclose(w.cpu().numpy()[keep], ref.w[keep], rtol=2e-5, atol=2e-6)
    print(f"{name}: {len(ties)} near-tie tokens excluded: {sorted(ties)[:16]}")


@pytest.mark.parametrize("name", CONFIGS)
def test_topk_bit_exact_given_fp32_logits(name):
    """Given the same fp32 logits (the oracle's), selection is identical for every token, no exclusions."""
    wl = synth.workload(name)
    ref = layer_ref(name)
    logits = torch.from_numpy(ref.logits32).cuda()
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device="cuda")
    N.topk_from_logits(logits, wl.k, wl.route, idx, w)
    assert (idx.cpu().numpy() == ref.idx).all()
    np.testing.assert_allclose(w.cpu().numpy(), ref.w, rtol=2e-6, atol=1e-7)


def test_topk_ties_and_modes_small():
    rng = np.random.default_rng(0)
    for E, k in ((8, 2), (33, 5), (256, 8), (1024, 32), (3, 3)):
        l = rng.integers(-2, 3, size=(97, E)).astype(np.float32)  # many exact ties
        for mode in ("topk_softmax", "softmax_topk_renorm", "sigmoid_topk_norm"):
            ri, rw = oracle.topk(l, k, mode)
            idx = torch.empty(97, k, dtype=torch.int32, device="cuda")
            w = torch.empty(97, k, dtype=torch.float32, device="cuda")
            N.topk_from_logits(torch.from_numpy(l).cuda(), k, mode, idx, w)
            assert (idx.cpu().numpy() == ri).all(), (E, k, mode)
            np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


ROUTER_CASES = [
    # T, d, E, k, mode, with bias: both sides of the tensor-core threshold (T >= 2048, E <= 128; top-k fused
    # there, a separate kernel otherwise), padded expert counts, every mode
    (2047, 256, 8, 2, "softmax_topk_renorm", False),
    (2048, 256, 8, 2, "softmax_topk_renorm", True),
    (2100, 520, 100, 8, "topk_softmax", True),
    (3000, 1024, 256, 8, "sigmoid_topk_norm", False),
    (2176, 264, 40, 12, "topk_softmax", True),
    (300, 7168, 256, 8, "sigmoid_topk_norm", True),
    (64, 2880, 32, 4, "topk_softmax", False),
    (1500, 2048, 384, 6, "topk_softmax", False),
    # fused top-k beyond 8 on the tensor-core path, and k = E (every expert selected) with a split-K cluster
    (2500, 1024, 128, 16, "softmax_topk_renorm", True),
    (2300, 640, 17, 17, "sigmoid_topk_norm", False),
]


@pytest.mark.parametrize("T,d,E,k,mode,with_bias", ROUTER_CASES)
def test_router_paths_match_oracle(T, d, E, k, mode, with_bias):
    x = synth.normal_bf16(7, 0, 0, T * d, 1.0).reshape(T, d)
    wr = synth.normal_f32(7, 1, 0, E * d, 0.02).reshape(E, d)
    bias = (synth.normal_f32(7, 4, 0, E, 1.0)) if with_bias else None
    l64 = oracle.router_logits(x, wr, bias)
    idx_ref, w_ref = oracle.topk(l64.astype(np.float32), k, mode)
    margin = oracle.topk_margin(l64, k)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    N.route_topk(to_dev_bf16(x), torch.from_numpy(wr).cuda(), torch.from_numpy(bias).cuda() if with_bias else None,
                 k, mode, logits, idx, w)
    assert N.get_device_error() == 0
    assert np.abs(logits.cpu().numpy() - l64).max() <= 1e-5 * max(np.abs(l64).max(), 1.0)
    keep = margin >= NEAR_TIE
    assert (idx.cpu().numpy()[keep] == idx_ref[keep]).all()
    np.testing.assert_allclose(w.cpu().numpy()[keep], w_ref[keep], rtol=2e-5, atol=2e-6)


def test_router_split_weights_pieces():
    """hi + mid + lo reproduces W_r to the split's bound: hi is W_r truncated to bf16, mid the truncated rest,
    lo the rounded remainder, so |W_r - (hi + mid + lo)| <= 2^-24 |W_r| (and hi, mid exact prefixes)."""
    E, d = 100, 520
    wr = synth.normal_f32(7, 1, 0, E * d, 0.02).reshape(E, d)
    wr[0, :4] = [0.0, -0.0, 1e-30, -3.5]
    wt = torch.from_numpy(wr).cuda()
    pieces = torch.empty(3, E, d, dtype=torch.bfloat16, device="cuda")
    N.router_split_weights(wt, pieces)
    pc = pieces.float().cpu().numpy().astype(np.float64)
    w64 = wr.astype(np.float64)
    assert (np.abs(w64 - pc.sum(0)) <= 2.0 ** -24 * np.abs(w64)).all()
    hi_bits = wr.view(np.uint32) & np.uint32(0xFFFF0000)
    assert (pc[0] == hi_bits.view(np.float32)).all()  # hi = truncation of W_r to its top 16 bits


@pytest.mark.parametrize("T,d,E,k,mode,with_bias", [c for c in ROUTER_CASES if c[0] >= 2048 and c[2] <= 128] +
                         [(300, 7168, 64, 8, "sigmoid_topk_norm", True)])
def test_route_topk_split_is_bit_identical(T, d, E, k, mode, with_bias):
    """The pre-split router gives the same logits, ids and weights as the one that splits W_r itself."""
    x = to_dev_bf16(synth.normal_bf16(8, 0, 0, T * d, 1.0).reshape(T, d))
    wr = torch.from_numpy(synth.normal_f32(8, 1, 0, E * d, 0.02).reshape(E, d)).cuda()
    bias = torch.from_numpy(synth.normal_f32(8, 4, 0, E, 1.0)).cuda() if with_bias else None
    pieces = torch.empty(3, E, d, dtype=torch.bfloat16, device="cuda")
    N.router_split_weights(wr, pieces)
    outs = []
    for split in (False, True):
        lg = torch.empty(T, E, device="cuda")
        idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, k, device="cuda")
        if split:
            N.route_topk_split(x, wr, pieces, bias, k, mode, lg, idx, w)
        else:
            N.route_topk(x, wr, bias, k, mode, lg, idx, w)
        outs.append((lg, idx, w))
    assert N.get_device_error() == 0
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


# ---- permutation -----------------------------------------------------------------------------------

def _gpu_permute(x_bits, idx_np, E):
    T, k = idx_np.shape
    R = T * k
    d = x_bits.shape[1]
    dev = "cuda"
    out = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm_src=torch.empty(R, dtype=torch.int32, device=dev),
               inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
               x_perm=torch.empty(R, d, dtype=torch.bfloat16, device=dev),
               ws=torch.empty(max(N.permute_workspace_size(T, E, k), 256), dtype=torch.uint8, device=dev))
    x = to_dev_bf16(x_bits)
    N.permute(x, torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda(), E, out["counts"],
              out["offsets"], out["perm_src"], out["inv_perm"], out["x_perm"], out["ws"])
    return x, out


@pytest.mark.parametrize("name", CONFIGS)
def test_permute_bit_exact(name):
    wl = synth.workload(name)
    ref = layer_ref(name)
    _, out = _gpu_permute(ref.x, ref.idx, wl.E)
    assert N.get_device_error() == 0
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), ref.counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), ref.offsets)
    np.testing.assert_array_equal(out["perm_src"].cpu().numpy(), ref.perm_src)
    np.testing.assert_array_equal(out["inv_perm"].cpu().numpy(), ref.inv_perm)
    assert (bf16_bits_of(out["x_perm"]) == ref.x[ref.perm_src]).all()


def test_permute_edge_sizes():
    rng = np.random.default_rng(1)
    for T, E, k in ((1, 1, 1), (1, 7, 7), (5000, 3, 2), (4097, 1024, 1), (2048, 16, 16), (9000, 64, 4)):
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        x_bits = synth.normal_bf16(9, 0, 0, T * 8, 1.0).reshape(T, 8)
        _, out = _gpu_permute(x_bits, idx, E)
        c, o, ps, ip = oracle.permute(idx, E)
        np.testing.assert_array_equal(out["counts"].cpu().numpy(), c)
        np.testing.assert_array_equal(out["offsets"].cpu().numpy(), o)
        np.testing.assert_array_equal(out["perm_src"].cpu().numpy(), ps)
        np.testing.assert_array_equal(out["inv_perm"].cpu().numpy(), ip)
        assert (bf16_bits_of(out["x_perm"]) == x_bits[ps]).all()
    assert N.get_device_error() == 0


def test_gather_row_widths():
    """Row gather x_perm = x[perm_src] bit-exact over row widths from one 16-byte vector to 12296 elements,
    including widths that are not a multiple of the 32 lanes x 16 bytes a warp moves per step."""
    rng = np.random.default_rng(4)
    T, E, k = 301, 5, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _, _, ps, _ = oracle.permute(idx, E)
    for d in (8, 2880, 3072, 3080, 6144, 6152, 12288, 12296):
        x_bits = synth.normal_bf16(5, 0, 0, T * d, 1.0).reshape(T, d)
        _, out = _gpu_permute(x_bits, idx, E)
        np.testing.assert_array_equal(out["perm_src"].cpu().numpy(), ps)
        assert (bf16_bits_of(out["x_perm"]) == x_bits[ps]).all(), d
    assert N.get_device_error() == 0


# ---- expert GEMMs + combine on ragged groups ---------------------------------------------------------

def _gpu_experts(x_bits, gu_bits, dn_bits, idx, w32, shared=None):
    """permute -> gate|up -> down -> combine on the GPU for a given routing."""
    T, d = x_bits.shape
    E, two_f, _ = gu_bits.shape
    f = two_f // 2
    k = idx.shape[1]
    R = T * k
    x, p = _gpu_permute(x_bits, idx, E)
    wgu, wdn = to_dev_bf16(gu_bits), to_dev_bf16(dn_bits)
    h = torch.empty(R, f, dtype=torch.bfloat16, device="cuda")
    y_perm = torch.empty(R, d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup(p["x_perm"], wgu, p["offsets"], h)
    N.grouped_gemm_down(h, wdn, p["offsets"], y_perm)
    sh = None
    if shared is not None:
        sgu, sdn = to_dev_bf16(shared[0]), to_dev_bf16(shared[1])
        fs = shared[0].shape[0] // 2
        so = torch.tensor([0, T], dtype=torch.int32, device="cuda")
        hs = torch.empty(T, fs, dtype=torch.bfloat16, device="cuda")
        sh = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        N.grouped_gemm_gateup(x, sgu.unsqueeze(0), so, hs)
        N.grouped_gemm_down(hs, sdn.unsqueeze(0), so, sh)
    N.unpermute_combine(y_perm, p["inv_perm"], torch.from_numpy(w32).cuda(), sh, y)
    assert N.get_device_error() == 0
    return bf16_to_host_f32(y), p


def _routing_with_counts(counts, k, rng):
    """Assignments (T = sum(counts)/k tokens, k distinct experts each) realising the given expert counts."""
    E = len(counts)
    if k == 1:
        idx = np.concatenate([np.full(c, e) for e, c in enumerate(counts)]).astype(np.int32)
        rng.shuffle(idx)
        return idx.reshape(-1, 1)
    raise ValueError("k == 1 only")


RAGGED = [
    # (name, counts per expert, d, f)
    ("empty_single_tail_full", [0, 1, 127, 128, 129, 257, 0], 200, 72),
    ("one_expert_takes_all", [0, 0, 300, 0], 256, 512),
    ("many_small", [3] * 40 + [0] * 24, 64, 96),
    ("wide_k_tail", [130, 5], 1000, 264),
    # CTA-pair kernel (groups average >= 128 rows): 256-row tiles, ragged and empty groups
    ("pair_ragged", [0, 1, 255, 256, 257, 600, 0, 129], 256, 200),
    ("pair_down_240_wide", [300, 0, 700, 45], 480, 136),
    ("pair_one_expert", [0, 0, 2000, 0], 256, 256),
    # last tiles of <= 128 rows run as M=128 pair MMAs: tails of exactly 128, 64, 65 and 1 rows, 240-wide down
    ("pair_half_tails", [128, 384, 64, 65, 320, 0, 256, 257], 264, 136),
    # gate|up whose last N tile is part-filled (f = 360, f = 120 < 128): one and two K blocks per stage
    ("pair_partial_h_tile", [300, 0, 700, 45], 264, 360),
    ("pair_partial_h_tile_two_kblocks", [129, 400, 260], 2112, 120),
    # CTA pair with two accumulators (gate|up K >= 8192, down K >= 2048): 240-wide gate|up; 256-wide down
    ("wide_gateup_240", [300, 0, 700, 45], 8192, 240),
    ("wide_down_256", [400, 1, 129], 512, 8192),
    ("wide_down_240_mid_k", [300, 0, 700, 45], 960, 2880),
    # CTA pair, two K blocks per ring stage (gate|up with K >= 2048), K tail inside the last stage
    ("pair_two_kblocks_per_stage", [0, 300, 1, 257], 4160, 136),
    # single-CTA kernel, 256 wide (many groups of a few rows) and 64 wide (one small group)
    ("single_wide", [2] * 160, 64, 256),
    ("single_group_narrow", [50], 512, 256),
]


@pytest.mark.parametrize("name,counts,d,f", RAGGED, ids=[r[0] for r in RAGGED])
def test_ragged_groups_match_oracle(name, counts, d, f):
    rng = np.random.default_rng(2)
    E = len(counts)
    idx = _routing_with_counts(counts, 1, rng)
    T = idx.shape[0]
    x = synth.normal_bf16(3, 0, 0, T * d, 1.0).reshape(T, d)
    gu = synth.normal_bf16(3, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    dn = synth.normal_bf16(3, 3, 0, E * d * f, 0.05).reshape(E, d, f)
    w = np.ones((T, 1), dtype=np.float32)
    y, p = _gpu_experts(x, gu, dn, idx, w)
    np.testing.assert_array_equal(p["counts"].cpu().numpy(), counts)
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, w.astype(np.float64), np.arange(T))
    check_close(y, ref, name)


def test_k2_random_routing_with_shared_expert():
    rng = np.random.default_rng(3)
    T, d, f, E, k, fs = 333, 128, 384, 5, 2, 136
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.normal_bf16(4, 0, 0, T * d, 1.0).reshape(T, d)
    gu = synth.normal_bf16(4, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    dn = synth.normal_bf16(4, 3, 0, E * d * f, 0.05).reshape(E, d, f)
    sgu = synth.normal_bf16(4, 5, 0, 2 * fs * d, 0.05).reshape(2 * fs, d)
    sdn = synth.normal_bf16(4, 6, 0, d * fs, 0.05).reshape(d, fs)
    y, _ = _gpu_experts(x, gu, dn, idx, w, shared=(sgu, sdn))
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, w.astype(np.float64), np.arange(T), sgu, sdn)
    check_close(y, ref, "k2+shared")


def test_identical_experts_equal_dense_swiglu():
    """All experts equal: the layer is one dense SwiGLU whatever the routing (weights sum to 1)."""
    rng = np.random.default_rng(5)
    T, d, f, E, k = 256, 256, 256, 8, 2
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.normal_bf16(5, 0, 0, T * d, 1.0).reshape(T, d)
    gu1 = synth.normal_bf16(5, 2, 0, 2 * f * d, 0.05).reshape(2 * f, d)
    dn1 = synth.normal_bf16(5, 3, 0, d * f, 0.05).reshape(d, f)
    y, _ = _gpu_experts(x, np.stack([gu1] * E), np.stack([dn1] * E), idx, w)
    ref = oracle.moe_tokens(x, [gu1], [dn1], np.zeros((T, 1), np.int32), np.ones((T, 1)), np.arange(T))
    check_close(y, ref, "identical experts")


# ---- full layer at the benchmark's sizes -------------------------------------------------------------

SAMPLE = {"tiny": None, "gpt-oss-20b-prefill": 48, "mixtral-8x7b-prefill": 24, "zipf-128e": 48,
          "decode-256e-shared": 8, "decode-256e-shared-mxfp4": 8}


def _sample_tokens(ref, n, rng):
    wl = ref.wl
    if n is None:
        return np.arange(wl.T)
    toks = set(rng.choice(wl.T, size=n, replace=False).tolist())
    nonempty = np.nonzero(ref.counts)[0]
    for e in (nonempty[np.argmin(ref.counts[nonempty])], int(np.argmax(ref.counts))):
        rows = np.nonzero((ref.idx == e).any(axis=1))[0]
        toks.update(rng.choice(rows, size=min(8, len(rows)), replace=False).tolist())
    return np.array(sorted(toks), dtype=np.int32)


@pytest.mark.parametrize("name", CONFIGS + ["decode-256e-shared-mxfp4"])
def test_full_layer_matches_oracle(name):
    wl = synth.workload(name)
    ref = layer_ref(name)
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"],
                   inp["w_gateup_shared"], inp["w_down_shared"], weights=wl.weights)
    y = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    # the device inputs are the oracle's inputs
    assert (bf16_bits_of(inp["x"]) == ref.x).all()
    gi = layer.buf["topk_idx"].cpu().numpy()
    ties = set(ref.near_ties(NEAR_TIE).tolist())
    toks = [t for t in _sample_tokens(ref, SAMPLE[name], np.random.default_rng(0)) if t not in ties]
    toks = np.array(toks, dtype=np.int32)
    assert (gi[toks] == ref.idx[toks]).all()
    yh = bf16_to_host_f32(y)[toks]
    want = ref.outputs(toks)
    fro = check_close(yh, want, name)
    print(f"{name}: {len(toks)} tokens compared, relative Frobenius error {fro:.2e}")
    # run again: bitwise identical (deterministic path)
    y2 = layer(inp["x"])
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))


# ---- MXFP4 expert weights -----------------------------------------------------------------------------

def _gpu_quantize(w_bits):
    w = to_dev_bf16(w_bits)
    G, Nr, K = w.shape
    q = torch.empty(G, Nr, K // 2, dtype=torch.uint8, device="cuda")
    sc = torch.empty(G, K // 32, Nr, dtype=torch.uint8, device="cuda")
    N.mxfp4_quantize(w, q, sc)
    return q, sc


def test_mxfp4_quantize_bit_exact():
    """The encoder against the oracle, byte for byte: normal weights, zero blocks, signed zeros, bf16 subnormals,
    huge magnitudes, the golden tie cases, and every code and scale range through a decode-encode round trip."""
    rng = np.random.default_rng(30)
    cases = []
    w = synth.normal_bf16(30, 2, 0, 3 * 200 * 96, 0.02).reshape(3, 200, 96)
    w[0, 0, :32] = 0
    w[0, 1, :32] = 0x8000
    w[1, 2, 32:64] = (rng.integers(1, 128, 32) | (rng.integers(0, 2, 32) << 15)).astype(np.uint16)  # subnormals
    w[2, 3, 64:] = synth.f32_to_bf16_bits(rng.standard_normal(32).astype(np.float32) * 3e37)
    cases.append(w)
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mxfp4_e2m1.json")))["rounding"]
    vals = [(-0.0 if v == "-0" else float(v)) for v in g["inputs"]] + [0.0] * (32 - len(g["inputs"]))
    cases.append(synth.f32_to_bf16_bits(np.array(vals, dtype=np.float32)).reshape(1, 1, 32))
    codes = rng.integers(0, 16, size=(2, 48, 128))
    codes[..., ::32] = rng.choice([6, 7, 14, 15], size=(2, 48, 4))
    scales = rng.integers(0, 253, size=(2, 4, 48)).astype(np.uint8)
    cases.append(oracle.mxfp4_dequantize(_pack_codes_layout(codes), scales))  # exact E2M1 values times scales
    cases.append(synth.normal_bf16(31, 3, 0, 4 * 7168 * 64, 0.02).reshape(4, 64, 7168))
    for w in cases:
        q, sc = _gpu_quantize(w)
        rq, rs = oracle.mxfp4_quantize(w)
        np.testing.assert_array_equal(q.cpu().numpy(), rq)
        np.testing.assert_array_equal(sc.cpu().numpy(), rs)
    assert N.get_device_error() == 0


def _pack_codes_layout(codes):
    c = np.asarray(codes, dtype=np.uint32)
    *lead, K = c.shape
    c = c.reshape(*lead, K // 8, 4, 2)
    shifts = (np.arange(4, dtype=np.uint32) * 4)[:, None] + np.array([0, 16], dtype=np.uint32)[None, :]
    return (c << shifts).sum(axis=(-1, -2)).astype("<u4").view(np.uint8).reshape(*lead, K // 2)


def _gpu_experts_mxfp4(x_bits, gu_bits, dn_bits, idx, w32, shared=None):
    """permute -> MXFP4 gate|up -> MXFP4 down -> combine on the GPU, weights encoded on the GPU."""
    T, d = x_bits.shape
    E, two_f, _ = gu_bits.shape
    f = two_f // 2
    R = T * idx.shape[1]
    x, p = _gpu_permute(x_bits, idx, E)
    qgu, sgu = _gpu_quantize(gu_bits)
    qdn, sdn = _gpu_quantize(dn_bits)
    h = torch.empty(R, f, dtype=torch.bfloat16, device="cuda")
    y_perm = torch.empty(R, d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup_mxfp4(p["x_perm"], qgu, sgu, p["offsets"], h)
    N.grouped_gemm_down_mxfp4(h, qdn, sdn, p["offsets"], y_perm)
    sh = None
    if shared is not None:
        fs = shared[0].shape[0] // 2
        q1, s1 = _gpu_quantize(shared[0][None])
        q2, s2 = _gpu_quantize(shared[1][None])
        so = torch.tensor([0, T], dtype=torch.int32, device="cuda")
        hs = torch.empty(T, fs, dtype=torch.bfloat16, device="cuda")
        sh = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        N.grouped_gemm_gateup_mxfp4(x, q1, s1, so, hs)
        N.grouped_gemm_down_mxfp4(hs, q2, s2, so, sh)
    N.unpermute_combine(y_perm, p["inv_perm"], torch.from_numpy(w32).cuda(), sh, y)
    assert N.get_device_error() == 0
    return bf16_to_host_f32(y), p, h


MXFP4_RAGGED = [
    # (name, counts per expert, d, f): token tiles of 16 (M <= 8 G), 32 (M <= 24 G) and 64 rows, groups larger than
    # the tile, empty groups, weight blocks cut by f or d (not multiples of 128), K tails inside the last 256-stage
    ("nt16_decode_like", [2, 0, 1, 3, 2, 0, 5, 16, 17, 1], 256, 128),
    ("nt16_tails", [1, 0, 9, 0, 2, 33], 288, 96),
    ("nt32_ragged", [20, 0, 31, 33, 1, 40], 160, 224),
    ("nt64_one_group", [200], 352, 160),
    ("nt64_many", [0, 65, 64, 130, 7], 512, 544),
    # the warp-MMA decode kernel at its limits: 1024 groups (group tables sized by G), K = 8192 (the whole token
    # rows of a tile in shared memory, a 2-stage ring), and K = 8224 just past it (gate|up on the tensor-memory
    # kernel, down on the warp kernel)
    ("warp_1024_groups", [2] * 1024, 64, 64),
    ("warp_k_8192", [3, 5, 0, 2], 8192, 64),
    ("past_warp_k_limit", [3, 5, 0, 2], 8224, 64),
]


@pytest.mark.parametrize("name,counts,d,f", MXFP4_RAGGED, ids=[r[0] for r in MXFP4_RAGGED])
def test_mxfp4_ragged_groups_match_oracle(name, counts, d, f):
    rng = np.random.default_rng(32)
    E = len(counts)
    idx = _routing_with_counts(counts, 1, rng)
    T = idx.shape[0]
    x = synth.normal_bf16(33, 0, 0, T * d, 1.0).reshape(T, d)
    gu = synth.normal_bf16(33, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    dn = synth.normal_bf16(33, 3, 0, E * d * f, 0.05).reshape(E, d, f)
    w = np.ones((T, 1), dtype=np.float32)
    y, p, _ = _gpu_experts_mxfp4(x, gu, dn, idx, w)
    np.testing.assert_array_equal(p["counts"].cpu().numpy(), counts)
    gu_dq = oracle.mxfp4_round_trip(gu)
    dn_dq = oracle.mxfp4_round_trip(dn)
    ref = oracle.moe_tokens(x, list(gu_dq), list(dn_dq), idx, w.astype(np.float64), np.arange(T))
    check_close(y, ref, name)


def test_mxfp4_large_scales_and_shared_expert():
    """Scale codes above 128 (the decoder's two-step multiply) next to ordinary ones, k = 2 routing with
    weights, and an MXFP4 shared expert; the encoded weights are exact E2M1 values times the scales."""
    rng = np.random.default_rng(34)
    T, d, f, E, k, fs = 90, 256, 160, 6, 2, 96
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    wts = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.f32_to_bf16_bits((rng.standard_normal((T, d)) * 1e-3).astype(np.float32))

    def encoded(shape, lo, hi):
        G, Nr, K = shape
        codes = rng.integers(0, 16, size=shape)
        codes[..., ::32] = rng.choice([6, 7, 14, 15], size=(G, Nr, K // 32))
        scales = rng.integers(lo, hi, size=(G, K // 32, Nr)).astype(np.uint8)
        return oracle.mxfp4_dequantize(_pack_codes_layout(codes), scales)

    gu = encoded((E, 2 * f, d), 100, 140)   # weights up to 6 * 2^12
    dn = encoded((E, d, f), 110, 131)
    sgu = encoded((1, 2 * fs, d), 115, 135)[0]
    sdn = encoded((1, d, fs), 118, 130)[0]
    y, _, _ = _gpu_experts_mxfp4(x, gu, dn, idx, wts, shared=(sgu, sdn))
    # the weights are their own encoding, so the oracle uses them as they are
    ref = oracle.moe_tokens(x, list(gu), list(dn), idx, wts.astype(np.float64), np.arange(T), sgu, sdn)
    check_close(y, ref, "mxfp4 large scales + shared")


def test_mxfp4_layer_folds_shared_expert_into_routed_gemms():
    """A decode-sized MXFP4 layer whose shared expert is as wide as a routed one computes the shared expert as group
    E of the routed GEMM launches (its rows after the routed rows): every token against the oracle, and the same
    layer with the shared expert run on its own within the same bar."""
    wl = synth.Workload(**{**synth.workload("tiny").__dict__, "name": "tiny-mxfp4-shared", "E": 32, "shared_f": 512,
                           "weights": "mxfp4", "route": "sigmoid_topk_norm"})
    ref = oracle.LayerReference(wl)
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"],
                   inp["w_gateup_shared"], inp["w_down_shared"], weights="mxfp4")
    twin = layer.sibling()
    twin.fold_shared = False
    assert layer._fold(wl.T) and not twin._fold(wl.T)
    assert layer.kernel_launches(wl.T) == twin.kernel_launches(wl.T) - 1
    y = bf16_to_host_f32(layer(inp["x"]).clone())
    y_own = bf16_to_host_f32(twin(inp["x"]).clone())
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    ties = set(ref.near_ties(NEAR_TIE).tolist())
    toks = np.array([t for t in range(wl.T) if t not in ties], dtype=np.int32)
    assert len(toks) >= wl.T - 4
    assert (layer.buf["topk_idx"].cpu().numpy()[toks] == ref.idx[toks]).all()
    want = ref.outputs(toks)
    check_close(y[toks], want, "shared expert folded into the routed GEMMs")
    check_close(y_own[toks], want, "shared expert on its own")


def test_mxfp4_gateup_matches_bf16_gemm_on_decoded_weights():
    """Decode-shaped problem: h from the MXFP4 kernel equals h from the bf16 grouped GEMM given the decoded
    weights, up to fp32 summation order (both round h to bf16 from fp32 sums of the same products)."""
    rng = np.random.default_rng(35)
    counts = [int(c) for c in rng.multinomial(512, np.ones(256) / 256)]
    idx = _routing_with_counts(counts, 1, rng)
    T, d, f = idx.shape[0], 1024, 256
    x_bits = synth.normal_bf16(35, 0, 0, T * d, 1.0).reshape(T, d)
    gu = synth.normal_bf16(35, 2, 0, 256 * 2 * f * d, 0.02).reshape(256, 2 * f, d)
    _, p = _gpu_permute(x_bits, idx, 256)
    q, sc = _gpu_quantize(gu)
    h4 = torch.empty(T, f, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup_mxfp4(p["x_perm"], q, sc, p["offsets"], h4)
    hb = torch.empty(T, f, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup(p["x_perm"], to_dev_bf16(oracle.mxfp4_round_trip(gu)), p["offsets"], hb)
    a, b = bf16_to_host_f32(h4).astype(np.float64), bf16_to_host_f32(hb).astype(np.float64)
    assert np.abs(a - b).max() <= 2 ** -7 * np.abs(b).max() + 1e-6
    assert N.get_device_error() == 0


def test_layer_at_maximum_sizes():
    """The API's largest routing sizes through the whole layer: E = 1024 experts, k = 32 per token (router on
    CUDA cores + the stand-alone top-k, 1024-group permute and GEMMs), every token against the oracle."""
    wl = synth.workload("tiny", T=300, d=128, f=64, E=1024, k=32, route="softmax_topk_renorm")
    ref = oracle.LayerReference(wl)
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"])
    y = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    np.testing.assert_array_equal(layer.buf["counts"].cpu().numpy(), ref.counts)
    ties = set(ref.near_ties(NEAR_TIE).tolist())
    toks = np.array([t for t in range(wl.T) if t not in ties], dtype=np.int32)
    assert len(toks) > wl.T // 2
    assert (layer.buf["topk_idx"].cpu().numpy()[toks] == ref.idx[toks]).all()
    check_close(bf16_to_host_f32(y)[toks], ref.outputs(toks), "E=1024, k=32")


@pytest.mark.parametrize("T,d,f,E,k,route", [
    (5, 8, 8, 3, 3, "softmax_topk_renorm"),  # smallest dims the API takes, k = E (every expert selected)
    (1, 64, 16, 1, 1, "topk_softmax"),       # one token, one expert: a dense SwiGLU with weight 1
    (7, 16, 24, 4, 2, "sigmoid_topk_norm"),  # d, f not multiples of 16
])
def test_layer_degenerate_shapes(T, d, f, E, k, route):
    wl = synth.workload("tiny", T=T, d=d, f=f, E=E, k=k, route=route)
    ref = oracle.LayerReference(wl)
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"])
    y = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    ties = set(ref.near_ties(NEAR_TIE).tolist())
    toks = np.array([t for t in range(T) if t not in ties], dtype=np.int32)
    assert (layer.buf["topk_idx"].cpu().numpy()[toks] == ref.idx[toks]).all()
    check_close(bf16_to_host_f32(y)[toks], ref.outputs(toks), f"T={T} d={d} f={f} E={E} k={k}")


def test_layer_empty_batch():
    """T = 0: every call returns at once and the output is empty (no launch reads an empty buffer)."""
    wl = synth.workload("tiny")
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"])
    y = layer(inp["x"][:0].contiguous())
    torch.cuda.synchronize()
    assert tuple(y.shape) == (0, wl.d)
    assert layer.kernel_launches(0) == 0
    assert N.get_device_error() == 0
    # and a normal batch afterwards still matches the first call of the same inputs
    a = layer(inp["x"]).clone()
    b = layer(inp["x"]).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_layer_is_deterministic():
    wl = synth.workload("gpt-oss-20b-prefill", T=1024)
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route)
    a = layer(inp["x"]).clone()
    b = layer(inp["x"]).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # permuting the tokens permutes the output rows exactly (rows never interact)
    perm = torch.randperm(wl.T, generator=torch.Generator().manual_seed(0)).cuda()
    c = layer(inp["x"][perm].contiguous()).clone()
    assert torch.equal(c.view(torch.int16), a[perm].view(torch.int16))


# ---- device-side anomalies are reported, not faulted -------------------------------------------------

def test_expert_id_out_of_range_is_flagged():
    T, E, k, d = 100, 4, 2, 16
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[7, 1] = E  # out of range
    x_bits = synth.normal_bf16(1, 0, 0, T * d, 1.0).reshape(T, d)
    _gpu_permute(x_bits, idx, E)
    err = N.get_device_error()
    assert err & 0x2
    assert N.get_device_error() == 0  # read clears


def test_bad_group_offsets_are_flagged():
    M, d, f = 200, 64, 64
    a = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3, 2 * f, d, dtype=torch.bfloat16, device="cuda")
    h = torch.zeros(M, f, dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, 100, 50, 500], dtype=torch.int32, device="cuda")  # decreasing, and past M
    N.grouped_gemm_gateup(a, w, offs, h)
    assert N.get_device_error() & 0x4

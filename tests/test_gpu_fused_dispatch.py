"""Dispatch and collect folded into the grouped GEMMs, B200: moe_grouped_gemm_gateup_gather (row gather in the
gate|up operand load), moe_grouped_gemm_down_combine (weighted combine in the down epilogue) and the stand-alone
row gather (moe_gather_rows).

The gathering GEMM reads row r of its operand as x[perm_src[r]] with TMA gather4 loads instead of reading a
grouped copy x_perm; the MMA and the epilogue are those of the swap kernel, so h must equal, bit for bit, the h of
moe_permute's gather followed by moe_grouped_gemm_gateup. The combining GEMM finishes each token in the tile that
brings its last slot, summing the slots in order with the combine kernel's arithmetic, so y_perm and y must equal
those of moe_grouped_gemm_down followed by moe_unpermute_combine, bit for bit, whatever order the tiles ran in.
Small problems (fewer than 128 rows per group on average) take the unfused paths.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_host_f32, check_close, to_dev_bf16
from test_gpu_gemm_kernels import CASES

pytestmark = pytest.mark.gpu

N = pytest.importorskip("mixture_experts_ffn_11_b200._native")
DEVERR_ROW_RANGE = 0x8  # MOE_DEVERR_ROW_RANGE in include/moe.h


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    torch.cuda.set_device(0)
    N.get_device_error()
    yield
    N.set_gemm_kernel("auto")


def _routing(counts, k, seed, E=None):
    """topk_idx: with k = 1, [sum(counts), 1] with expert e chosen counts[e] times; else [counts, k] (counts = T)
    with k distinct random experts of E per token."""
    rng = np.random.default_rng(seed)
    if k == 1:
        idx = np.concatenate([np.full(c, e) for e, c in enumerate(counts)]).astype(np.int32)
        rng.shuffle(idx)
        return idx.reshape(-1, 1)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(counts)]).astype(np.int32)


def _group(x_bits, idx, E):
    T, d = x_bits.shape
    k = idx.shape[1]
    R = T * k
    dev = "cuda"
    p = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
             offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
             perm_src=torch.empty(R, dtype=torch.int32, device=dev),
             inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
             x_perm=torch.empty(R, d, dtype=torch.bfloat16, device=dev),
             ws=torch.empty(max(N.permute_workspace_size(T, E, k), 256), dtype=torch.uint8, device=dev))
    x = to_dev_bf16(x_bits)
    N.permute(x, torch.from_numpy(idx).cuda(), E, p["counts"], p["offsets"], p["perm_src"], p["inv_perm"],
              p["x_perm"], p["ws"])
    return x, p


def _gather_h(x, p, w, f):
    R = p["perm_src"].shape[0]
    E = w.shape[0]
    d = x.shape[1]
    h = torch.full((R, f), float("nan"), dtype=torch.bfloat16, device="cuda")
    nws = N.grouped_gemm_gateup_gather_workspace_size(E, R, d)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda") if nws else None
    N.grouped_gemm_gateup_gather(x, p["perm_src"], w, p["offsets"], h, ws)
    return h, nws


@pytest.mark.parametrize("name,counts,d,f", CASES, ids=[c[0] for c in CASES])
def test_gather_gemm_bitwise_equals_grouped_copy(name, counts, d, f):
    idx = _routing(counts, 1, 2)
    E = len(counts)
    x_bits = synth.normal_bf16(3, 0, 0, idx.shape[0] * d, 1.0).reshape(-1, d)
    gu_bits = synth.normal_bf16(3, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    x, p = _group(x_bits, idx, E)
    w = to_dev_bf16(gu_bits)
    h_ref = torch.empty(idx.shape[0], f, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup(p["x_perm"], w, p["offsets"], h_ref)
    h, nws = _gather_h(x, p, w, f)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    assert (nws == 0) == (idx.shape[0] >= 128 * E), name
    assert not torch.isnan(h.float()).any(), f"{name}: rows of h left unwritten"
    assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16)), f"{name}: gathered h differs"


@pytest.mark.parametrize("T,E,k,d,f", [(700, 5, 4, 256, 136), (300, 2, 2, 2880, 192), (64, 16, 4, 128, 64)],
                         ids=["k4_swap_path", "gpt_oss_width", "workspace_path"])
def test_gather_gemm_repeated_tokens_match_oracle(T, E, k, d, f):
    """k > 1: every token row is read by k groups. The layer output through the gathering GEMM meets the parity
    bar against the oracle, and h equals the grouped-copy path bit for bit."""
    idx = _routing(T, k, 5, E)
    x_bits = synth.normal_bf16(4, 0, 0, T * d, 1.0).reshape(T, d)
    gu_bits = synth.normal_bf16(4, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d)
    dn_bits = synth.normal_bf16(4, 3, 0, E * d * f, 0.05).reshape(E, d, f)
    x, p = _group(x_bits, idx, E)
    w = to_dev_bf16(gu_bits)
    h, _ = _gather_h(x, p, w, f)
    h_ref = torch.empty_like(h)
    N.grouped_gemm_gateup(p["x_perm"], w, p["offsets"], h_ref)
    R = T * k
    y_perm = torch.empty(R, d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_down(h, to_dev_bf16(dn_bits), p["offsets"], y_perm)
    N.unpermute_combine(y_perm, p["inv_perm"], torch.ones(T, k, dtype=torch.float32, device="cuda"), None, y)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16))
    ref = oracle.moe_tokens(x_bits, list(gu_bits), list(dn_bits), idx, np.ones((T, k)), np.arange(T))
    check_close(bf16_to_host_f32(y), ref, f"gathered gate|up, T={T} E={E} k={k}")


@pytest.mark.parametrize("R_per_group", [200, 3], ids=["swap_path", "workspace_path"])
def test_gather_gemm_row_out_of_range_flagged(R_per_group):
    """A row_src entry outside [0, T) is flagged (MOE_DEVERR_ROW_RANGE); every other row of h is unaffected."""
    E, d, f = 2, 128, 64
    R = R_per_group * E
    T = R
    x_bits = synth.normal_bf16(6, 0, 0, T * d, 1.0).reshape(T, d)
    x = to_dev_bf16(x_bits)
    w = to_dev_bf16(synth.normal_bf16(6, 2, 0, E * 2 * f * d, 0.05).reshape(E, 2 * f, d))
    offsets = torch.tensor([0, R_per_group, R], dtype=torch.int32, device="cuda")
    src = torch.randperm(T, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    bad = src.clone()
    bad[5] = T  # out of range
    good = src.clone()
    good[5] = 0
    h_bad, _ = _gather_h(x, {"perm_src": bad.cuda(), "offsets": offsets}, w, f)
    torch.cuda.synchronize()
    assert N.get_device_error() & DEVERR_ROW_RANGE
    h_good, _ = _gather_h(x, {"perm_src": good.cuda(), "offsets": offsets}, w, f)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    keep = torch.ones(R, dtype=torch.bool, device="cuda")
    keep[5] = False
    assert torch.equal(h_bad.view(torch.int16)[keep], h_good.view(torch.int16)[keep])


def test_gather_rows_exact():
    T, d, R = 37, 72, 100
    x_bits = synth.normal_bf16(8, 0, 0, T * d, 1.0).reshape(T, d)
    src = np.random.default_rng(3).integers(0, T, size=R).astype(np.int32)
    src[7] = -1  # out of range: zero row, flagged
    out = torch.full((R, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    N.gather_rows(to_dev_bf16(x_bits), torch.from_numpy(src).cuda(), out)
    torch.cuda.synchronize()
    assert N.get_device_error() & DEVERR_ROW_RANGE
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for r in range(R):
        want = x_bits[src[r]] if 0 <= src[r] < T else np.zeros(d, dtype=np.uint16)
        assert np.array_equal(got[r], want), r


def _down_combine_case(idx, E, d, f, seed, with_shared):
    T, k = idx.shape
    R = T * k
    x_bits = synth.normal_bf16(seed, 0, 0, T * d, 1.0).reshape(T, d)
    x, p = _group(x_bits, idx, E)
    h = to_dev_bf16(synth.normal_bf16(seed, 7, 0, R * f, 1.0).reshape(R, f))
    w = to_dev_bf16(synth.normal_bf16(seed, 3, 0, E * d * f, 0.05).reshape(E, d, f))
    rng = np.random.default_rng(seed)
    tw = torch.from_numpy(rng.uniform(0.05, 1.0, size=(T, k)).astype(np.float32)).cuda()
    shared = to_dev_bf16(synth.normal_bf16(seed, 8, 0, T * d, 1.0).reshape(T, d)) if with_shared else None
    yp_ref = torch.empty(R, d, dtype=torch.bfloat16, device="cuda")
    y_ref = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_down(h, w, p["offsets"], yp_ref)
    N.unpermute_combine(yp_ref, p["inv_perm"], tw, shared, y_ref)
    ws = torch.empty(N.grouped_gemm_down_combine_workspace_size(T, d), dtype=torch.uint8, device="cuda")
    ws.fill_(0x5A)  # the call clears what it uses
    outs = []
    for _ in range(2):
        yp = torch.full((R, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        y = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        N.grouped_gemm_down_combine(h, w, p["offsets"], p["perm_src"], p["inv_perm"], tw, shared, yp, y, ws)
        outs.append((yp, y))
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    for yp, y in outs:
        assert torch.equal(yp.view(torch.int16), yp_ref.view(torch.int16)), "y_perm differs"
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "y differs"


@pytest.mark.parametrize("name,counts,d,f", CASES, ids=[c[0] for c in CASES])
def test_down_combine_bitwise_equals_separate_k1(name, counts, d, f):
    _down_combine_case(_routing(counts, 1, 2), len(counts), d, f, 9, False)


@pytest.mark.parametrize("T,E,k,d,f,shared", [
    (700, 5, 4, 256, 136, False),   # every token finished by one of four tiles
    (640, 4, 4, 200, 64, True),     # d = 200: the last 32-column block holds 8 columns; shared expert added
    (300, 2, 2, 2880, 192, False),  # gpt-oss width: 90 column blocks, 12 weight blocks
    (1024, 8, 8, 512, 128, True),   # k = 8
    (64, 16, 4, 128, 64, False),    # fewer than 128 rows per group: the unfused path
], ids=["k4", "d200_shared", "gpt_oss_width", "k8_shared", "unfused_path"])
def test_down_combine_bitwise_equals_separate(T, E, k, d, f, shared):
    _down_combine_case(_routing(T, k, 11, E), E, d, f, 10, shared)


def test_down_combine_rejects_bad_sizes():
    h = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(1, 64, 64, dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    i32 = torch.zeros(8, dtype=torch.int32, device="cuda")
    tw = torch.ones(3, 2, dtype=torch.float32, device="cuda")  # T*k = 6 != M = 8
    y = torch.empty(3, 64, dtype=torch.bfloat16, device="cuda")
    yp = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(N.MoEError):
        N.grouped_gemm_down_combine(h, w, off, i32, i32, tw, None, yp, y, ws)


@pytest.mark.parametrize("name,over", [
    ("gpt-oss-20b-prefill", {"T": 1024}),
    ("zipf-128e", {"T": 2048}),
    ("decode-256e-shared", {"T": 4096, "d": 256, "f": 128, "shared_f": 64}),
], ids=["gpt_oss_T1024", "zipf_T2048", "shared_expert_prefill"])
def test_fused_layer_bitwise_equals_separate(name, over):
    """MoEFFN(fused=True) against the default layer on prefill-shaped routing: the same output bits, and the
    backward after a fused forward (which gathers x_perm itself) gives the same gradients."""
    from mixture_experts_ffn_11_b200 import MoEFFN

    wl = synth.workload(name, **over)
    inp = synth.device_inputs(wl)
    args = (inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"], inp["w_gateup_shared"],
            inp["w_down_shared"])
    plain, fused = MoEFFN(*args), MoEFFN(*args, fused=True)
    assert fused._fused(wl.T) and not plain._fused(wl.T)
    y0 = plain(inp["x"]).clone()
    y1 = fused(inp["x"]).clone()
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    dy = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    synth.fill_device(dy, wl.seed, synth.TID_DY, 0, synth.X_SIGMA)
    g0 = {k: v.clone() for k, v in plain.backward(dy).items() if v is not None}
    g1 = fused.backward(dy)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    for key, v in g0.items():
        assert torch.equal(v.view(torch.int16) if v.dtype == torch.bfloat16 else v, g1[key].view(torch.int16)
                           if g1[key].dtype == torch.bfloat16 else g1[key]), key


def test_empty_problems_launch_nothing():
    """Zero rows: the gathering, combining and saving GEMMs and the row gather return at once (no launch, no
    device error), as the other entry points do."""
    dev = "cuda"
    bf = torch.bfloat16
    x = torch.empty(0, 64, dtype=bf, device=dev)
    w = torch.zeros(2, 128, 64, dtype=bf, device=dev)
    wd = torch.zeros(2, 64, 64, dtype=bf, device=dev)
    off = torch.zeros(3, dtype=torch.int32, device=dev)
    src = torch.empty(0, dtype=torch.int32, device=dev)
    h = torch.empty(0, 64, dtype=bf, device=dev)
    gu = torch.empty(0, 128, dtype=bf, device=dev)
    N.grouped_gemm_gateup_gather(x, src, w, off, h, None)
    N.grouped_gemm_gateup_save(x, w, off, h, gu)
    N.gather_rows(x, src, torch.empty(0, 64, dtype=bf, device=dev))
    tw = torch.empty(0, 2, dtype=torch.float32, device=dev)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    N.grouped_gemm_down_combine(h, wd, off, src, src, tw, None, torch.empty(0, 64, dtype=bf, device=dev),
                                torch.empty(0, 64, dtype=bf, device=dev), ws)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0

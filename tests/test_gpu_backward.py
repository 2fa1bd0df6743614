"""Backward pass of the MoE layer on a B200, through the C-ABI, against the CPU oracle.

The oracle's backward (moe_backward, router_backward, weight_grad_entries, LayerReference.input_grad) is pinned by
fp64 autograd and finite differences on the CPU (tests/test_oracle_pins.py). Here the GPU gradients of whole layer
calls are compared with it at the forward's parity bar (gpu_util.check_close); the building blocks are checked
alone against fp64 numpy on small ragged problems.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_bits_of, bf16_to_host_f32, check_close, to_dev_bf16

pytestmark = pytest.mark.gpu

N = pytest.importorskip("mixture_experts_ffn_11_b200._native")
from mixture_experts_ffn_11_b200 import MoEFFN  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    synth.build_cuda()
    torch.cuda.set_device(0)
    N.get_device_error()
    yield
    torch.cuda.synchronize()


def _f64(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def _ragged(counts, seed):
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return offs, rng


# ---- building blocks -------------------------------------------------------------------------------------

def test_transpose_weights_exact():
    G, R, C = 3, 200, 136
    w = synth.normal_bf16(21, 2, 0, G * R * C, 1.0).reshape(G, R, C)
    wt = torch.empty(G, C, R, dtype=torch.bfloat16, device="cuda")
    N.transpose_weights(to_dev_bf16(w), wt)
    assert (bf16_bits_of(wt) == w.transpose(0, 2, 1)).all()


@pytest.mark.parametrize("counts,d,f", [([0, 1, 127, 300, 45, 0], 200, 136), ([447, 569, 0, 512], 2880, 2880)])
def test_gateup_preactivations_match_fp64(counts, d, f):
    offs, _ = _ragged(counts, 0)
    M, G = int(offs[-1]), len(counts)
    a = synth.normal_bf16(22, 0, 0, M * d, 1.0).reshape(M, d)
    w = synth.normal_bf16(22, 2, 0, G * 2 * f * d, 0.05).reshape(G, 2 * f, d)
    gu = torch.full((M, 2 * f), float("nan"), dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup_preact(to_dev_bf16(a), to_dev_bf16(w), torch.from_numpy(offs).cuda(), gu)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    got = bf16_to_host_f32(gu)
    af, wf = _f64(a), _f64(w)
    rows = np.concatenate([np.arange(offs[g], min(offs[g + 1], offs[g] + 40)) for g in range(G)])  # rows of every group
    want = np.stack([af[r] @ wf[np.searchsorted(offs, r, side="right") - 1].T for r in rows])
    check_close(got[rows], want, "gate|up pre-activations")


def test_swiglu_backward_matches_fp64():
    M, f = 300, 136
    dh = synth.normal_bf16(23, 0, 0, M * f, 1.0).reshape(M, f)
    gu = synth.normal_bf16(23, 1, 0, M * 2 * f, 4.0).reshape(M, 2 * f)
    gu[0, :8] = synth.f32_to_bf16_bits(np.array([-200, -90, -30, 0, 30, 90, 200, -0.0], dtype=np.float32))
    dgu = torch.empty(M, 2 * f, dtype=torch.bfloat16, device="cuda")
    N.swiglu_backward(to_dev_bf16(dh), to_dev_bf16(gu), dgu)
    got = bf16_to_host_f32(dgu).astype(np.float64)
    h, g, u = _f64(dh), _f64(gu[:, :f]), _f64(gu[:, f:])
    s = 0.5 * (1.0 + np.tanh(0.5 * g))  # logistic function, overflow-free
    want = np.concatenate([h * u * s * (1 + g * (1 - s)), h * g * s], axis=1)
    check_close(got, want, "SwiGLU derivative")


def test_permute_backward_matches_fp64():
    rng = np.random.default_rng(24)
    T, d, E, k = 333, 264, 9, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _, _, perm_src, inv_perm = oracle.permute(idx, E)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    dy = synth.normal_bf16(24, 7, 0, T * d, 1.0).reshape(T, d)
    yp = synth.normal_bf16(24, 3, 0, T * k * d, 1.0).reshape(T * k, d)
    dy_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    N.permute_backward(to_dev_bf16(dy), torch.from_numpy(inv_perm).cuda(), torch.from_numpy(w).cuda(),
                       to_dev_bf16(yp), dy_perm, dw)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    a = np.arange(T * k)
    t, r = a // k, inv_perm
    want_dyp = np.zeros((T * k, d))
    want_dyp[r] = w.reshape(-1, 1).astype(np.float64) * _f64(dy)[t]
    check_close(bf16_to_host_f32(dy_perm), want_dyp, "dy_perm")
    want_dw = (_f64(dy)[t] * _f64(yp)[r]).sum(axis=1).reshape(T, k)
    np.testing.assert_allclose(dw.cpu().numpy(), want_dw, rtol=1e-4, atol=1e-3)


@pytest.mark.parametrize("counts,P,Q", [([0, 1, 63, 64, 65, 300, 0], 200, 136), ([447, 0, 569], 2880, 264),
                                        ([5] * 40, 64, 96)])
def test_grouped_weight_grad_matches_fp64(counts, P, Q):
    offs, _ = _ragged(counts, 1)
    M, G = int(offs[-1]), len(counts)
    a = synth.normal_bf16(25, 0, 0, M * P, 1.0).reshape(M, P)
    b = synth.normal_bf16(25, 1, 0, M * Q, 1.0).reshape(M, Q)
    dw = torch.full((G, P, Q), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(N.grouped_weight_grad_workspace_size(M, G, P, Q), dtype=torch.uint8, device="cuda")
    N.grouped_weight_grad(to_dev_bf16(a), to_dev_bf16(b), torch.from_numpy(offs).cuda(), dw, ws)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    got = dw.cpu().numpy().astype(np.float64)
    af, bf = _f64(a), _f64(b)
    for g in range(G):
        want = af[offs[g]:offs[g + 1]].T @ bf[offs[g]:offs[g + 1]]
        if counts[g] == 0:
            assert (got[g] == 0).all(), f"empty group {g} not zero"
        else:
            check_close(got[g], want, f"dW of group {g}")


# ---- the layer ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("counts,d,f", [([0, 1, 127, 300, 45, 0], 200, 136), ([447, 569, 0, 512], 2880, 2880),
                                         ([3, 0, 5, 2], 256, 128)],
                         ids=["ragged_small", "gpt_oss_width", "few_rows_two_calls"])
def test_gateup_save_equals_gateup_and_preact(counts, d, f):
    """The training forward's gate|up GEMM: h bit-identical to moe_grouped_gemm_gateup and the kept
    pre-activations bit-identical to moe_grouped_gemm_gateup_preact (one kernel on the prefill path, the two
    calls below 128 rows per group)."""
    offs, _ = _ragged(counts, 0)
    M, G = int(offs[-1]), len(counts)
    a = to_dev_bf16(synth.normal_bf16(23, 0, 0, M * d, 1.0).reshape(M, d))
    w = to_dev_bf16(synth.normal_bf16(23, 2, 0, G * 2 * f * d, 0.05).reshape(G, 2 * f, d))
    o = torch.from_numpy(offs).cuda()
    h_ref = torch.empty(M, f, dtype=torch.bfloat16, device="cuda")
    gu_ref = torch.empty(M, 2 * f, dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup(a, w, o, h_ref)
    N.grouped_gemm_gateup_preact(a, w, o, gu_ref)
    h = torch.full((M, f), float("nan"), dtype=torch.bfloat16, device="cuda")
    gu = torch.full((M, 2 * f), float("nan"), dtype=torch.bfloat16, device="cuda")
    N.grouped_gemm_gateup_save(a, w, o, h, gu)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16))
    assert torch.equal(gu.view(torch.int16), gu_ref.view(torch.int16))


def _layer_and_grads(wl):
    inp = synth.device_inputs(wl)
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"],
                   inp["w_gateup_shared"], inp["w_down_shared"])
    layer(inp["x"])
    dy_bits = synth.dy_host(wl)
    out = layer.backward(to_dev_bf16(dy_bits))
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    return layer, out, dy_bits


TINY = [("tiny", {}), ("tiny", {"route": "softmax_topk_renorm"}),
        ("tiny", {"route": "sigmoid_topk_norm", "zipf_s": 1.2, "shared_f": 128})]


@pytest.mark.parametrize("name,over", TINY, ids=["topk_softmax", "softmax_topk_renorm", "sigmoid_bias_shared"])
def test_layer_backward_matches_oracle(name, over):
    wl = synth.workload(name, **over)
    layer, out, dy_bits = _layer_and_grads(wl)
    ref = oracle.LayerReference(wl)
    assert (layer.buf["topk_idx"].cpu().numpy() == ref.idx).all(), "routing differs from the oracle"
    gu = [synth.w_gateup_expert_host(wl, e) for e in range(wl.E)]
    dn = [synth.w_down_expert_host(wl, e) for e in range(wl.E)]
    sgu, sdn = synth.shared_host(wl)
    dy = _f64(dy_bits)
    exp = oracle.moe_backward(ref.x, gu, dn, ref.idx, ref.w, dy, sgu, sdn)
    rt = oracle.router_backward(ref.x, ref.w_router, ref.logits32, ref.idx, ref.w, exp["dw"], wl.route)
    check_close(bf16_to_host_f32(out["dx"]), exp["dx"] + rt["dx"], "dx")
    check_close(out["dtopk_w"].cpu().numpy(), exp["dw"], "routing-weight gradient")
    check_close(out["dw_gateup"].cpu().numpy(), exp["dw_gateup"], "dW_gateup")
    check_close(out["dw_down"].cpu().numpy(), exp["dw_down"], "dW_down")
    check_close(out["dw_router"].cpu().numpy(), rt["dw_router"], "dW_router")
    if wl.zipf_s > 0:
        check_close(out["dbias"].cpu().numpy(), rt["dbias"], "dbias")
    if wl.shared_f:
        check_close(out["dw_gateup_shared"].cpu().numpy()[0], exp["dw_gateup_shared"], "dW_gateup shared")
        check_close(out["dw_down_shared"].cpu().numpy()[0], exp["dw_down_shared"], "dW_down shared")
    # deterministic: a second backward gives the same bits
    dx1 = out["dx"].clone()
    dwg1 = out["dw_gateup"].clone()
    out2 = layer.backward(to_dev_bf16(dy_bits))
    assert torch.equal(out2["dx"].view(torch.int16), dx1.view(torch.int16))
    assert torch.equal(out2["dw_gateup"], dwg1)


def test_layer_backward_gpt_oss_sampled():
    """gpt-oss-shaped prefill: dx and the routing-weight gradient of sampled tokens (experts + router), and
    sampled entries of two experts' weight gradients, each summed over every token routed to the expert."""
    wl = synth.workload("gpt-oss-20b-prefill")
    layer, out, dy_bits = _layer_and_grads(wl)
    ref = oracle.LayerReference(wl)
    rng = np.random.default_rng(5)
    ties = set(ref.near_ties(1e-5).tolist())
    toks = np.array(sorted(t for t in rng.choice(wl.T, size=40, replace=False) if t not in ties), dtype=np.int32)
    gi = layer.buf["topk_idx"].cpu().numpy()
    mismatch = np.nonzero((gi != ref.idx).any(axis=1))[0]
    assert set(mismatch.tolist()) <= ties, "routing differs outside near-ties"
    check_close(bf16_to_host_f32(out["dx"])[toks], ref.input_grad(dy_bits, toks), "dx (sampled tokens)")
    sgu, sdn = ref._load_weights(toks)
    exp = oracle.moe_backward(ref.x[toks], ref._gu, ref._dn, ref.idx[toks], ref.w[toks], _f64(dy_bits)[toks], sgu,
                              sdn, weight_grads=False)
    check_close(out["dtopk_w"].cpu().numpy()[toks], exp["dw"], "routing-weight gradient (sampled tokens)")
    if mismatch.size:  # weight gradients sum over all tokens: only meaningful when routing agrees everywhere
        pytest.skip(f"{mismatch.size} near-tie tokens routed differently; weight-gradient entries not compared")
    dy = _f64(dy_bits)
    for e in (int(np.argmin(ref.counts)), int(np.argmax(ref.counts))):
        gu_e, dn_e = synth.w_gateup_expert_host(wl, e), synth.w_down_expert_host(wl, e)
        r_dn, c_dn = rng.integers(0, wl.d, 48), rng.integers(0, wl.f, 48)
        want = oracle.weight_grad_entries(ref.x, gu_e, dn_e, e, ref.idx, ref.w, dy, "down", r_dn, c_dn)
        check_close(out["dw_down"][e].cpu().numpy()[r_dn, c_dn], want, f"dW_down entries, expert {e}")
        r_gu, c_gu = rng.integers(0, 2 * wl.f, 48), rng.integers(0, wl.d, 48)
        want = oracle.weight_grad_entries(ref.x, gu_e, dn_e, e, ref.idx, ref.w, dy, "gateup", r_gu, c_gu)
        check_close(out["dw_gateup"][e].cpu().numpy()[r_gu, c_gu], want, f"dW_gateup entries, expert {e}")


@pytest.mark.parametrize("name,over", [("gpt-oss-20b-prefill", {"T": 1024}), TINY[2]],
                         ids=["gpt_oss_T1024", "tiny_sigmoid_bias_shared"])
def test_training_forward_keeps_preactivations(name, over):
    """forward(train=True) gives the same output, and the backward after it (no pre-activation recompute) the
    same gradients, bit for bit, as forward() + backward()."""
    wl = synth.workload(name, **over)
    inp = synth.device_inputs(wl)
    args = (inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"], inp["w_gateup_shared"],
            inp["w_down_shared"])
    a, b = MoEFFN(*args), MoEFFN(*args)
    dy = to_dev_bf16(synth.dy_host(wl))
    ya = a(inp["x"]).clone()
    ga = {k: v.clone() for k, v in a.backward(dy).items() if v is not None}
    yb = b.forward(inp["x"], train=True).clone()
    gb = b.backward(dy)
    torch.cuda.synchronize()
    assert N.get_device_error() == 0
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    for key, v in ga.items():
        w = gb[key]
        if v.dtype == torch.bfloat16:
            v, w = v.view(torch.int16), w.view(torch.int16)
        assert torch.equal(v, w), key

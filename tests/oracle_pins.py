"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes an oracle library handle (``oracle.load()``) so the mutation
test can run the same pins against deliberately broken copies of the oracle.
References used here are independent of the oracle's code: numpy/scipy/torch
fp64 library routines, brute-force enumeration, closed forms derived by hand
(tests/golden/), and algebraic invariants. None of them comes from the CUDA
path.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import scipy.special

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(a):
    """Round fp64/fp32 values to bf16 bits (RNE)."""
    return synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _random_bf16(rng, shape, scale):
    return _bf16(rng.standard_normal(shape) * scale)


def _dense_swiglu_torch(x_bits, gu_bits, dn_bits):
    import torch

    x = torch.from_numpy(_f64(x_bits))
    gu = torch.from_numpy(_f64(gu_bits))
    dn = torch.from_numpy(_f64(dn_bits))
    f = gu.shape[0] // 2
    g = x @ gu[:f].T
    u = x @ gu[f:].T
    return (torch.nn.functional.silu(g) * u @ dn.T).numpy()


# ---- routing ---------------------------------------------------------------------------------------

def pin_router_logits_numpy(lib):
    rng = _rng(1)
    T, d, E = 13, 40, 7
    x = _random_bf16(rng, (T, d), 1.0)
    wr = (rng.standard_normal((E, d)) * 0.02).astype(np.float32)
    bias = rng.standard_normal(E).astype(np.float32)
    got = oracle.router_logits(x, wr, bias, lib=lib)
    ref = _f64(x) @ wr.astype(np.float64).T + bias.astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    got0 = oracle.router_logits(x, wr, None, lib=lib)
    np.testing.assert_allclose(got0, _f64(x) @ wr.astype(np.float64).T, rtol=1e-12, atol=1e-14)


def pin_topk_golden(lib):
    g = json.load(open(os.path.join(GOLDEN, "topk_closed_form.json")))
    for c in g["cases"]:
        l = np.array([c["logits"]], dtype=np.float32)
        idx, w = oracle.topk(l, c["k"], c["mode"], lib=lib)
        assert idx[0].tolist() == c["idx"], (c["name"], idx[0].tolist())
        want = [eval(e, {"math": math}) for e in c["w_expr"]]
        np.testing.assert_allclose(w[0], want, rtol=2e-7, atol=1e-9, err_msg=c["name"])


def _brute_topk(l, k):
    return sorted(range(len(l)), key=lambda e: (-float(l[e]), e))[:k]


def pin_topk_bruteforce(lib):
    rng = _rng(2)
    T, E, k = 300, 9, 3
    # many exact ties: small integers plus a few distinct values
    l = rng.integers(-3, 4, size=(T, E)).astype(np.float32)
    l[::3] += rng.standard_normal((len(l[::3]), E)).astype(np.float32)
    for mode in ("topk_softmax", "softmax_topk_renorm", "sigmoid_topk_norm"):
        idx, w = oracle.topk(l, k, mode, lib=lib)
        for t in range(T):
            sel = _brute_topk(l[t], k)
            assert idx[t].tolist() == sel, (mode, t, idx[t], sel)
            ls = l[t].astype(np.float64)
            if mode == "topk_softmax":
                ref = scipy.special.softmax(ls[sel])
            elif mode == "softmax_topk_renorm":
                p = scipy.special.softmax(ls)
                ref = p[sel] / p[sel].sum()
            else:
                s = scipy.special.expit(ls[sel])
                ref = s / s.sum()
            np.testing.assert_allclose(w[t], ref, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def pin_topk_k_equals_E(lib):
    rng = _rng(3)
    l = (rng.standard_normal((50, 6)) * 2).astype(np.float32)
    idx, w = oracle.topk(l, 6, "topk_softmax", lib=lib)
    full = scipy.special.softmax(l.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, idx, axis=1), rtol=1e-12)
    idx2, w2 = oracle.topk(l, 6, "softmax_topk_renorm", lib=lib)
    assert (idx2 == idx).all()
    np.testing.assert_allclose(w2, w, rtol=1e-12)


def pin_renorm_equals_topk_softmax(lib):
    """Softmax over all experts then renormalising the top-k equals softmax over the top-k logits."""
    rng = _rng(4)
    l = (rng.standard_normal((200, 8)) * 3).astype(np.float32)
    i1, w1 = oracle.topk(l, 2, "topk_softmax", lib=lib)
    i2, w2 = oracle.topk(l, 2, "softmax_topk_renorm", lib=lib)
    assert (i1 == i2).all()
    np.testing.assert_allclose(w1, w2, rtol=1e-12)


def pin_margin(lib):
    rng = _rng(5)
    l = rng.standard_normal((100, 10))
    for k in (1, 3, 9, 10):
        m = oracle.topk_margin(l, k, lib=lib)
        s = -np.sort(-l, axis=1)
        ref = s[:, k - 1] - s[:, k] if k < 10 else np.full(100, np.inf)
        np.testing.assert_array_equal(m, ref)


# ---- grouping by expert ----------------------------------------------------------------------------

def pin_permute_argsort(lib):
    rng = _rng(6)
    for T, E, k in ((300, 11, 4), (1, 5, 5), (64, 128, 8), (0, 4, 2)):
        # leave some experts empty
        pool = rng.choice(E, size=max(k, E - 3), replace=False)
        idx = np.stack([rng.choice(pool, size=k, replace=False) for _ in range(T)]) if T else np.zeros((0, k))
        idx = idx.astype(np.int32)
        counts, offsets, perm_src, inv_perm = oracle.permute(idx, E, lib=lib)
        flat = idx.ravel()
        order = np.argsort(flat, kind="stable")
        np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        np.testing.assert_array_equal(perm_src, order // k)
        inv = np.empty_like(order)
        inv[order] = np.arange(len(order))
        np.testing.assert_array_equal(inv_perm, inv)


def pin_permute_invariants(lib):
    rng = _rng(7)
    T, E, k = 257, 16, 4
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm_src, inv_perm = oracle.permute(idx, E, lib=lib)
    R = T * k
    assert counts.sum() == R and offsets[-1] == R and offsets[0] == 0
    assert (np.diff(offsets) == counts).all()
    assert sorted(inv_perm.tolist()) == list(range(R))  # bijection
    a = np.arange(R)
    assert (perm_src[inv_perm] == a // k).all()
    # rows sorted by expert, and stable (flat assignment order) inside each expert
    row_expert = idx.ravel()[np.argsort(inv_perm)]
    assert (np.diff(row_expert) >= 0).all()
    for e in range(E):
        rows = np.arange(offsets[e], offsets[e + 1])
        assign = np.argsort(inv_perm)[rows]
        assert (np.diff(assign) > 0).all()


# ---- expert MLP + combine --------------------------------------------------------------------------

def _random_layer(rng, T, d, f, E, k, scale=0.3):
    x = _random_bf16(rng, (T, d), 1.0)
    gu = [_random_bf16(rng, (2 * f, d), scale) for _ in range(E)]
    dn = [_random_bf16(rng, (d, f), scale) for _ in range(E)]
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = scipy.special.softmax(rng.standard_normal((T, k)), axis=1)
    return x, gu, dn, idx, w


def pin_moe_dense_masked(lib):
    """Evaluate every expert for every token (fp64 numpy), weight by a dense mask that is zero off the
    selection, and sum: must equal the per-token loop over the selected experts."""
    rng = _rng(8)
    T, d, f, E, k = 7, 24, 10, 5, 2
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    X = _f64(x)
    dense_w = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            dense_w[t, idx[t, j]] += w[t, j]
    ref = np.zeros((T, d))
    for e in range(E):
        G = X @ _f64(gu[e][:f]).T
        U = X @ _f64(gu[e][f:]).T
        H = G * scipy.special.expit(G) * U
        ref += dense_w[:, e:e + 1] * (H @ _f64(dn[e]).T)
    got = oracle.moe_tokens(x, gu, dn, idx, w, np.arange(T), lib=lib)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    # a subset of tokens, in a shuffled order, gives the same rows
    sub = np.array([5, 0, 3])
    got_sub = oracle.moe_tokens(x, gu, dn, idx, w, sub, lib=lib)
    np.testing.assert_allclose(got_sub, ref[sub], rtol=1e-10, atol=1e-12)


def pin_moe_e1_k1_is_dense_swiglu(lib):
    """E = 1, k = 1: routing weight is 1 in every mode, so the layer is one dense SwiGLU FFN."""
    rng = _rng(9)
    T, d, f = 6, 32, 12
    x = _random_bf16(rng, (T, d), 1.0)
    gu = _random_bf16(rng, (2 * f, d), 0.2)
    dn = _random_bf16(rng, (d, f), 0.2)
    for mode in ("topk_softmax", "softmax_topk_renorm", "sigmoid_topk_norm"):
        logits = rng.standard_normal((T, 1)).astype(np.float32)
        idx, w = oracle.topk(logits, 1, mode, lib=lib)
        assert (idx == 0).all() and (w == 1.0).all()
        got = oracle.moe_tokens(x, [gu], [dn], idx, w, np.arange(T), lib=lib)
        np.testing.assert_allclose(got, _dense_swiglu_torch(x, gu, dn), rtol=1e-10, atol=1e-12)


def pin_identical_experts(lib):
    """All experts equal and weights summing to 1: output equals the dense SwiGLU whatever the routing."""
    rng = _rng(10)
    T, d, f, E, k = 9, 16, 8, 6, 3
    x = _random_bf16(rng, (T, d), 1.0)
    gu = _random_bf16(rng, (2 * f, d), 0.3)
    dn = _random_bf16(rng, (d, f), 0.3)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = scipy.special.softmax(rng.standard_normal((T, k)), axis=1)
    got = oracle.moe_tokens(x, [gu] * E, [dn] * E, idx, w, np.arange(T), lib=lib)
    np.testing.assert_allclose(got, _dense_swiglu_torch(x, gu, dn), rtol=1e-10, atol=1e-12)


def pin_down_linearity(lib):
    """Doubling every down weight (exact in bf16) doubles the output exactly."""
    rng = _rng(11)
    T, d, f, E, k = 5, 16, 12, 4, 2
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    dn2 = [_bf16(_f64(m) * 2) for m in dn]
    a = oracle.moe_tokens(x, gu, dn, idx, w, np.arange(T), lib=lib)
    b = oracle.moe_tokens(x, gu, dn2, idx, w, np.arange(T), lib=lib)
    np.testing.assert_array_equal(b, 2 * a)


def pin_swiglu_golden(lib):
    g = json.load(open(os.path.join(GOLDEN, "swiglu_closed_form.json")))
    x = _bf16(g["x"])
    gu = [_bf16(m) for m in g["w_gateup"]]
    dn = [_bf16(m) for m in g["w_down"]]
    idx = np.array(g["idx"], dtype=np.int32)
    w = np.array(g["w"], dtype=np.float64)
    got = oracle.moe_tokens(x, gu, dn, idx, w, [0], lib=lib)
    want = [eval(e, {"math": math}) for e in g["out_expr"]]
    np.testing.assert_allclose(got[0], want, rtol=1e-14, atol=1e-15)
    got0 = oracle.moe_tokens(x, gu, dn, idx[:, :1], np.ones((1, 1)), [0], lib=lib)
    np.testing.assert_allclose(got0[0], [eval(e, {"math": math}) for e in g["expert0_only_expr"]], rtol=1e-14)


def pin_shared_expert(lib):
    """The shared expert is added with weight 1: zero routed down weights leave exactly the shared
    expert's dense SwiGLU; with both, the output is the sum of the two parts."""
    rng = _rng(12)
    T, d, f, E, k, fs = 6, 16, 8, 5, 2, 12
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    sgu = _random_bf16(rng, (2 * fs, d), 0.3)
    sdn = _random_bf16(rng, (d, fs), 0.3)
    zero = [np.zeros_like(m) for m in dn]
    got = oracle.moe_tokens(x, gu, zero, idx, w, np.arange(T), sgu, sdn, lib=lib)
    np.testing.assert_allclose(got, _dense_swiglu_torch(x, sgu, sdn), rtol=1e-10, atol=1e-12)
    both = oracle.moe_tokens(x, gu, dn, idx, w, np.arange(T), sgu, sdn, lib=lib)
    routed = oracle.moe_tokens(x, gu, dn, idx, w, np.arange(T), lib=lib)
    np.testing.assert_allclose(both, routed + _dense_swiglu_torch(x, sgu, sdn), rtol=1e-10, atol=1e-12)


# ---- MXFP4 weights -----------------------------------------------------------------------------------

def _mx_golden():
    return json.load(open(os.path.join(GOLDEN, "mxfp4_e2m1.json")))


def _num(v):
    return -0.0 if v == "-0" else float(v)


def _pack_codes(codes):
    """Codes [..., N, K] (0..15) -> bytes [..., N, K/2] in the documented layout, written independently of the
    oracle: within each group of 8 elements, even elements fill the low 16 bits, odd ones the high 16 bits."""
    c = np.asarray(codes, dtype=np.uint32)
    *lead, K = c.shape
    c = c.reshape(*lead, K // 8, 4, 2)  # [..., word, i, parity]
    shifts = (np.arange(4, dtype=np.uint32) * 4)[:, None] + np.array([0, 16], dtype=np.uint32)[None, :]
    words = (c << shifts).sum(axis=(-1, -2)).astype("<u4")
    return words.view(np.uint8).reshape(*lead, K // 2)


def _unpack_codes(q):
    w = np.ascontiguousarray(q).view("<u4").astype(np.uint32)
    nib = (w[..., None] >> (np.arange(8, dtype=np.uint32) * 4)) & 15  # [..., word, nibble]
    order = np.array([0, 4, 1, 5, 2, 6, 3, 7])  # element e of the word sits in nibble order[e]
    return nib[..., order].reshape(*q.shape[:-1], q.shape[-1] * 2)


def pin_e2m1_table(lib):
    vals = [_num(v) for v in _mx_golden()["values"]]
    for code, want in enumerate(vals):
        got = oracle.e2m1_value(code, lib=lib)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)


def pin_mxfp4_rounding_golden(lib):
    g = _mx_golden()["rounding"]
    vals = [_num(v) for v in g["inputs"]] + [0.0] * (32 - len(g["inputs"]))
    w = _bf16(np.array(vals, dtype=np.float32))[None, :]
    q, s = oracle.mxfp4_quantize(w, lib=lib)
    assert s.shape == (1, 1) and int(s[0, 0]) == g["scale_code"]
    codes = _unpack_codes(q)[0]
    assert codes[: len(g["codes"])].tolist() == g["codes"], codes.tolist()
    assert (codes[len(g["codes"]):] == 0).all()


def pin_mxfp4_packing_golden(lib):
    g = _mx_golden()
    vals = [_num(g["values"][c]) for c in g["packing"]["codes"]] + [0.0] * 24
    q, s = oracle.mxfp4_quantize(_bf16(np.array(vals, dtype=np.float32))[None, :], lib=lib)
    assert q[0, :4].tolist() == g["packing"]["bytes"]
    assert int(s[0, 0]) == 127


def pin_mxfp4_round_trip(lib):
    """Blocks made of E2M1 values times a power of two, with at least one magnitude of 4 or 6 (which fixes the
    scale), decode to exact bf16 numbers and encode back to the same bytes; the decode agrees with an
    independent numpy decode of the documented layout and the specification's value table."""
    rng = _rng(20)
    G, N, K = 3, 5, 96  # N != K/32, so a transposed scale layout would show
    codes = rng.integers(0, 16, size=(G, N, K))
    codes[..., ::32] = rng.choice([6, 7, 14, 15], size=(G, N, K // 32))
    scales = rng.integers(0, 253, size=(G, K // 32, N)).astype(np.uint8)
    scales[0, 0, :] = [0, 1, 126, 127, 252]
    q = _pack_codes(codes)
    w = oracle.mxfp4_dequantize(q, scales, lib=lib)
    table = np.array([_num(v) for v in _mx_golden()["values"]])
    sc = np.repeat(np.transpose(scales, (0, 2, 1)).astype(np.float64), 32, axis=-1)  # [G, N, K]
    want = table[_unpack_codes(q)] * np.exp2(sc - 127)
    np.testing.assert_array_equal(_f64(w), want)
    q2, s2 = oracle.mxfp4_quantize(w, lib=lib)
    np.testing.assert_array_equal(s2, scales)
    np.testing.assert_array_equal(q2, q)


def pin_mxfp4_scale_closed_form(lib):
    """Shared scale = 2^(floor(log2 max|v|) - 2), clamped to the E8M0 range; an all-zero block gets code 0."""
    cases = [  # (max |v| of the block, expected scale code)
        (0.0, 0), (1.0, 125), (0.02, 119), (4.0, 127), (7.9, 127), (8.0, 128),
        (2.0 ** -130, 0), (2.0 ** -120, 5), (3.0e38, 252),
    ]
    rows = []
    for amax, _ in cases:
        r = np.zeros(32, dtype=np.float32)
        r[7] = -amax
        r[3] = amax / 3
        rows.append(r)
    w = _bf16(np.stack(rows))
    q, s = oracle.mxfp4_quantize(w, lib=lib)
    assert s[0].tolist() == [c for _, c in cases], s[0].tolist()
    # the element holding max |v| decodes to -4 or -6 times the scale whenever it is not clamped away
    amax_bf = np.abs(_f64(w[:, 7]))
    dq = _f64(oracle.mxfp4_dequantize(q, s, lib=lib))
    for i, (amax, code) in enumerate(cases):
        X = 2.0 ** (int(code) - 127)
        if amax == 0:
            assert (dq[i] == 0).all()
        elif amax_bf[i] / X >= 4:
            assert abs(dq[i, 7]) in (4 * X, 6 * X) and dq[i, 7] < 0


def pin_mxfp4_error_bound(lib):
    """Encode then decode of random weights: max|v| / scale lies in [4, 8); every element is within half the
    E2M1 grid spacing at its magnitude (0.25 below 2, 0.5 in [2, 4), 1 in [4, 6]) times the scale, and
    magnitudes above 6 times the scale decode to exactly 6 times the scale."""
    rng = _rng(21)
    w = _random_bf16(rng, (4, 64, 256), 0.02)
    q, s = oracle.mxfp4_quantize(w, lib=lib)
    dq = _f64(oracle.mxfp4_dequantize(q, s, lib=lib))
    v = _f64(w)
    X = np.repeat(np.exp2(np.transpose(s, (0, 2, 1)).astype(np.float64) - 127), 32, axis=-1)
    p = np.abs(v) / X
    blocks = p.reshape(4, 64, 8, 32).max(-1)
    assert ((blocks >= 4) & (blocks < 8)).all()
    half = np.where(p < 2, 0.25, np.where(p < 4, 0.5, 1.0))
    inside = p <= 6
    assert (np.abs(dq - v)[inside] <= half[inside] * X[inside]).all()
    assert (np.abs(dq)[~inside] == 6 * X[~inside]).all()
    assert (np.signbit(dq) == np.signbit(v)).all()


# ---- backward (training) ---------------------------------------------------------------------------------

def _torch_expert_grads(x_bits, gu, dn, idx, w, dy, sgu=None, sdn=None):
    """Gradients of sum(dy * out) through the per-token layer, by torch fp64 autograd (an independent
    derivation of what the oracle's hand-written backward computes)."""
    import torch

    X = torch.tensor(_f64(x_bits), requires_grad=True)
    GU = [torch.tensor(_f64(m), requires_grad=True) for m in gu]
    DN = [torch.tensor(_f64(m), requires_grad=True) for m in dn]
    W = torch.tensor(np.asarray(w, np.float64), requires_grad=True)
    SG = torch.tensor(_f64(sgu), requires_grad=True) if sgu is not None else None
    SD = torch.tensor(_f64(sdn), requires_grad=True) if sdn is not None else None
    T, k = idx.shape
    f = gu[0].shape[0] // 2

    def mlp(gum, dnm, xt, ff):
        return dnm @ (torch.nn.functional.silu(gum[:ff] @ xt) * (gum[ff:] @ xt))

    rows = []
    for t in range(T):
        acc = sum(W[t, j] * mlp(GU[idx[t, j]], DN[idx[t, j]], X[t], f) for j in range(k))
        if SG is not None:
            acc = acc + mlp(SG, SD, X[t], SG.shape[0] // 2)
        rows.append(acc)
    (torch.stack(rows) * torch.tensor(np.asarray(dy, np.float64))).sum().backward()
    z = lambda P, ref: np.zeros(ref.shape) if P.grad is None else P.grad.numpy()
    out = {"dx": X.grad.numpy(), "dw_gateup": np.stack([z(P, m) for P, m in zip(GU, gu)]),
           "dw_down": np.stack([z(P, m) for P, m in zip(DN, dn)]), "dw": W.grad.numpy()}
    if SG is not None:
        out["dw_gateup_shared"], out["dw_down_shared"] = SG.grad.numpy(), SD.grad.numpy()
    return out


def pin_backward_autograd(lib):
    rng = _rng(40)
    T, d, f, E, k, fs = 6, 12, 8, 5, 2, 6
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    sgu = _random_bf16(rng, (2 * fs, d), 0.3)
    sdn = _random_bf16(rng, (d, fs), 0.3)
    dy = rng.standard_normal((T, d))
    got = oracle.moe_backward(x, gu, dn, idx, w, dy, sgu, sdn, lib=lib)
    want = _torch_expert_grads(x, gu, dn, idx, w, dy, sgu, sdn)
    for key in want:
        np.testing.assert_allclose(got[key], want[key], rtol=1e-10, atol=1e-12, err_msg=key)


def pin_backward_routing_weights_finite_difference(lib):
    """The layer is linear in each routing weight, so a central difference of the forward oracle gives
    d sum(dy * out) / d w[t, j] up to rounding."""
    rng = _rng(41)
    T, d, f, E, k = 5, 10, 6, 4, 3
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    dy = rng.standard_normal((T, d))
    got = oracle.moe_backward(x, gu, dn, idx, w, dy, lib=lib)["dw"]
    h = 1e-3
    for t in range(T):
        for j in range(k):
            wp, wm = w.copy(), w.copy()
            wp[t, j] += h
            wm[t, j] -= h
            fp = oracle.moe_tokens(x, gu, dn, idx, wp, np.arange(T), lib=lib)
            fm = oracle.moe_tokens(x, gu, dn, idx, wm, np.arange(T), lib=lib)
            num = ((fp - fm) * dy).sum() / (2 * h)
            assert abs(num - got[t, j]) <= 1e-9 * max(1.0, abs(num)), (t, j, num, got[t, j])


def pin_backward_linear_in_dy(lib):
    rng = _rng(42)
    x, gu, dn, idx, w = _random_layer(rng, 4, 8, 8, 3, 2)
    a, b = rng.standard_normal((4, 8)), rng.standard_normal((4, 8))
    ga = oracle.moe_backward(x, gu, dn, idx, w, a, lib=lib)
    gb = oracle.moe_backward(x, gu, dn, idx, w, b, lib=lib)
    gab = oracle.moe_backward(x, gu, dn, idx, w, a + 2 * b, lib=lib)
    for key in ga:
        np.testing.assert_allclose(gab[key], ga[key] + 2 * gb[key], rtol=1e-10, atol=1e-12, err_msg=key)


def _router_case(rng, T, E, k):
    """fp32 logits whose k-th and (k+1)-th values are well apart (the selection survives small steps)."""
    l = np.empty((T, E), dtype=np.float32)
    for t in range(T):
        v = rng.permutation(E).astype(np.float64) * 0.37 + rng.uniform(-0.05, 0.05, E)
        l[t] = (v - v.mean()).astype(np.float32)
    return l


def pin_router_backward_autograd(lib):
    import torch

    rng = _rng(43)
    T, d, E, k = 7, 16, 9, 3
    x = _random_bf16(rng, (T, d), 1.0)
    wr = (rng.standard_normal((E, d)) * 0.3).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.2).astype(np.float32)
    for mode in ("topk_softmax", "softmax_topk_renorm", "sigmoid_topk_norm"):
        X = torch.tensor(_f64(x), requires_grad=True)
        WR = torch.tensor(wr.astype(np.float64), requires_grad=True)
        B = torch.tensor(bias.astype(np.float64), requires_grad=True)
        L = X @ WR.T + B
        l32 = L.detach().numpy().astype(np.float32)
        idx, w = oracle.topk(l32, k, mode, lib=lib)
        dw = rng.standard_normal((T, k))
        sel = L.gather(1, torch.tensor(idx, dtype=torch.int64))
        if mode == "topk_softmax":
            ww = torch.softmax(sel, dim=1)
        elif mode == "softmax_topk_renorm":
            p = torch.softmax(L, dim=1).gather(1, torch.tensor(idx, dtype=torch.int64))
            ww = p / p.sum(1, keepdim=True)
        else:
            s = torch.sigmoid(sel)
            ww = s / s.sum(1, keepdim=True)
        L.retain_grad()
        (ww * torch.tensor(dw)).sum().backward()
        got = oracle.router_backward(x, wr, l32, idx, w, dw, mode, lib=lib)
        # the oracle works from the fp32-rounded logits; autograd from the fp64 ones
        np.testing.assert_allclose(got["dlogits"], L.grad.numpy(), rtol=1e-5, atol=1e-7, err_msg=mode)
        np.testing.assert_allclose(got["dw_router"], WR.grad.numpy(), rtol=1e-5, atol=1e-6, err_msg=mode)
        np.testing.assert_allclose(got["dbias"], B.grad.numpy(), rtol=1e-5, atol=1e-7, err_msg=mode)
        np.testing.assert_allclose(got["dx"], X.grad.numpy(), rtol=1e-5, atol=1e-7, err_msg=mode)


def pin_router_backward_finite_difference(lib):
    """Central differences of topk's routing weights in each logit (selection unchanged by the step)."""
    rng = _rng(44)
    T, E, k = 5, 8, 3
    l = _router_case(rng, T, E, k)
    x = _random_bf16(rng, (T, 4), 1.0)
    wr = np.zeros((E, 4), dtype=np.float32)
    for mode in ("topk_softmax", "softmax_topk_renorm", "sigmoid_topk_norm"):
        idx, w = oracle.topk(l, k, mode, lib=lib)
        dw = rng.standard_normal((T, k))
        got = oracle.router_backward(x, wr, l, idx, w, dw, mode, lib=lib)["dlogits"]
        for t in range(T):
            for e in range(E):
                lp, lm = l.copy(), l.copy()
                lp[t, e] += np.float32(1e-2)
                lm[t, e] -= np.float32(1e-2)
                ip, wp = oracle.topk(lp, k, mode, lib=lib)
                im, wm = oracle.topk(lm, k, mode, lib=lib)
                assert (ip == idx).all() and (im == idx).all()
                step = float(lp[t, e]) - float(lm[t, e])
                num = ((wp - wm) * dw).sum() / step
                assert abs(num - got[t, e]) <= 2e-4 * max(1.0, abs(num)), (mode, t, e, num, got[t, e])


def pin_weight_grad_entries(lib):
    """Sampled weight-gradient entries equal the corresponding entries of the full backward (which autograd pins)."""
    rng = _rng(45)
    T, d, f, E, k = 9, 16, 12, 4, 2
    x, gu, dn, idx, w = _random_layer(rng, T, d, f, E, k)
    dy = rng.standard_normal((T, d))
    full = oracle.moe_backward(x, gu, dn, idx, w, dy, lib=lib)
    for e in range(E):
        rows, cols = rng.integers(0, d, 20), rng.integers(0, f, 20)
        got = oracle.weight_grad_entries(x, gu[e], dn[e], e, idx, w, dy, "down", rows, cols, lib=lib)
        np.testing.assert_allclose(got, full["dw_down"][e][rows, cols], rtol=1e-12, atol=1e-14)
        rows, cols = rng.integers(0, 2 * f, 20), rng.integers(0, d, 20)
        got = oracle.weight_grad_entries(x, gu[e], dn[e], e, idx, w, dy, "gateup", rows, cols, lib=lib)
        np.testing.assert_allclose(got, full["dw_gateup"][e][rows, cols], rtol=1e-12, atol=1e-14)


def pin_layer_input_grad_autograd(lib):
    """The whole layer's input gradient (experts + router, selection held fixed) on the tiny workload equals torch
    fp64 autograd through the router projection, the routing-weight formula and the experts."""
    import torch

    wl = synth.workload("tiny")
    ref = oracle.LayerReference(wl, lib=lib)
    dy_bits = synth.dy_host(wl)
    toks = np.arange(wl.T)
    got = ref.input_grad(dy_bits, toks)
    X = torch.tensor(_f64(ref.x), requires_grad=True)
    L = X @ torch.tensor(ref.w_router.astype(np.float64)).T
    sel = torch.tensor(ref.idx, dtype=torch.int64)
    w = torch.softmax(L.gather(1, sel), dim=1)  # the tiny workload routes by softmax over the selected logits
    assert wl.route == "topk_softmax"
    gus = {e: torch.tensor(_f64(synth.w_gateup_expert_host(wl, e))) for e in np.unique(ref.idx)}
    dns = {e: torch.tensor(_f64(synth.w_down_expert_host(wl, e))) for e in np.unique(ref.idx)}
    f = wl.f
    rows = []
    for t in range(wl.T):
        acc = 0
        for j in range(wl.k):
            e = int(ref.idx[t, j])
            hh = torch.nn.functional.silu(gus[e][:f] @ X[t]) * (gus[e][f:] @ X[t])
            acc = acc + w[t, j] * (dns[e] @ hh)
        rows.append(acc)
    (torch.stack(rows) * torch.tensor(_f64(dy_bits))).sum().backward()
    want = X.grad.numpy()
    # the oracle takes its routing weights from the fp32-rounded logits; autograd from the fp64 ones
    np.testing.assert_allclose(got, want, rtol=1e-4, atol=1e-5 * np.abs(want).max())


PINS = [
    pin_router_logits_numpy,
    pin_topk_golden,
    pin_topk_bruteforce,
    pin_topk_k_equals_E,
    pin_renorm_equals_topk_softmax,
    pin_margin,
    pin_permute_argsort,
    pin_permute_invariants,
    pin_moe_dense_masked,
    pin_moe_e1_k1_is_dense_swiglu,
    pin_identical_experts,
    pin_down_linearity,
    pin_swiglu_golden,
    pin_shared_expert,
    pin_e2m1_table,
    pin_mxfp4_rounding_golden,
    pin_mxfp4_packing_golden,
    pin_mxfp4_round_trip,
    pin_mxfp4_scale_closed_form,
    pin_mxfp4_error_bound,
    pin_backward_autograd,
    pin_backward_routing_weights_finite_difference,
    pin_backward_linear_in_dy,
    pin_router_backward_autograd,
    pin_router_backward_finite_difference,
    pin_layer_input_grad_autograd,
    pin_weight_grad_entries,
]

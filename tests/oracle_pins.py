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
]

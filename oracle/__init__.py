"""CPU oracle for the sparse MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY: the plain, slow, obviously correct CPU definition
that the CUDA path is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it. It shares no code with the CUDA path (``mixture_experts_ffn_11_b200``)
and does not import it; both take their inputs from the ``synth`` module.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 accumulation); this
module builds it, marshals numpy arrays, and strings the steps together.
Citations are to the blog post "Mixture of Experts (MoEs) in Transformers".

Parity status per function (what pins it, see tests/test_oracle_pins.py):
  router_logits  pinned: numpy fp64 matmul; closed-form golden cases
  topk           pinned: brute-force full sort; golden ties; closed-form weights
  permute        pinned: numpy stable argsort; invariants (bijection, scan)
  moe_tokens     pinned: dense-masked brute force over all experts (numpy fp64);
                 E=1,k=1 dense SwiGLU (torch fp64); identical experts; linearity
                 in W_down; hand-derived golden values
  e2m1_value     pinned: the FP4 E2M1 value table of the OCP MX v1.0 specification
                 (tests/golden/mxfp4_e2m1.json, codes 0..15 including -0)
  mxfp4_quantize pinned: round-trip of encodable blocks; the tie and clamp cases of
                 round-to-nearest-even on the E2M1 grid; closed-form scales (zero,
                 subnormal and power-of-two blocks); the error bound of the grid;
                 a hand-packed word of the documented nibble layout
  mxfp4_dequantize pinned: inverse of the above on every code and scale range;
                 numpy decode of the documented layout
  moe_backward   pinned: torch fp64 autograd of the same per-token loop (dx, every
                 weight gradient, routing-weight gradients, shared expert); central
                 differences of moe_tokens in the routing weights; linearity in dy
  router_backward pinned: torch fp64 autograd of each mode's weight formula and of the
                 router projection; central differences of topk's weights in the logits
  weight_grad_entries pinned: equal to the matching entries of moe_backward's full
                 weight gradients on random small layers
  LayerReference.input_grad pinned: torch fp64 autograd of the whole layer per token
                 (router projection, routing weights and experts) on the tiny workload
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "_moe_oracle.so")

ROUTE_MODES = {"topk_softmax": 0, "softmax_topk_renorm": 1, "sigmoid_topk_norm": 2}


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", src, "-o", out, "-lm"])
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` selects another build of it."""
    lib = ctypes.CDLL(path or build())
    vp, ci = ctypes.c_void_p, ctypes.c_int
    lib.oracle_router_logits.argtypes = [vp, vp, vp, ci, ci, ci, vp]
    lib.oracle_router_logits.restype = None
    lib.oracle_topk.argtypes = [vp, ci, ci, ci, ci, vp, vp]
    lib.oracle_topk.restype = ci
    lib.oracle_topk_margin.argtypes = [vp, ci, ci, ci, vp]
    lib.oracle_topk_margin.restype = ci
    lib.oracle_permute.argtypes = [vp, ci, ci, ci, vp, vp, vp, vp]
    lib.oracle_permute.restype = ci
    lib.oracle_moe_tokens.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, ci, vp, ci, vp, ci]
    lib.oracle_moe_tokens.restype = ci
    lib.oracle_e2m1_value.argtypes = [ci]
    lib.oracle_e2m1_value.restype = ctypes.c_double
    lib.oracle_mxfp4_quantize.argtypes = [vp, ci, ci, ci, vp, vp, ci]
    lib.oracle_mxfp4_quantize.restype = ci
    lib.oracle_mxfp4_dequantize.argtypes = [vp, vp, ci, ci, ci, vp, ci]
    lib.oracle_mxfp4_dequantize.restype = ci
    lib.oracle_moe_backward.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp, vp, vp]
    lib.oracle_moe_backward.restype = ci
    lib.oracle_router_backward.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_router_backward.restype = ci
    lib.oracle_weight_grad_entries.argtypes = [vp, ci, ci, ci, ci, vp, vp, ci, vp, vp, vp, ci, vp, vp, ci, vp]
    lib.oracle_weight_grad_entries.restype = ci
    return lib


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def _threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def router_logits(x_bits: np.ndarray, w_router: np.ndarray, bias: np.ndarray | None = None, lib=None) -> np.ndarray:
    """fp64 logits x . W_r^T (+bias): the router scores every expert from the token's hidden state
    (section "From Dense to Sparse"). x_bits: [T,d] bf16 bits; w_router: [E,d] fp32."""
    lib = lib or _L()
    x = _c(x_bits, np.uint16)
    wr = _c(w_router, np.float32)
    T, d = x.shape
    E = wr.shape[0]
    b = _c(bias, np.float32) if bias is not None else None
    out = np.empty((T, E), dtype=np.float64)
    lib.oracle_router_logits(x.ctypes.data, wr.ctypes.data, b.ctypes.data if b is not None else None, T, d, E,
                             out.ctypes.data)
    return out


def topk(logits_f32: np.ndarray, k: int, mode: str, lib=None):
    """Top-k experts per token on fp32 logits (descending, lower id first on ties) and their weights (fp64)."""
    lib = lib or _L()
    l = _c(logits_f32, np.float32)
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    rc = lib.oracle_topk(l.ctypes.data, T, E, k, ROUTE_MODES[mode], idx.ctypes.data, w.ctypes.data)
    if rc:
        raise ValueError("oracle_topk: bad arguments")
    return idx, w


def topk_margin(logits64: np.ndarray, k: int, lib=None) -> np.ndarray:
    lib = lib or _L()
    l = _c(logits64, np.float64)
    T, E = l.shape
    m = np.empty(T, dtype=np.float64)
    if lib.oracle_topk_margin(l.ctypes.data, T, E, k, m.ctypes.data):
        raise ValueError("oracle_topk_margin: bad arguments")
    return m


def permute(idx: np.ndarray, E: int, lib=None):
    """Stable grouping of the T*k assignments by expert id ("sort tokens by expert ID, group them",
    section "Expert Backend"). Returns counts[E], offsets[E+1], perm_src[R], inv_perm[R]."""
    lib = lib or _L()
    ix = _c(idx, np.int32)
    T, k = ix.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm_src = np.empty(T * k, dtype=np.int32)
    inv_perm = np.empty(T * k, dtype=np.int32)
    if lib.oracle_permute(ix.ctypes.data, T, E, k, counts.ctypes.data, offsets.ctypes.data, perm_src.ctypes.data,
                          inv_perm.ctypes.data):
        raise ValueError("oracle_permute: expert index out of range")
    return counts, offsets, perm_src, inv_perm


def moe_tokens(x_bits, expert_gateup, expert_down, idx, w, tokens, shared_gateup=None, shared_down=None,
               nthreads: int | None = None, lib=None) -> np.ndarray:
    """Per-token loop over the selected experts (the eager backend of section "Expert Backend"):
    out[q] = sum_j w[t,j] * down_e(silu(gate_e x_t) * up_e x_t) (+ shared expert), fp64.

    expert_gateup / expert_down: sequences of length E holding [2f,d] / [d,f] bf16-bit arrays, or None
    for experts that no listed token selects.
    """
    lib = lib or _L()
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    E = len(expert_gateup)
    ix = _c(idx, np.int32)
    k = ix.shape[1]
    ww = _c(w, np.float64)
    toks = _c(tokens, np.int32)
    f = None
    keep = []
    gu_ptrs = (ctypes.c_void_p * E)()
    dn_ptrs = (ctypes.c_void_p * E)()
    for e in range(E):
        gu, dn = expert_gateup[e], expert_down[e]
        if gu is None or dn is None:
            continue
        gu = _c(gu, np.uint16)
        dn = _c(dn, np.uint16)
        f = gu.shape[0] // 2
        keep += [gu, dn]
        gu_ptrs[e] = gu.ctypes.data
        dn_ptrs[e] = dn.ctypes.data
    if f is None:
        raise ValueError("no expert weights given")
    sgu = _c(shared_gateup, np.uint16) if shared_gateup is not None else None
    sdn = _c(shared_down, np.uint16) if shared_down is not None else None
    fs = sgu.shape[0] // 2 if sgu is not None else 0
    out = np.empty((len(toks), d), dtype=np.float64)
    n = nthreads or max(1, len(os.sched_getaffinity(0)))
    rc = lib.oracle_moe_tokens(x.ctypes.data, T, d, f, E, k, gu_ptrs, dn_ptrs, ix.ctypes.data, ww.ctypes.data,
                               sgu.ctypes.data if sgu is not None else None,
                               sdn.ctypes.data if sdn is not None else None, fs, toks.ctypes.data, len(toks),
                               out.ctypes.data, n)
    if rc:
        raise ValueError(f"oracle_moe_tokens failed ({rc})")
    return out


def e2m1_value(code: int, lib=None) -> float:
    """Value of one FP4 E2M1 code (OCP Microscaling Formats v1.0 element format)."""
    return (lib or _L()).oracle_e2m1_value(int(code))


def mxfp4_quantize(w_bits: np.ndarray, lib=None):
    """MXFP4 encoding of bf16 weights [G, N, K] (or [N, K]) along K: blocks of 32 share one E8M0 scale, each
    element is an E2M1 code (the "native mxfp4 quantization" of gpt-oss, blog post section "From Dense to
    Sparse: What Are MoEs?"). Returns codes [G, N, K/2] uint8 and scales [G, K/32, N] uint8 (layout in
    moe_oracle.c)."""
    lib = lib or _L()
    w = _c(w_bits, np.uint16)
    squeeze = w.ndim == 2
    if squeeze:
        w = w[None]
    G, N, K = w.shape
    q = np.empty((G, N, K // 2), dtype=np.uint8)
    s = np.empty((G, K // 32, N), dtype=np.uint8)
    if lib.oracle_mxfp4_quantize(w.ctypes.data, G, N, K, q.ctypes.data, s.ctypes.data, _threads()):
        raise ValueError(f"oracle_mxfp4_quantize: K={K} is not a multiple of 32")
    return (q[0], s[0]) if squeeze else (q, s)


def mxfp4_dequantize(q: np.ndarray, s: np.ndarray, lib=None) -> np.ndarray:
    """The bf16 weights (bits) that MXFP4 codes [G, N, K/2] and scales [G, K/32, N] encode (exactly)."""
    lib = lib or _L()
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    squeeze = q.ndim == 2
    if squeeze:
        q, s = q[None], s[None]
    G, N, K2 = q.shape
    K = 2 * K2
    if s.shape != (G, K // 32, N):
        raise ValueError(f"scales {s.shape} do not match codes {q.shape}")
    w = np.empty((G, N, K), dtype=np.uint16)
    rc = lib.oracle_mxfp4_dequantize(q.ctypes.data, s.ctypes.data, G, N, K, w.ctypes.data, _threads())
    if rc:
        raise ValueError(f"oracle_mxfp4_dequantize failed ({rc}): a value is not a finite bf16 number")
    return w[0] if squeeze else w


def mxfp4_round_trip(w_bits: np.ndarray, lib=None) -> np.ndarray:
    """The weights an MXFP4 layer computes with: bf16 weights encoded, then decoded."""
    q, s = mxfp4_quantize(w_bits, lib=lib)
    return mxfp4_dequantize(q, s, lib=lib)


def moe_backward(x_bits, expert_gateup, expert_down, idx, w, dy, shared_gateup=None, shared_down=None, lib=None,
                 weight_grads: bool = True):
    """Gradients of the expert part of the layer (section "Training MoEs with Transformers" trains through the
    same expert backend): given dy = d loss / d out for every token, returns a dict with dx [T, d], dw [T, k]
    (routing weights) and, with weight_grads, dw_gateup [E, 2f, d], dw_down [E, d, f] and the shared expert's two
    weight gradients. Weights as for moe_tokens (bf16 bits, every expert that a token selects must be given). fp64."""
    lib = lib or _L()
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    E = len(expert_gateup)
    ix = _c(idx, np.int32)
    k = ix.shape[1]
    ww = _c(w, np.float64)
    g = _c(dy, np.float64)
    f = next(a.shape[0] // 2 for a in expert_gateup if a is not None)
    keep = []
    gu_p, dn_p = (ctypes.c_void_p * E)(), (ctypes.c_void_p * E)()
    dgu_p, ddn_p = (ctypes.c_void_p * E)(), (ctypes.c_void_p * E)()
    dgu = np.zeros((E, 2 * f, d)) if weight_grads else None
    ddn = np.zeros((E, d, f)) if weight_grads else None
    for e in range(E):
        if expert_gateup[e] is None or expert_down[e] is None:
            continue
        gu, dn = _c(expert_gateup[e], np.uint16), _c(expert_down[e], np.uint16)
        keep += [gu, dn]
        gu_p[e], dn_p[e] = gu.ctypes.data, dn.ctypes.data
        if weight_grads:
            dgu_p[e], ddn_p[e] = dgu[e].ctypes.data, ddn[e].ctypes.data
    sgu = _c(shared_gateup, np.uint16) if shared_gateup is not None else None
    sdn = _c(shared_down, np.uint16) if shared_down is not None else None
    fs = sgu.shape[0] // 2 if sgu is not None else 0
    dsgu = np.zeros((2 * fs, d)) if fs and weight_grads else None
    dsdn = np.zeros((d, fs)) if fs and weight_grads else None
    dx = np.empty((T, d))
    dw = np.empty((T, k))
    rc = lib.oracle_moe_backward(x.ctypes.data, T, d, f, E, k, gu_p, dn_p, ix.ctypes.data, ww.ctypes.data, g.ctypes.data,
                                 sgu.ctypes.data if fs else None, sdn.ctypes.data if fs else None, fs,
                                 dx.ctypes.data, dgu_p if weight_grads else None, ddn_p if weight_grads else None,
                                 dw.ctypes.data, dsgu.ctypes.data if dsgu is not None else None,
                                 dsdn.ctypes.data if dsdn is not None else None)
    if rc:
        raise ValueError(f"oracle_moe_backward failed ({rc})")
    out = {"dx": dx, "dw": dw}
    if weight_grads:
        out["dw_gateup"], out["dw_down"] = dgu, ddn
        if fs:
            out["dw_gateup_shared"], out["dw_down_shared"] = dsgu, dsdn
    return out


def weight_grad_entries(x_bits, w_gateup_e, w_down_e, e: int, idx, w, dy, which: str, rows, cols, lib=None):
    """Entries (rows[q], cols[q]) of expert e's weight gradient, summed over every token that selects e:
    which = "down" -> dW_down[e] [d, f]; which = "gateup" -> dW_gateup[e] [2f, d]. fp64. The same sums as
    moe_backward, for a sample of entries (full-size layers)."""
    lib = lib or _L()
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    gu, dn = _c(w_gateup_e, np.uint16), _c(w_down_e, np.uint16)
    f = gu.shape[0] // 2
    ix = _c(idx, np.int32)
    a, b = _c(rows, np.int32), _c(cols, np.int32)
    out = np.empty(len(a))
    rc = lib.oracle_weight_grad_entries(x.ctypes.data, T, d, f, ix.shape[1], gu.ctypes.data, dn.ctypes.data, int(e),
                                        ix.ctypes.data, _c(w, np.float64).ctypes.data, _c(dy, np.float64).ctypes.data,
                                        0 if which == "down" else 1, a.ctypes.data, b.ctypes.data, len(a),
                                        out.ctypes.data)
    if rc:
        raise ValueError(f"oracle_weight_grad_entries failed ({rc})")
    return out


def router_backward(x_bits, w_router, logits_f32, idx, w, dw, mode: str, lib=None):
    """Router gradients with the top-k selection held fixed: from dw = d loss / d w (routing weights computed by
    topk from these fp32 logits), returns dlogits [T, E], dw_router [E, d], dbias [E] and the router's share of
    dx [T, d]. fp64."""
    lib = lib or _L()
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    wr = _c(w_router, np.float32)
    E = wr.shape[0]
    l = _c(logits_f32, np.float32)
    ix = _c(idx, np.int32)
    k = ix.shape[1]
    dl = np.empty((T, E))
    dwr = np.empty((E, d))
    db = np.empty(E)
    dx = np.empty((T, d))
    rc = lib.oracle_router_backward(x.ctypes.data, wr.ctypes.data, l.ctypes.data, T, d, E, k, ROUTE_MODES[mode],
                                    ix.ctypes.data, _c(w, np.float64).ctypes.data, _c(dw, np.float64).ctypes.data,
                                    dl.ctypes.data, dwr.ctypes.data, db.ctypes.data, dx.ctypes.data)
    if rc:
        raise ValueError(f"oracle_router_backward failed ({rc})")
    return {"dlogits": dl, "dw_router": dwr, "dbias": db, "dx": dx}


class LayerReference:
    """The whole layer for one synthetic workload, computed by the oracle.

    Routing and grouping are computed for all tokens; expert outputs only for the tokens asked for,
    generating only the experts those tokens select (so multi-gigabyte layers stay cheap on the host).
    """

    def __init__(self, wl, lib=None):
        import synth

        self.wl = wl
        self.lib = lib or _L()
        self.x = synth.x_host(wl)
        self.w_router = synth.w_router_host(wl)
        self.bias = synth.zipf_bias(wl)
        self.logits64 = router_logits(self.x, self.w_router, self.bias, lib=self.lib)
        self.logits32 = self.logits64.astype(np.float32)
        self.idx, self.w = topk(self.logits32, wl.k, wl.route, lib=self.lib)
        self.margin = topk_margin(self.logits64, wl.k, lib=self.lib)
        self.counts, self.offsets, self.perm_src, self.inv_perm = permute(self.idx, wl.E, lib=self.lib)
        self._gu = [None] * wl.E
        self._dn = [None] * wl.E
        self._shared = None

    def input_grad(self, dy_bits, tokens, nthreads: int | None = None) -> np.ndarray:
        """d loss / d x for the given tokens (rows of dy = d loss / d y as bf16 bits [T, d]): the experts' share
        (moe_backward) plus the router's (router_backward), the top-k selection held fixed. A token's input
        gradient depends only on that token, so a sample of tokens is computed alone. fp64."""
        import synth

        wl = self.wl
        tokens = np.asarray(tokens, dtype=np.int32)
        sgu, sdn = self._load_weights(tokens)
        dy = synth.bf16_bits_to_f32(np.asarray(dy_bits)[tokens]).astype(np.float64)
        xs = self.x[tokens]
        exp = moe_backward(xs, self._gu, self._dn, self.idx[tokens], self.w[tokens], dy, sgu, sdn, lib=self.lib,
                           weight_grads=False)
        rt = router_backward(xs, self.w_router, self.logits32[tokens], self.idx[tokens], self.w[tokens], exp["dw"],
                             wl.route, lib=self.lib)
        return exp["dx"] + rt["dx"]

    def near_ties(self, eps: float = 1e-5) -> np.ndarray:
        return np.nonzero(self.margin < eps)[0]

    def _load_weights(self, tokens):
        """Generate (once) the weights of the experts these tokens select, and the shared expert's."""
        import synth

        wl = self.wl
        need = np.unique(self.idx[tokens].ravel()) if len(tokens) else np.zeros(0, np.int32)
        # MXFP4 workloads compute with the weights their encoding represents
        enc = (lambda a: mxfp4_round_trip(a, lib=self.lib)) if wl.weights == "mxfp4" else (lambda a: a)
        for e in need:
            if self._gu[e] is None:
                self._gu[e] = enc(synth.w_gateup_expert_host(wl, int(e)))
                self._dn[e] = enc(synth.w_down_expert_host(wl, int(e)))
        if wl.shared_f and self._shared is None:
            self._shared = tuple(enc(a) for a in synth.shared_host(wl))
        return self._shared if self._shared else (None, None)

    def outputs(self, tokens, nthreads: int | None = None) -> np.ndarray:
        wl = self.wl
        tokens = np.asarray(tokens, dtype=np.int32)
        sgu, sdn = self._load_weights(tokens)
        if len(tokens) == 0:
            return np.zeros((0, wl.d))
        return moe_tokens(self.x, self._gu, self._dn, self.idx, self.w, tokens, sgu, sdn, nthreads=nthreads,
                          lib=self.lib)

"""The sparse MoE feed-forward layer as a sequence of C-ABI calls.

Blog post "Mixture of Experts (MoEs) in Transformers": the layer keeps the transformer backbone and
replaces the dense feed-forward block with experts and a router (section "From Dense to Sparse"); at
run time it dispatches tokens to their selected experts, runs the projections, applies the routing
weights and collects the results in token order (section "Expert Backend"), here the grouped_mm way:
sort by expert id, group, one grouped GEMM over all experts.

This module owns device buffers (allocated with torch; the library never allocates) and calls the five
library entry points in order on one stream. It does no arithmetic of its own.
"""
from __future__ import annotations

import copy

import torch

from . import _native as N


def _encode_mxfp4(*ws):
    """bf16 weights [G_i, N, K] (one or more tensors, stacked on dim 0 in the order given) -> (codes
    [sum G_i, N, K/2], scales [sum G_i, K/32, N]) on the weights' device."""
    G = sum(w.shape[0] for w in ws)
    _, Nr, K = ws[0].shape
    q = torch.empty(G, Nr, K // 2, dtype=torch.uint8, device=ws[0].device)
    s = torch.empty(G, K // 32, Nr, dtype=torch.uint8, device=ws[0].device)
    g = 0
    for w in ws:
        N.mxfp4_quantize(w, q[g:g + w.shape[0]], s[g:g + w.shape[0]])
        g += w.shape[0]
    return q, s


class MoEFFN:
    """One MoE feed-forward layer with packed expert weights.

    w_router [E, d] fp32; w_gateup [E, 2f, d] bf16 (gate rows, then up rows); w_down [E, d, f] bf16;
    bias [E] fp32 or None; optional shared expert w_gateup_shared [2fs, d], w_down_shared [d, fs].
    weights: "bf16" keeps the expert weights as given; "mxfp4" encodes them once (moe_mxfp4_quantize, 4.25 bits
    per weight) and the layer then computes with the weights the encoding represents, through the MXFP4 grouped
    GEMMs; the bf16 tensors are not kept.
    fused: with bf16 weights and groups of 128 rows or more on average (prefill), let the dispatch and the
    collect steps ride in the grouped GEMMs: the gate|up GEMM reads its rows straight from x through perm_src
    (moe_grouped_gemm_gateup_gather) instead of a grouped copy x_perm made by moe_permute, and the down GEMM's
    epilogue does the weighted combine (moe_grouped_gemm_down_combine). Same results, bit for bit; the backward
    pass then gathers x_perm itself. Off by default: on B200 the separate gather and combine kernels are faster
    (the per-row gather loads and the combine's arrival counting slow the GEMMs by more than the two kernels
    take).
    """

    def __init__(self, w_router, w_gateup, w_down, k: int, route: str = "topk_softmax", bias=None,
                 w_gateup_shared=None, w_down_shared=None, weights: str = "bf16", fused: bool = False):
        self.E, self.d = w_router.shape
        self.f = w_gateup.shape[1] // 2
        self.k = k
        self.route = route
        if route not in N.ROUTE_MODES:
            raise ValueError(f"unknown routing mode {route!r}")
        if weights not in ("bf16", "mxfp4"):
            raise ValueError(f"unknown weight format {weights!r}")
        self.weights = weights
        self.fused = fused
        self._x_perm_valid = False
        self.w_router, self.w_gateup, self.w_down, self.bias = w_router, w_gateup, w_down, bias
        self.w_gateup_shared, self.w_down_shared = w_gateup_shared, w_down_shared
        self.shared_f = w_gateup_shared.shape[0] // 2 if w_gateup_shared is not None else 0
        self.device = w_gateup.device
        # MXFP4 with a shared expert as wide as a routed one: its weights are encoded as group E of the routed
        # tensors; for decode-sized T (_fold) its T rows (x itself) follow the R routed rows, and the routed GEMM
        # launches compute it as one more group, spread over every SM like the rest (on its own it is one group of
        # T rows, which the MXFP4 kernels run on a few SMs: 139 us on the decode layer's side stream, half of it
        # after the routing and grouping beside it; folded in, it adds 3.6% to the routed GEMMs' work, and on one
        # box the decode layer took 1.206-1.212 ms against 1.210-1.216 ms, at a power-capped clock 2-3% lower)
        self.fold_shared = weights == "mxfp4" and self.shared_f == self.f and self.shared_f > 0
        if weights == "mxfp4":
            E = self.E
            if self.fold_shared:  # the routed and shared names are views of the stacked tensors
                qg, sg = self.mx_gateup_all = _encode_mxfp4(w_gateup, w_gateup_shared.unsqueeze(0))
                qd, sd = self.mx_down_all = _encode_mxfp4(w_down, w_down_shared.unsqueeze(0))
                self.mx_gateup, self.mx_down = (qg[:E], sg[:E]), (qd[:E], sd[:E])
                self.mx_gateup_shared, self.mx_down_shared = (qg[E:], sg[E:]), (qd[E:], sd[E:])
            else:
                self.mx_gateup = _encode_mxfp4(w_gateup)
                self.mx_down = _encode_mxfp4(w_down)
                if self.shared_f:
                    self.mx_gateup_shared = _encode_mxfp4(w_gateup_shared.unsqueeze(0))
                    self.mx_down_shared = _encode_mxfp4(w_down_shared.unsqueeze(0))
            self.w_gateup = self.w_down = self.w_gateup_shared = self.w_down_shared = None
        self._T = None
        self.buf = {}
        # the tensor-core router (E <= 128) reads W_r as three bf16 pieces: split once here, not in every call
        self.w_pieces = None
        if self.E <= 128:
            self.w_pieces = torch.empty(3, self.E, self.d, dtype=torch.bfloat16, device=self.device)
            self.refresh_router()
        # the shared expert depends only on x: it runs on a side stream, beside routing and grouping (which
        # leave most SMs free), and the routed GEMMs wait for it
        self._side = torch.cuda.Stream(self.device) if self.shared_f else None

    def sibling(self) -> "MoEFFN":
        """Another layer over the same weights (nothing is copied or re-encoded) with its own intermediate buffers
        and side stream, so that two calls can be in flight at once."""
        twin = copy.copy(self)
        twin.buf, twin._T = {}, None
        twin._gbuf, twin._gT, twin._gu_saved = None, None, False  # its own backward buffers too
        twin._side = torch.cuda.Stream(self.device) if self.shared_f else None
        return twin

    def refresh_router(self):
        """Re-split the router weights; call after changing w_router in place."""
        if self.w_pieces is not None:
            N.router_split_weights(self.w_router, self.w_pieces)

    def buffers(self, T: int) -> dict:
        """Allocate (once per T) every intermediate the layer writes."""
        if self._T == T:
            return self.buf
        dev, E, d, f, k = self.device, self.E, self.d, self.f, self.k
        R = T * k
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        b = {
            "logits": torch.empty(T, E, dtype=f32, device=dev),
            "topk_idx": torch.empty(T, k, dtype=i32, device=dev),
            "topk_w": torch.empty(T, k, dtype=f32, device=dev),
            "counts": torch.empty(E, dtype=i32, device=dev),
            "offsets": torch.empty(E + 1, dtype=i32, device=dev),
            "perm_src": torch.empty(R, dtype=i32, device=dev),
            "inv_perm": torch.empty(R, dtype=i32, device=dev),
            "x_perm": torch.empty(R, d, dtype=bf, device=dev),
            "h": torch.empty(R, f, dtype=bf, device=dev),
            "y_perm": torch.empty(R, d, dtype=bf, device=dev),
            "ws": torch.empty(max(N.permute_workspace_size(T, E, k), 256), dtype=torch.uint8, device=dev),
            "combine_ws": torch.empty(max(N.grouped_gemm_down_combine_workspace_size(T, d), 256), dtype=torch.uint8,
                                      device=dev),
            "y": torch.empty(T, d, dtype=bf, device=dev),
        }
        if self._fold(T):
            # the R routed rows, then the shared expert's T rows (group E, offsets[E + 1] = R + T); the routed-only
            # names are views of the first R rows and E + 1 offsets
            b["offsets_all"] = torch.full((E + 2,), R + T, dtype=i32, device=dev)
            b["x_perm_all"] = torch.empty(R + T, d, dtype=bf, device=dev)
            b["h_all"] = torch.empty(R + T, f, dtype=bf, device=dev)
            b["y_perm_all"] = torch.empty(R + T, d, dtype=bf, device=dev)
            b["offsets"] = b["offsets_all"][:E + 1]
            b["x_perm"], b["h"], b["y_perm"] = b["x_perm_all"][:R], b["h_all"][:R], b["y_perm_all"][:R]
            b["shared_rows"] = torch.arange(T, dtype=i32, device=dev)
            b["shared"] = b["y_perm_all"][R:]
        elif self.shared_f:
            b["shared_offsets"] = torch.tensor([0, T], dtype=i32, device=dev)
            b["h_shared"] = torch.empty(T, self.shared_f, dtype=bf, device=dev)
            b["shared"] = torch.empty(T, d, dtype=bf, device=dev)
        self.buf, self._T = b, T
        return b

    def forward(self, x, stream=None, timing=None, train: bool = False):
        """y = MoE(x) for x [T, d] bf16 on the GPU. Returns the layer's output buffer [T, d] (bf16).

        train: keep the routed experts' gate|up pre-activations (moe_grouped_gemm_gateup_save, bf16 weights) so
        that the following backward() does not recompute them; the output is the same.

        timing: optional dict; if given, a (start, end) pair of CUDA events is recorded around each stage
        ("route", "permute", "gateup", "down", "combine" on the layer's stream; "shared", the always-on
        expert, on the side stream where it overlaps routing and grouping: its GEMMs, or, folded into the routed
        GEMMs (MXFP4), the copy of its rows).
        """
        T = x.shape[0]
        b = self.buffers(T)
        s = stream if stream is not None else torch.cuda.current_stream(x.device)
        self._x = x  # the backward pass reads the forward's input and intermediates

        def mark(name, first):
            if timing is None:
                return
            if first:
                timing[name] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            timing[name][0 if first else 1].record(s)

        shared = None
        if self.shared_f:
            side = self._side
            x_ready = torch.cuda.Event()
            x_ready.record(s)
            side.wait_event(x_ready)  # also orders after the previous call's combine, which read `shared`
            if timing is not None:
                timing["shared"] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                timing["shared"][0].record(side)
            if self._fold(T):  # its rows after the routed ones; the routed GEMMs compute it
                N.gather_rows(x, b["shared_rows"], b["x_perm_all"][T * self.k:], side)
            else:
                self._gateup(x, "shared", b["shared_offsets"], b["h_shared"], side)
                self._down(b["h_shared"], "shared", b["shared_offsets"], b["shared"], side)
            shared_done = torch.cuda.Event()
            shared_done.record(side)
            if timing is not None:
                timing["shared"][1].record(side)
            shared = b["shared"]
        mark("route", True)
        if self.w_pieces is not None:
            N.route_topk_split(x, self.w_router, self.w_pieces, self.bias, self.k, self.route, b["logits"],
                               b["topk_idx"], b["topk_w"], s)
        else:
            N.route_topk(x, self.w_router, self.bias, self.k, self.route, b["logits"], b["topk_idx"], b["topk_w"], s)
        mark("route", False)
        fused = self._fused(T) and not train  # the saving gate|up GEMM reads x_perm
        save = train and self.weights == "bf16"
        self._gu_saved = False
        mark("permute", True)
        if fused:  # grouping only; the gate|up GEMM gathers its rows from x
            N.permute(None, b["topk_idx"], self.E, b["counts"], b["offsets"], b["perm_src"], b["inv_perm"], None,
                      b["ws"], s)
        else:
            N.permute(x, b["topk_idx"], self.E, b["counts"], b["offsets"], b["perm_src"], b["inv_perm"], b["x_perm"],
                      b["ws"], s)
        self._x_perm_valid = not fused
        mark("permute", False)
        if shared is not None:
            # the routed GEMMs are persistent kernels sized to every SM: they start once the shared expert is done
            # (or, folded, its rows are in place)
            s.wait_event(shared_done)
        mark("gateup", True)
        if fused:
            N.grouped_gemm_gateup_gather(x, b["perm_src"], self.w_gateup, b["offsets"], b["h"], None, s)
        elif save:
            N.grouped_gemm_gateup_save(b["x_perm"], self.w_gateup, b["offsets"], b["h"], self._grad_buffers(T)["gu"], s)
            self._gu_saved = True
        else:
            self.routed_gateup(b, s)
        mark("gateup", False)
        mark("down", True)
        if fused:  # y_perm and, in the same kernel, y
            N.grouped_gemm_down_combine(b["h"], self.w_down, b["offsets"], b["perm_src"], b["inv_perm"],
                                        b["topk_w"], shared, b["y_perm"], b["y"], b["combine_ws"], s)
            mark("down", False)
            return b["y"]
        self.routed_down(b, s)
        mark("down", False)
        mark("combine", True)
        N.unpermute_combine(b["y_perm"], b["inv_perm"], b["topk_w"], shared, b["y"], s)
        mark("combine", False)
        return b["y"]

    __call__ = forward

    def _fused(self, T: int) -> bool:
        """Whether forward() folds the row gather into the gate|up GEMM and the combine into the down GEMM for
        T tokens."""
        return (self.fused and self.weights == "bf16" and T > 0
                and N.grouped_gemm_gateup_gather_workspace_size(self.E, T * self.k, self.d) == 0)

    def _fold(self, T: int) -> bool:
        """Whether forward() computes the shared expert inside the routed MXFP4 GEMMs for T tokens: when the
        R + T rows stay within the decode kernel's range (at most 8 rows per group on average, as the library's
        dispatch decides), so that the routed experts keep that kernel, and E + 1 groups are within the grouped
        GEMMs' limit of 1024."""
        return (self.fold_shared and T > 0 and T * self.k + T <= 8 * (self.E + 1)
                and self.E + 1 <= N.MAX_GEMM_GROUPS)

    def routed_gateup(self, b, stream):
        """The routed gate|up GEMM of forward() on buffers b (with the folded shared expert as group E)."""
        if "x_perm_all" in b:
            q, sc = self.mx_gateup_all
            N.grouped_gemm_gateup_mxfp4(b["x_perm_all"], q, sc, b["offsets_all"], b["h_all"], stream)
        else:
            self._gateup(b["x_perm"], "routed", b["offsets"], b["h"], stream)

    def routed_down(self, b, stream):
        """The routed down GEMM of forward() on buffers b (with the folded shared expert as group E)."""
        if "x_perm_all" in b:
            q, sc = self.mx_down_all
            N.grouped_gemm_down_mxfp4(b["h_all"], q, sc, b["offsets_all"], b["y_perm_all"], stream)
        else:
            self._down(b["h"], "routed", b["offsets"], b["y_perm"], stream)

    def _gateup(self, a, which, offsets, h, stream):
        if self.weights == "mxfp4":
            q, sc = self.mx_gateup if which == "routed" else self.mx_gateup_shared
            N.grouped_gemm_gateup_mxfp4(a, q, sc, offsets, h, stream)
        else:
            w = self.w_gateup if which == "routed" else self.w_gateup_shared.unsqueeze(0)
            N.grouped_gemm_gateup(a, w, offsets, h, stream)

    def _down(self, h, which, offsets, y, stream):
        if self.weights == "mxfp4":
            q, sc = self.mx_down if which == "routed" else self.mx_down_shared
            N.grouped_gemm_down_mxfp4(h, q, sc, offsets, y, stream)
        else:
            w = self.w_down if which == "routed" else self.w_down_shared.unsqueeze(0)
            N.grouped_gemm_down(h, w, offsets, y, stream)

    # ---- training: gradients of the last forward() call ----------------------------------------------------

    def _transposed(self):
        """Per-expert transposed weight copies for the backward GEMMs, made once (call refresh_backward after
        changing the weights in place)."""
        if getattr(self, "_wt", None) is None:
            if self.weights != "bf16":
                raise NotImplementedError("the backward pass needs the bf16 expert weights")
            E, d, f = self.E, self.d, self.f
            wt = {"down": torch.empty(E, f, d, dtype=torch.bfloat16, device=self.device),
                  "gateup": torch.empty(E, d, 2 * f, dtype=torch.bfloat16, device=self.device)}
            N.transpose_weights(self.w_down, wt["down"])
            N.transpose_weights(self.w_gateup, wt["gateup"])
            if self.shared_f:
                fs = self.shared_f
                wt["down_shared"] = torch.empty(1, fs, d, dtype=torch.bfloat16, device=self.device)
                wt["gateup_shared"] = torch.empty(1, d, 2 * fs, dtype=torch.bfloat16, device=self.device)
                N.transpose_weights(self.w_down_shared.unsqueeze(0), wt["down_shared"])
                N.transpose_weights(self.w_gateup_shared.unsqueeze(0), wt["gateup_shared"])
            self._wt = wt
        return self._wt

    def refresh_backward(self):
        """Drop the transposed weight copies (rebuilt by the next backward)."""
        self._wt = None

    def _grad_buffers(self, T: int) -> dict:
        if getattr(self, "_gT", None) == T:
            return self._gbuf
        dev, E, d, f, k = self.device, self.E, self.d, self.f, self.k
        R = T * k
        bf, f32 = torch.bfloat16, torch.float32
        g = {"dy_perm": torch.empty(R, d, dtype=bf, device=dev), "dtopk_w": torch.empty(T, k, dtype=f32, device=dev),
             "dh": torch.empty(R, f, dtype=bf, device=dev), "gu": torch.empty(R, 2 * f, dtype=bf, device=dev),
             "dgu": torch.empty(R, 2 * f, dtype=bf, device=dev), "dx_perm": torch.empty(R, d, dtype=bf, device=dev),
             "dx_router": torch.empty(T, d, dtype=bf, device=dev), "dx": torch.empty(T, d, dtype=bf, device=dev),
             "ones": torch.ones(T, k, dtype=f32, device=dev),
             "router_ws": torch.empty(max(N.router_backward_workspace_size(T, d, E, k), 256), dtype=torch.uint8,
                                      device=dev),
             "dw_router": torch.empty(E, d, dtype=f32, device=dev),
             "dbias": torch.empty(E, dtype=f32, device=dev) if self.bias is not None else None,
             "dw_down": torch.empty(E, d, f, dtype=f32, device=dev),
             "dw_gateup": torch.empty(E, 2 * f, d, dtype=f32, device=dev)}
        wsz = max(N.grouped_weight_grad_workspace_size(max(R, 1), E, d, f),
                  N.grouped_weight_grad_workspace_size(max(R, 1), E, 2 * f, d))
        if self.shared_f:
            fs = self.shared_f
            g.update({"dh_s": torch.empty(T, fs, dtype=bf, device=dev), "gu_s": torch.empty(T, 2 * fs, dtype=bf, device=dev),
                      "dgu_s": torch.empty(T, 2 * fs, dtype=bf, device=dev), "dx_s": torch.empty(T, d, dtype=bf, device=dev),
                      "dw_down_shared": torch.empty(1, d, fs, dtype=f32, device=dev),
                      "dw_gateup_shared": torch.empty(1, 2 * fs, d, dtype=f32, device=dev)})
            wsz = max(wsz, N.grouped_weight_grad_workspace_size(max(T, 1), 1, d, fs),
                      N.grouped_weight_grad_workspace_size(max(T, 1), 1, 2 * fs, d))
        g["wgrad_ws"] = torch.empty(max(wsz, 256), dtype=torch.uint8, device=dev)
        self._gbuf, self._gT = g, T
        return g

    def backward(self, dy, stream=None, weight_grads: bool = True, timing=None) -> dict:
        """Gradients of the last forward() call for the upstream gradient dy [T, d] (bf16), the top-k selection
        held fixed. Returns a dict of device tensors owned by the layer (overwritten by the next backward):
        dx [T, d] bf16 (experts and router), dtopk_w [T, k] (routing weights), dw_router [E, d], dbias [E] (with
        a router bias), and with weight_grads dw_gateup [E, 2f, d], dw_down [E, d, f] (fp32), plus the shared
        expert's dw_gateup_shared [1, 2fs, d] and dw_down_shared [1, d, fs].
        timing: optional dict; if given, (start, end) CUDA events are recorded around each stage ("bwd_permute",
        "bwd_dh", "bwd_preact", "bwd_swiglu", "bwd_dx_perm", "bwd_shared", "bwd_router", "bwd_combine", "bwd_dw_down",
        "bwd_dw_gateup", "bwd_dw_shared")."""
        T = dy.shape[0]
        if self._T != T or getattr(self, "_x", None) is None or self._x.shape[0] != T:
            raise RuntimeError("backward() follows a forward() over the same tokens")
        s = stream if stream is not None else torch.cuda.current_stream(dy.device)
        b = self.buf
        wt = self._transposed()
        g = self._grad_buffers(T)
        x = self._x

        def mark(name, first):
            if timing is None:
                return
            if first:
                timing[name] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            timing[name][0 if first else 1].record(s)

        mark("bwd_permute", True)
        N.permute_backward(dy, b["inv_perm"], b["topk_w"], b["y_perm"], g["dy_perm"], g["dtopk_w"], s)
        mark("bwd_permute", False)
        mark("bwd_dh", True)
        N.grouped_gemm_down(g["dy_perm"], wt["down"], b["offsets"], g["dh"], s)
        mark("bwd_dh", False)
        mark("bwd_preact", True)
        if not self._x_perm_valid:  # the forward gathered its rows inside the GEMM: x_perm is made here
            N.gather_rows(x, b["perm_src"], b["x_perm"], s)
            self._x_perm_valid = True
        if not getattr(self, "_gu_saved", False):  # a training forward kept them
            N.grouped_gemm_gateup_preact(b["x_perm"], self.w_gateup, b["offsets"], g["gu"], s)
        mark("bwd_preact", False)
        mark("bwd_swiglu", True)
        N.swiglu_backward(g["dh"], g["gu"], g["dgu"], s)
        mark("bwd_swiglu", False)
        mark("bwd_dx_perm", True)
        N.grouped_gemm_down(g["dgu"], wt["gateup"], b["offsets"], g["dx_perm"], s)
        mark("bwd_dx_perm", False)
        addend = None
        if self.shared_f:
            mark("bwd_shared", True)
            so = b["shared_offsets"]
            N.grouped_gemm_down(dy, wt["down_shared"], so, g["dh_s"], s)
            N.grouped_gemm_gateup_preact(x, self.w_gateup_shared.unsqueeze(0), so, g["gu_s"], s)
            N.swiglu_backward(g["dh_s"], g["gu_s"], g["dgu_s"], s)
            N.grouped_gemm_down(g["dgu_s"], wt["gateup_shared"], so, g["dx_s"], s)
            addend = g["dx_s"]
            mark("bwd_shared", False)
        mark("bwd_router", True)
        N.router_backward(x, self.w_router, b["logits"], b["topk_idx"], b["topk_w"], g["dtopk_w"], b["perm_src"],
                          b["inv_perm"], b["offsets"], self.route, g["dx_router"], g["dw_router"], g["dbias"], addend,
                          g["router_ws"], s)
        mark("bwd_router", False)
        mark("bwd_combine", True)
        N.unpermute_combine(g["dx_perm"], b["inv_perm"], g["ones"], g["dx_router"], g["dx"], s)
        mark("bwd_combine", False)
        out = {"dx": g["dx"], "dtopk_w": g["dtopk_w"], "dw_router": g["dw_router"], "dbias": g["dbias"]}
        if weight_grads:
            mark("bwd_dw_down", True)
            N.grouped_weight_grad(g["dy_perm"], b["h"], b["offsets"], g["dw_down"], g["wgrad_ws"], s)
            mark("bwd_dw_down", False)
            mark("bwd_dw_gateup", True)
            N.grouped_weight_grad(g["dgu"], b["x_perm"], b["offsets"], g["dw_gateup"], g["wgrad_ws"], s)
            mark("bwd_dw_gateup", False)
            out["dw_down"], out["dw_gateup"] = g["dw_down"], g["dw_gateup"]
            if self.shared_f:
                mark("bwd_dw_shared", True)
                so = b["shared_offsets"]
                N.grouped_weight_grad(dy, b["h_shared"], so, g["dw_down_shared"], g["wgrad_ws"], s)
                N.grouped_weight_grad(g["dgu_s"], x, so, g["dw_gateup_shared"], g["wgrad_ws"], s)
                mark("bwd_dw_shared", False)
                out["dw_down_shared"], out["dw_gateup_shared"] = g["dw_down_shared"], g["dw_gateup_shared"]
        return out

    def backward_kernel_launches(self, T: int, weight_grads: bool = True, train_forward: bool = False) -> int:
        """Kernels one backward() launches: permute-backward 1, dh 1, pre-activations 1 (none after a training
        forward, which kept them; + 1 gather of x_perm after a forward that folded it into the gate|up GEMM),
        SwiGLU-backward 1, dx_perm 1, router 5, combine 1, and per weight gradient 4 (padded offsets, two
        transposes, the GEMM); the shared expert 4 more (+ 8 with weight gradients)."""
        if T <= 0:
            return 0
        n = 11 + (8 if weight_grads else 0)
        if train_forward:
            n -= 1
        elif self._fused(T):
            n += 1
        if self.shared_f:
            n += 4 + (8 if weight_grads else 0)
        return n

    def kernel_launches(self, T: int, train: bool = False) -> int:
        """Kernels one forward() launches (mirrors the library's dispatch): the router is one kernel when the
        tensor-core path with fused top-k is taken (E <= 128, T >= 2048), else logits + top-k;
        permute 4, gate|up, down, combine 1 each (fused: permute 3, gate|up 1, down with combine 1; train: the
        gate|up that keeps its pre-activations is 1 kernel with 128 rows or more per expert, else 2); the shared
        expert 2 more (1 folded: the copy of its rows)."""
        if T <= 0:
            return 0
        route = 1 if (self.E <= 128 and T >= 2048) else 2
        if train and self.weights == "bf16":
            body = 4 + 3 + (0 if T * self.k >= 128 * self.E else 1)
        else:
            body = 3 + 2 if self._fused(T) else 4 + 3
        return route + body + ((1 if self._fold(T) else 2) if self.shared_f else 0)

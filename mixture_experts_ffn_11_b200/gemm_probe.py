"""Run one grouped-GEMM configuration on its own, for timing or for a profiler.

    python -m mixture_experts_ffn_11_b200.gemm_probe --weights mxfp4 --experts 64 --rows 2 --d 7168 --f 2048

Draws random bf16 weights (seeded torch generator, N(0, 0.02)) and activations (N(0, 1)), encodes the weights when
--weights mxfp4, gives every expert --rows rows, and calls the chosen projection (--proj gateup or down) --launches
times through the C-ABI, printing the mean device time per launch (CUDA events, after the first launch). A profiler
can select one launch of the kernel with its skip / count options.
"""
from __future__ import annotations

import argparse

import torch

from . import _native as N


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--weights", choices=["bf16", "mxfp4"], default="mxfp4")
    ap.add_argument("--proj", choices=["gateup", "down"], default="gateup")
    ap.add_argument("--experts", type=int, default=64)
    ap.add_argument("--rows", type=int, default=2, help="rows per expert")
    ap.add_argument("--d", type=int, default=7168)
    ap.add_argument("--f", type=int, default=2048)
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args(argv)
    torch.cuda.set_device(0)
    G, d, f, rows = a.experts, a.d, a.f, a.rows
    M = G * rows
    gen = torch.Generator(device="cuda").manual_seed(0)
    n_rows, K, n_out = (2 * f, d, f) if a.proj == "gateup" else (d, f, d)
    w = (torch.randn(G, n_rows, K, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    if a.weights == "mxfp4":
        q = torch.empty(G, n_rows, K // 2, dtype=torch.uint8, device="cuda")
        s = torch.empty(G, K // 32, n_rows, dtype=torch.uint8, device="cuda")
        N.mxfp4_quantize(w, q, s)
        del w
    x = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
    off = torch.arange(0, M + 1, rows, dtype=torch.int32, device="cuda")
    out = torch.empty(M, n_out, dtype=torch.bfloat16, device="cuda")

    def launch():
        if a.weights == "mxfp4":
            fn = N.grouped_gemm_gateup_mxfp4 if a.proj == "gateup" else N.grouped_gemm_down_mxfp4
            fn(x, q, s, off, out)
        else:
            fn = N.grouped_gemm_gateup if a.proj == "gateup" else N.grouped_gemm_down
            fn(x, w, off, out)

    launch()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(a.launches - 1):
        launch()
    t1.record()
    torch.cuda.synchronize()
    if N.get_device_error():
        raise SystemExit("device error word set")
    per = t0.elapsed_time(t1) * 1e3 / max(a.launches - 1, 1)
    print(f"{a.weights} {a.proj} G={G} rows={rows} d={d} f={f}: {per:.1f} us per launch (after the first)")


if __name__ == "__main__":
    main()

"""bench.py's roofline arithmetic on the CPU: algorithmic FLOPs and bytes of the grouped GEMMs and the layer, the
choice of bound, and the keying of the captured DRAM traffic on the GEMM sources (comments do not count)."""
import os
import shutil

import numpy as np
import pytest

import bench
import synth


def test_gemm_figures_gpt_oss_shape():
    wl = synth.workload("gpt-oss-20b-prefill")
    counts = np.full(wl.E, wl.R // wl.E)
    active, gu, dn = bench.gemm_figures(wl, counts)
    R, d, f = wl.R, wl.d, wl.f
    assert active == wl.E
    assert gu["flop"] == 4.0 * R * d * f and dn["flop"] == 2.0 * R * d * f
    # weights once (bf16) + activations in + outputs out
    assert gu["bytes"] == wl.E * 2 * f * d * 2 + R * d * 2 + R * f * 2
    assert dn["bytes"] == wl.E * d * f * 2 + R * f * 2 + R * d * 2


def test_gemm_figures_count_only_active_experts_and_mxfp4_bytes():
    wl = synth.workload("decode-256e-shared-mxfp4")
    counts = np.zeros(wl.E, dtype=np.int64)
    counts[:200] = 2
    counts[200] = wl.R - 400
    active, gu, _ = bench.gemm_figures(wl, counts)
    assert active == 201
    wb = 0.5 + 1.0 / 32  # a 4-bit code and 1/32 of an 8-bit scale per weight
    assert bench.weight_bytes(wl) == wb
    assert gu["bytes"] == pytest.approx(201 * 2 * wl.f * wl.d * wb + wl.R * wl.d * 2 + wl.R * wl.f * 2)


def test_gemm_figures_count_a_folded_shared_expert_once():
    wl = synth.workload("decode-256e-shared-mxfp4")
    counts = np.zeros(wl.E, dtype=np.int64)
    counts[:wl.R // 2] = 2
    a0, gu0, dn0 = bench.gemm_figures(wl, counts)
    a1, gu1, dn1 = bench.gemm_figures(wl, counts, folded_shared=True)
    assert a1 == a0 == wl.R // 2
    T, d, f, wb = wl.T, wl.d, wl.f, bench.weight_bytes(wl)
    # one more group: its weights once, its T rows in and out
    assert gu1["bytes"] - gu0["bytes"] == pytest.approx(2 * f * d * wb + T * d * 2 + T * f * 2)
    assert dn1["bytes"] - dn0["bytes"] == pytest.approx(d * f * wb + T * f * 2 + T * d * 2)
    assert gu1["flop"] - gu0["flop"] == 4.0 * T * d * f and dn1["flop"] - dn0["flop"] == 2.0 * T * d * f


def test_roofline_entry_picks_the_slower_bound():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    # 1 TFLOP and 1 GB: 1 ms of tensor work against 0.2 ms of bytes -> tensor-bound; 2 ms measured -> 0.5
    e = bench.roofline_entry("k", {"flop": 1e12, "bytes": 1e9}, 2.0, peaks, "bf16_tflops", 123)
    assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s"
    assert e["achieved"] == pytest.approx(500.0) and e["frac"] == pytest.approx(0.5)
    assert e["traffic"] == 123
    # 1 GFLOP and 10 GB: 2 ms of bytes -> HBM-bound; 4 ms measured -> 2500 GB/s, 0.5
    e = bench.roofline_entry("k", {"flop": 1e9, "bytes": 1e10}, 4.0, peaks, "bf16_tflops", None)
    assert e["bound"] == "hbm" and e["unit"] == "GB/s"
    assert e["achieved"] == pytest.approx(2500.0) and e["frac"] == pytest.approx(0.5)


def test_layer_figures_include_shared_expert_and_router():
    wl = synth.workload("decode-256e-shared")
    flop, nbytes = bench.layer_figures(wl, active=222)
    wb = 2.0
    assert nbytes == 222 * 3 * wl.d * wl.f * wb + 3 * wl.d * wl.shared_f * wb + wl.T * wl.d * 2 * 2 + wl.E * wl.d * 4
    assert flop == wl.flops()


def test_traffic_table_is_keyed_on_one_capture():
    """The recorded figures come from one capture (one source hash) and cover the headline GEMMs; the bench reports
    them only while the GEMM sources still hash to that value (else traffic is null)."""
    h = bench.kernel_source_hash()
    assert len(h) == 16
    keys = {k[2] for k in bench.TRAFFIC}
    assert len(keys) == 1
    assert {(k[0], k[1]) for k in bench.TRAFFIC} >= {("grouped_gemm_gateup", "gpt-oss-20b-prefill"),
                                                    ("grouped_gemm_down", "gpt-oss-20b-prefill")}
    if keys != {h}:
        pytest.skip("the GEMM sources changed since the traffic capture: the bench reports traffic as null")


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    src_dir = tmp_path / "mixture_experts_ffn_11_b200" / "csrc"
    src_dir.mkdir(parents=True)
    for p in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, p), tmp_path / p)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    target = tmp_path / bench.KERNEL_SOURCES[0]
    target.write_text("// a comment\n\n" + target.read_text() + "\n/* block\ncomment */\n")
    assert bench.kernel_source_hash() == h0
    target.write_text(target.read_text() + "\nint moe_extra_symbol;\n")
    assert bench.kernel_source_hash() != h0

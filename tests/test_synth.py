"""The seeded input generator (shared by the oracle and the CUDA path; no layer arithmetic)."""
import numpy as np

import oracle
import synth


def test_deterministic_and_subrange_consistent():
    a = synth.normal_bf16(0, 2, 0, 50_000, 0.02)
    b = synth.normal_bf16(0, 2, 0, 50_000, 0.02)
    assert (a == b).all()
    c = synth.normal_bf16(0, 2, 12_345, 1000, 0.02)
    assert (c == a[12_345:13_345]).all()
    assert not (synth.normal_bf16(1, 2, 0, 1000, 0.02) == a[:1000]).all()
    assert not (synth.normal_bf16(0, 3, 0, 1000, 0.02) == a[:1000]).all()


def test_bf16_is_rne_of_f32():
    f = synth.normal_f32(0, 0, 0, 100_000, 1.0)
    b = synth.normal_bf16(0, 0, 0, 100_000, 1.0)
    assert (synth.f32_to_bf16_bits(f) == b).all()
    # RNE: |bf16 - f32| <= half an ulp of bf16
    err = np.abs(synth.bf16_bits_to_f32(b).astype(np.float64) - f)
    assert (err <= np.abs(f) * 2.0 ** -8 + 1e-30).all()


def test_moments():
    f = synth.normal_f32(0, 7, 0, 2_000_000, 1.0).astype(np.float64)
    assert abs(f.mean()) < 3e-3
    assert abs(f.std() - 1.0) < 3e-3
    # Irwin-Hall(12) excess kurtosis is -0.1
    k = ((f - f.mean()) ** 4).mean() / f.var() ** 2 - 3
    assert -0.13 < k < -0.07
    assert np.abs(f).max() <= 6.0


def test_zipf_bias_skews_load():
    """Zipf(1.2) router bias on the 128-expert workload leaves some experts empty and a few above 5%."""
    wl = synth.workload("zipf-128e")
    ref = oracle.LayerReference(wl)
    share = ref.counts / wl.R
    assert (ref.counts == 0).sum() >= 1
    assert (share > 0.05).sum() >= 1
    assert ref.counts.sum() == wl.R


def test_workload_table():
    for name, w in synth.WORKLOADS.items():
        assert w.k <= w.E and w.d % 8 == 0 and w.f % 8 == 0
    assert synth.workload("gpt-oss-20b-prefill").flops() == 6.0 * 4096 * 4 * 2880 * 2880

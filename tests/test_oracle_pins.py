"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
import synth
from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.load())


def test_layer_reference_tiny_invariants():
    """The whole oracle pipeline on the tiny workload: routing and grouping invariants."""
    wl = synth.workload("tiny")
    ref = oracle.LayerReference(wl)
    assert ref.idx.shape == (wl.T, wl.k)
    assert ((ref.idx >= 0) & (ref.idx < wl.E)).all()
    assert all(len(set(r)) == wl.k for r in ref.idx.tolist())
    np.testing.assert_allclose(ref.w.sum(1), 1.0, atol=1e-12)
    # every selected logit >= every unselected logit (on the fp32 logits that decided)
    for t in range(wl.T):
        sel = set(ref.idx[t].tolist())
        lo = min(ref.logits32[t, e] for e in sel)
        hi = max((ref.logits32[t, e] for e in range(wl.E) if e not in sel), default=-np.inf)
        assert lo >= hi
    assert ref.counts.sum() == wl.R
    out = ref.outputs(np.arange(wl.T))
    assert out.shape == (wl.T, wl.d) and np.isfinite(out).all()

"""The seeded input generator: deterministic, independent of threading, shaped as stated."""
import numpy as np

import synth


def test_noise_and_filters_do_not_depend_on_threads():
    w = synth.Workload("t", 3, 5, 64, 4, "f32", 1e-3, 1e-1)
    assert np.array_equal(synth.noise(w, 7, threads=1), synth.noise(w, 7, threads=4))
    assert np.array_equal(synth.filters(w, 7, threads=1), synth.filters(w, 7, threads=3))


def test_filter_law_and_shapes():
    w = synth.Workload("t", 2, 3, 256, 1, "f32", 0.01, 0.02)
    h = synth.filters(w, 1)
    assert h.shape == (2, 3, 256) and h.dtype == np.float32
    lam = synth.decay_rates(w, 1)
    assert np.all((lam >= 0.01) & (lam <= 0.02))
    # dividing out the envelope leaves the unit normal draws
    g = h.astype(np.float64) / np.exp(-lam[..., None] * np.arange(256))
    assert abs(g.std() - 1.0) < 0.15
    sub = synth.filter_layer(w, 1, 1, lam, np.array([2]))
    assert np.array_equal(sub[0], h[1, 2])


def test_workloads_cover_the_five_shapes():
    names = set(synth.WORKLOADS)
    for n in ("tiny-1x16-L1K", "hyena-8x768-L8K", "hyena-18x864-L32K-B4", "longrange-4x1024-L128K-bf16",
              "sweep-8x2048-L16K-bf16-B1", "sweep-8x2048-L16K-bf16-B64"):
        assert n in names
    assert synth.WORKLOADS[synth.HEADLINE].layers == 18

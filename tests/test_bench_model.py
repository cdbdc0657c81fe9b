"""The roofline arithmetic of bench.py, on CPU.

The per-class byte model must add up to the closed form the schedule implies
(every block side on FFT: per (layer, channel) a spectrum of about 8U bytes,
per (layer, sequence, channel) U sources and an accumulator read-modify-write),
classify every block side exactly once, and count L - 1 blocks per stream in
total (one per step).
"""
import math

import pytest

import bench
import synth


@pytest.mark.parametrize("name", ["tiny-1x16-L1K", "hyena-18x864-L32K-B4", "sweep-8x2048-L16K-bf16-B64"])
def test_block_bytes_match_the_closed_form(name):
    w = synth.WORKLOADS[name]
    # chunk 1 puts no block on chip; FFT from side 1 up to L/2 puts every block on FFT
    model, _ = bench.cost_model(w, chunk=1, fft_from=1, fft_max=w.length)
    s = 2 if w.dtype == "bf16" else 4
    # the model's spectra hold U+1 values per side; the closed form counts U
    extra = sum(n * w.layers * w.channels * 8 for U, n in bench.schedule_levels(w.length))
    assert model["fft"]["bytes"] - extra == pytest.approx(bench.closed_form_block_bytes(w), rel=1e-12)
    assert model["fft"]["blocks"] == w.length - 1
    assert model["direct"]["bytes"] == 0 and model["tc"]["bytes"] == 0


def test_every_side_is_counted_once():
    w = synth.WORKLOADS["hyena-18x864-L32K-B4"]
    model, tot = bench.cost_model(w, chunk=64, fft_from=128, fft_max=1 << 14, tc_max=64)
    blocks = sum(v["blocks"] for v in model.values())
    assert blocks == w.length - 1
    levels = dict(bench.schedule_levels(w.length))
    assert model["chunk"]["blocks"] == sum(n for U, n in levels.items() if U < 64)
    assert model["tc"]["blocks"] == levels[64]
    assert model["fft"]["blocks"] == sum(n for U, n in levels.items() if 128 <= U <= 1 << 14)
    assert tot["bytes"] == pytest.approx(sum(v["bytes"] for v in model.values()))


def test_fft_flop_model():
    # two real transforms of 2U points at 2.5 * n * log2(n) each, plus 7U for the product
    assert bench.fft_flops(64) == pytest.approx(2 * 2.5 * 128 * 7 + 7 * 64)
    assert bench.fft_flops(1 << 14) == pytest.approx(5 * (1 << 15) * 15 + 7 * (1 << 14))
    assert math.isclose(bench.fft_flops(1024) / bench.fft_flops(512), 2 * 11 / 10, rel_tol=0.02)


@pytest.mark.parametrize("mlp_hidden", [0, 768])
def test_per_position_classes(mlp_hidden):
    # fi_step and the channel-mixing path add blocks of side <= 8 inside their
    # per-position launches ("token"); sides 16 and 32 are direct launches and
    # sides from fft_from FFT launches; every block is counted once.
    w = synth.WORKLOADS["hyena-18x864-L32K-B4"]
    model, tot = bench.per_position_model(w, fft_from=64, tc_max=0, mlp_hidden=mlp_hidden)
    levels = dict(bench.schedule_levels(w.length))
    assert model["token"]["blocks"] == sum(n for U, n in levels.items() if U <= 8)
    assert model["direct"]["blocks"] == levels[16] + levels[32]
    assert model["fft"]["blocks"] == sum(n for U, n in levels.items() if U >= 64)
    assert model["chunk"]["bytes"] == 0
    assert sum(v["blocks"] for v in model.values()) == w.length - 1
    assert tot["bytes"] == pytest.approx(sum(v["bytes"] for v in model.values()))


def test_per_token_path_of_a_deep_stack_fuses_no_block():
    # fi_step fuses blocks only for stacks of up to 32 layers
    w = synth.Workload("deep", 40, 8, 1024, 1, "f32", 1e-3, 1e-1)
    model, _ = bench.per_position_model(w, fft_from=64, tc_max=0)
    assert model["token"]["blocks"] == 0
    mlp, _ = bench.per_position_model(w, fft_from=64, tc_max=0, mlp_hidden=16)
    assert mlp["token"]["blocks"] == sum(n for U, n in bench.schedule_levels(w.length) if U <= 8)

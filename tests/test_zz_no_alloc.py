"""fi_generate_noalloc: the generation for callers that cannot allocate device memory.

Such callers (a thread with a hard latency budget, a framework that owns all
device memory, code running where allocation is not allowed) get their working
memory from one fixed device array inside the library. This file checks, through
the C-ABI, that two calls in a row give what the allocating path (fi_init +
fi_generate) gives, within the fp32 / bf16 tolerances the other parity tests use;
that the tiny workload matches the float64 oracle's own closed loop; that a second
call leaves the device's free memory unchanged; that a call does not disturb a
live context with a larger on-chip window; and that a configuration too large for
the fixed array is refused cleanly.
It sorts last so that a run stopping at its first failure has run everything else.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import (TOL, gpu_inputs, oracle_filters, read_all_activations,
                        teacher_forced_errors)

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _allocating_path(fi, w, inp):
    # The same plan as the fixed-memory path (direct blocks from the chunk side
    # up, FFT disabled), so the two runs sum in the same order.
    ctx = fi.Context(inp["h"], w.batch, w.dtype, fft_from=1 << 20)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1)
    ctx.sync()
    ctx.close()
    return y.cpu().numpy()


def _stream_errors(y, ref):
    # [n][B][D] -> per (b, d) stream, normwise over positions
    return oracle.stream_error(np.moveaxis(y, 0, -1), np.moveaxis(ref, 0, -1))


@pytest.mark.gpu
def test_noalloc_matches_allocating_path_twice(fi):
    cases = [synth.Workload("noalloc-a", 3, 16, 1024, 2, "f32", 1e-3, 1e-1),
             synth.Workload("noalloc-b", 2, 24, 512, 3, "bf16", 1e-5, 1e-3)]
    for k, w in enumerate(cases):
        inp = gpu_inputs(w, 40 + k)
        y = torch.full((w.length, w.batch, w.channels), float("nan"), dtype=torch.float32, device="cuda")
        fi.generate_noalloc(inp["h"], w.batch, w.length, inp["x0"], inp["eps"], y, w.dtype)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert np.all(np.isfinite(got))
        ref = _allocating_path(fi, w, inp)
        assert _stream_errors(got, ref) <= TOL[w.dtype], k


@pytest.mark.gpu
def test_noalloc_rejects_oversized_configuration(fi):
    w = synth.Workload("noalloc-big", 8, 512, 4096, 1, "f32", 1e-3, 1e-1)   # needs ~36 Mi floats
    h = torch.zeros((w.layers, w.channels, w.length), dtype=torch.float32, device="cuda")
    x0 = torch.zeros((1, w.channels), dtype=torch.float32, device="cuda")
    eps = torch.zeros((16, 1, w.channels), dtype=torch.float32, device="cuda")
    y = torch.zeros((16, 1, w.channels), dtype=torch.float32, device="cuda")
    with pytest.raises(fi.FiError) as e:
        fi.generate_noalloc(h, 1, 16, x0, eps, y)
    assert e.value.status == fi.FI_E_INVALID
    assert "floats of working memory" in str(e.value)


@pytest.mark.gpu
def test_noalloc_matches_oracle_closed_loop(fi):
    # Closed loop against the float64 oracle's own closed loop. The feedback of
    # the standard workloads is chaotic (rounding differences grow), so this case
    # uses short, scaled-down filters (decay rates 0.1..0.5, taps x 0.1) whose
    # loop gain is below one: differences stay at rounding level over all 1024
    # positions (a relative perturbation of 1e-6 moves the oracle's output by
    # 3e-6), and every position can be held to the fp32 tolerance.
    w = synth.Workload("noalloc-contractive", 2, 16, 1024, 2, "f32", 0.1, 0.5)
    h = (synth.filters(w, 9) * np.float32(0.1)).astype(np.float32)
    x0 = synth.first_token(w, 9)
    eps = synth.noise(w, 9)
    d_of = np.arange(w.streams) % w.channels
    y_ref, _ = oracle.online_lcsm(h.astype(np.float64)[:, d_of, :], x0.reshape(-1).astype(np.float64),
                                  eps.reshape(w.length, w.streams).astype(np.float64))
    h_d = torch.from_numpy(h).cuda()
    x0_d = torch.from_numpy(x0).cuda()
    eps_d = torch.from_numpy(eps).cuda()
    for _ in range(2):
        y = torch.full((w.length, w.batch, w.channels), float("nan"), dtype=torch.float32, device="cuda")
        fi.generate_noalloc(h_d, w.batch, w.length, x0_d, eps_d, y, w.dtype)
        torch.cuda.synchronize()
        got = y.cpu().numpy().reshape(w.length, w.streams).T
        assert oracle.stream_error(got, y_ref[-1]) <= TOL["f32"]


@pytest.mark.gpu
def test_noalloc_allocates_nothing(fi):
    w = synth.Workload("noalloc-c", 2, 32, 512, 2, "f32", 1e-3, 1e-1)
    inp = gpu_inputs(w, 11)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    fi.generate_noalloc(inp["h"], w.batch, w.length, inp["x0"], inp["eps"], y, w.dtype)   # warm-up call
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    fi.generate_noalloc(inp["h"], w.batch, w.length, inp["x0"], inp["eps"], y, w.dtype)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


@pytest.mark.gpu
def test_noalloc_leaves_a_wider_live_context_working(fi):
    # A context whose on-chip window is wide (18 layers, 3456 streams) is created
    # first; a small fixed-memory call in between must not shrink what its chunk
    # kernel may use, and the context must still match the oracle afterwards.
    big = synth.Workload("noalloc-live", 18, 864, 256, 4, "f32", 1e-3, 1e-1)
    inp = gpu_inputs(big, 13)
    ctx = fi.Context(inp["h"], big.batch, big.dtype)
    small = synth.WORKLOADS["tiny-1x16-L1K"]
    sinp = gpu_inputs(small, 14)
    ys = torch.empty((small.length, small.batch, small.channels), dtype=torch.float32, device="cuda")
    fi.generate_noalloc(sinp["h"], small.batch, small.length, sinp["x0"], sinp["eps"], ys, small.dtype)
    y = torch.empty((big.length, big.batch, big.channels), dtype=torch.float32, device="cuda")
    rec = torch.empty((big.layers, big.length, big.batch, big.channels), dtype=torch.float32, device="cuda")
    ctx.generate(big.length, inp["x0"], inp["eps"], y, 0.1, rec)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, big.length)]
    ctx.close()
    h64 = oracle_filters(inp["h_np"], big.dtype)
    streams = [(0, 0), (1, 5), (3, 863), (2, 431)]
    r = teacher_forced_errors(h64, acts, rec.cpu().numpy(), streams, big.dtype)
    assert r["y"] <= TOL["f32"], r["y"]

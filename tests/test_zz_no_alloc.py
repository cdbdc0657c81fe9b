"""fi_generate_noalloc: the generation for callers that cannot allocate device memory.

Such callers (a thread with a hard latency budget, a framework that owns all
device memory, code running where allocation is not allowed) get their working
memory from one fixed device array inside the library. This file checks, through
the C-ABI, that two calls in a row give what the allocating path (fi_init +
fi_generate) gives, within the fp32 / bf16 tolerances the other parity tests use,
and that a configuration too large for the fixed array is refused cleanly.
It sorts last so that a run stopping at its first failure has run everything else.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import TOL, gpu_inputs

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

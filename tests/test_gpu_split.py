"""The multi-GPU partition, checked on one GPU: every (sequence, channel) stream
is independent under the elementwise block and sampler, so the path shards by
channels or by sequences with no collective. Two contexts that each hold half of
the channels (or half of the batch), run one after the other, must reproduce one
full context's outputs bit for bit, with the same plan forced on all of them.
The FFT blocks transform two sequences of a channel together when the batch is
even, so a batch split keeps each half's batch even (as a multi-GPU split must,
to stay bit-identical).
"""
import numpy as np
import pytest

import synth
from fi_testlib import gpu_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _generate(fi, h, x0, eps, batch, dtype, plan):
    ctx = fi.Context(h.contiguous(), batch, dtype, **plan)
    L, D = h.shape[2], h.shape[1]
    y = torch.empty((L, batch, D), dtype=torch.float32, device="cuda")
    rec = torch.empty((h.shape[0], L, batch, D), dtype=torch.float32, device="cuda")
    ctx.generate(L, x0.contiguous(), eps.contiguous(), y, 0.1, rec)
    ctx.sync()
    ctx.close()
    return y, rec


@pytest.mark.parametrize("M,D,L,B,dtype", [(4, 48, 4096, 4, "f32"), (3, 40, 2048, 4, "bf16")])
def test_channel_and_batch_split_is_exact(fi, M, D, L, B, dtype):
    w = synth.Workload(f"split-{M}x{D}x{L}x{B}{dtype}", M, D, L, B, dtype, 1e-3, 1e-1)
    inp = gpu_inputs(w, 21)
    plan = dict(chunk=64, fft_from=64, tc_max=-1)
    h, x0, eps = inp["h"], inp["x0"], inp["eps"]
    y, rec = _generate(fi, h, x0, eps, B, dtype, plan)
    # channels split in two
    half = D // 2
    ya, ra = _generate(fi, h[:, :half], x0[:, :half], eps[:, :, :half], B, dtype, plan)
    yb, rb = _generate(fi, h[:, half:], x0[:, half:], eps[:, :, half:], B, dtype, plan)
    assert torch.equal(torch.cat([ya, yb], dim=2), y)
    assert torch.equal(torch.cat([ra, rb], dim=3), rec)
    # sequences split in two
    hb = B // 2
    yc, rc = _generate(fi, h, x0[:hb], eps[:, :hb], hb, dtype, plan)
    yd, rd = _generate(fi, h, x0[hb:], eps[:, hb:], B - hb, dtype, plan)
    assert torch.equal(torch.cat([yc, yd], dim=1), y)
    assert torch.equal(torch.cat([rc, rd], dim=2), rec)
    assert np.isfinite(y.cpu().numpy()).all()

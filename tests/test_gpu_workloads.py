"""Parity at the workloads' full sizes, in the launch configuration the benchmark
times (automatic plan, one closed-loop generation of all L positions).

Full sizes are too large for the O(L^2) oracle on every output, so each test
checks sampled (sequence, channel) streams at sampled positions, every layer:
the library's recorded inputs a^{l-1} give the oracle's y^l at a position by its
O(t) defining sum; layer M is compared with the returned y, earlier layers
through their recorded blocks a^l = R(tanh(y^l)). Sampled positions include the
first ones, both sides of the largest block boundaries and the last.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import TOL, oracle_filters

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _positions(L, rng, k=24):
    fixed = {0, 1, 2, 3, 63, 64, 65, 127, 128, L // 4 - 1, L // 4, L // 2 - 1, L // 2, L // 2 + 1,
             3 * L // 4, L - 2, L - 1}
    extra = rng.integers(0, L, k)
    return sorted(p for p in fixed.union(int(e) for e in extra) if 0 <= p < L)


def _streams(w, rng, k=6):
    fixed = {(0, 0), (w.batch - 1, w.channels - 1)}
    extra = {(int(rng.integers(w.batch)), int(rng.integers(w.channels))) for _ in range(k)}
    return sorted(fixed | extra)


def _run_full(fi, w, seed):
    rng = np.random.default_rng(seed + 99)
    h = synth.filters(w, seed)
    x0 = synth.first_token(w, seed)
    eps = synth.noise(w, seed)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    ctx = fi.Context(torch.from_numpy(h).cuda().to(td), w.batch, w.dtype)
    x0_d = torch.from_numpy(x0).cuda().to(td)
    eps_d = torch.from_numpy(eps).cuda()
    del eps
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(w.length, x0_d, eps_d, y, 0.1)
    ctx.sync()
    del eps_d
    streams = _streams(w, rng)
    pos = _positions(w.length, rng)
    bi = torch.tensor([b for b, _ in streams], device="cuda")
    di = torch.tensor([d for _, d in streams], device="cuda")
    acts = []
    buf = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    for layer in range(w.layers):
        ctx.read_activations(layer, buf)
        acts.append(buf[:, bi, di].T.contiguous().cpu().numpy().astype(np.float64))   # [streams][L]
    y_s = y[:, bi, di].T.contiguous().cpu().numpy().astype(np.float64)
    ctx.close()
    del buf, y
    torch.cuda.empty_cache()
    h64 = oracle_filters(h, w.dtype)
    return h64, streams, pos, acts, y_s


def _check(w, h64, streams, pos, acts, y_s):
    R = oracle.bf16_round if w.dtype == "bf16" else (lambda v: v)
    tol = TOL[w.dtype]
    worst_y, worst_a = 0.0, 0.0
    for k, (b, d) in enumerate(streams):
        for l in range(w.layers):
            y_ref = oracle.causal_conv_at(h64[l, d], acts[l][k], pos)
            if l + 1 == w.layers:
                got = y_s[k][pos]
                worst_y = max(worst_y, np.max(np.abs(got - y_ref)) / max(np.max(np.abs(y_ref)), 1e-30))
            else:
                want = R(np.tanh(y_ref))
                got = acts[l + 1][k][pos]
                worst_a = max(worst_a, np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-30))
    assert worst_y <= tol, worst_y
    assert worst_a <= tol, worst_a
    return worst_y, worst_a


@pytest.mark.parametrize("name", ["hyena-8x768-L8K", "hyena-18x864-L32K-B4", "longrange-4x1024-L128K-bf16",
                                  "sweep-8x2048-L16K-bf16-B1", "sweep-8x2048-L16K-bf16-B8",
                                  "sweep-8x2048-L16K-bf16-B32", "sweep-8x2048-L16K-bf16-B64"])
def test_full_size_workload(fi, name):
    w = synth.WORKLOADS[name]
    h64, streams, pos, acts, y_s = _run_full(fi, w, seed=3)
    wy, wa = _check(w, h64, streams, pos, acts, y_s)
    print(f"{name}: last-layer error {wy:.2e}, block-rule error {wa:.2e} over {len(streams)} streams x {len(pos)} positions")

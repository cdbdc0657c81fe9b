"""Prompt prefill (fi_prefill) followed by generation, against the float64 oracle.

A prompt of p tokens is prefilled (every layer's outputs over the prompt by one
offline FFT convolution), then the rest of the sequence is generated closed loop
from a given next token. Checked: the prefill's outputs of every layer against
the oracle's prompt model (every stream, every prompt position); the recorded
activations (the prompt tokens exactly, the block rule elsewhere); the generated
part teacher-forced against the plain causal convolution of the recorded
activations over the whole sequence (so the prompt's contributions to later
positions, which reach them through the blocks that straddle the prompt's end,
are checked too); and that prefill leaves the state p calls of fi_step leave.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import TOL, gpu_inputs, oracle_filters, read_all_activations, teacher_forced_errors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _prompt(w, p, seed):
    r = np.random.default_rng(seed)
    x = r.standard_normal((p, w.batch, w.channels)).astype(np.float32)
    if w.dtype == "bf16":
        x = oracle.bf16_round(x.astype(np.float64)).astype(np.float32)
    return x


def _prefill_then_generate(fi, w, inp, p, x_np, plan):
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    ctx = fi.Context(inp["h"], w.batch, w.dtype, **plan)
    x = torch.from_numpy(x_np).cuda().to(td).contiguous()
    M, L = w.layers, w.length
    y_p = torch.empty((p, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rec_p = torch.empty((M, p, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.prefill(p, x, y_p, rec_p)
    assert ctx.position == p
    n = L - p
    rec_g = torch.empty((M, n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    y_g = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    if n > 0:
        ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y_g, 0.1, rec_g)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, L)]
    ctx.close()
    rec = torch.cat([rec_p, rec_g], dim=1).cpu().numpy()
    return y_p.cpu().numpy(), rec, acts, y_g.cpu().numpy()


CASES = [
    (synth.Workload("prefill-3x8-L4K", 3, 8, 4096, 2, "f32", 1e-3, 1e-1), dict(chunk=64, fft_from=64)),
    (synth.Workload("prefill-2x8-L2K-bf16", 2, 8, 2048, 1, "bf16", 1e-3, 1e-1), dict(chunk=32, fft_from=64)),
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("pfrac", ["1", "63", "64", "1000", "L/2"])
def test_prefill_then_generate(fi, case, pfrac):
    w, plan = CASES[case]
    p = w.length // 2 if pfrac == "L/2" else int(pfrac)
    inp = gpu_inputs(w, 50 + case)
    x_np = _prompt(w, p, 60 + p)
    y_p, rec, acts, y_g = _prefill_then_generate(fi, w, inp, p, x_np, plan)
    h64 = oracle_filters(inp["h_np"], w.dtype)
    tol = TOL[w.dtype]
    # prefill outputs, every layer, stream and prompt position, against the prompt model
    d_of = np.arange(w.streams) % w.channels
    y_ref, a_ref = oracle.prompt_lcsm(h64[:, d_of, :], x_np.reshape(p, -1).T.astype(np.float64), w.dtype == "bf16")
    got = rec[:, :p].reshape(w.layers, p, -1).transpose(0, 2, 1)
    assert oracle.stream_error(got, y_ref) <= tol
    assert np.array_equal(y_p.reshape(p, -1).T, got[-1].astype(np.float32))
    # the prompt tokens are stored exactly; the block rule holds on the prompt
    assert np.array_equal(acts[0][:p], x_np)
    # teacher-forced over the whole sequence (prompt and generated positions)
    streams = [(b, d) for b in range(w.batch) for d in range(w.channels)]
    r = teacher_forced_errors(h64, acts, rec, streams, w.dtype)
    assert r["y"] <= tol, r["y"]
    assert r["block"] <= (2e-2 if w.dtype == "bf16" else 1e-5), r["block"]


def test_prefill_state_equals_step_calls(fi):
    # After a prompt, fi_prefill and p calls of fi_step leave states that generate
    # the same continuation (within the fp32 tolerance over the first positions,
    # before the closed loops drift apart).
    w, plan = CASES[0]
    p = 1000
    inp = gpu_inputs(w, 70)
    x_np = _prompt(w, p, 71)
    x = torch.from_numpy(x_np).cuda()
    n = 256
    outs = []
    for use_prefill in (True, False):
        ctx = fi.Context(inp["h"], w.batch, w.dtype, **plan)
        if use_prefill:
            ctx.prefill(p, x)
        else:
            y_t = torch.empty((w.batch, w.channels), dtype=torch.float32, device="cuda")
            for t in range(p):
                ctx.step(x[t].contiguous(), y_t)
        y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
        ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y, 0.1)
        ctx.sync()
        outs.append(y.cpu().numpy())
        ctx.close()
    a, b = (o[:64].reshape(64, -1).T for o in outs)
    assert oracle.stream_error(a, b) <= TOL["f32"]


@pytest.mark.parametrize("name", ["hyena-18x864-L32K-B4"])
def test_prefill_full_size_half_prompt(fi, name):
    # The headline stack with a prompt of L/2 = 16384 positions (the largest
    # prefill transform), sampled streams and positions, every layer.
    w = synth.WORKLOADS[name]
    p = w.length // 2
    rng = np.random.default_rng(80)
    h = synth.filters(w, 81)
    x_np = _prompt(w, p, 82)
    ctx = fi.Context(torch.from_numpy(h).cuda(), w.batch, w.dtype)
    rec = torch.empty((w.layers, p, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.prefill(p, torch.from_numpy(x_np).cuda(), None, rec)
    ctx.sync()
    streams = sorted({(int(rng.integers(w.batch)), int(rng.integers(w.channels))) for _ in range(8)})
    pos = sorted({0, 1, 63, 64, 1023, 1024, p - 2, p - 1} | {int(v) for v in rng.integers(0, p, 24)})
    bi = torch.tensor([b for b, _ in streams], device="cuda")
    di = torch.tensor([d for _, d in streams], device="cuda")
    buf = torch.empty((p, w.batch, w.channels), dtype=torch.float32, device="cuda")
    acts = []
    for layer in range(w.layers):
        ctx.read_activations(layer, buf)
        acts.append(buf[:, bi, di].T.cpu().numpy().astype(np.float64))
    ys = rec[:, :, bi, di].permute(0, 2, 1).cpu().numpy().astype(np.float64)
    ctx.close()
    h64 = oracle_filters(h, w.dtype)
    worst = 0.0
    for k, (b, d) in enumerate(streams):
        assert np.array_equal(acts[0][k], x_np[:, b, d].astype(np.float64))
        for l in range(w.layers):
            y_ref = oracle.causal_conv_at(h64[l, d], acts[l][k], pos)
            worst = max(worst, oracle.stream_error(ys[l, k, pos], y_ref))
            if l + 1 < w.layers:
                assert np.max(np.abs(acts[l + 1][k][pos] - np.tanh(ys[l, k, pos]))) <= 1e-5
    assert worst <= TOL["f32"], worst

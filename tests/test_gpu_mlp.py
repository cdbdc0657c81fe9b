"""Channel-mixing block (MLP + GELU after every layer) against the float64 oracle.

Checked teacher-forced on every layer, stream and position: each recorded y^l
equals the causal convolution of the recorded a^{l-1}; each recorded a^l
equals R(block^l(y^l)) recomputed in float64 from the recorded y^l; the tokens
follow the sampler rule. With small (contractive) weights the closed loop is
also compared with the oracle's own closed loop over the whole sequence.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import TOL, gpu_inputs, oracle_filters, read_all_activations

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _weights(M, D, Dh, seed, scale=0.3):
    rng = np.random.default_rng(seed)
    w1 = (scale * rng.standard_normal((M, Dh, D)) / np.sqrt(D)).astype(np.float32)
    b1 = (0.1 * rng.standard_normal((M, Dh))).astype(np.float32)
    w2 = (scale * rng.standard_normal((M, D, Dh)) / np.sqrt(Dh)).astype(np.float32)
    b2 = (0.1 * rng.standard_normal((M, D))).astype(np.float32)
    return w1, b1, w2, b2


def _set(ctx, ws):
    ctx.set_mlp_block(*(torch.from_numpy(a).cuda() for a in ws))


def _check_teacher_forced(w, h64, ws, acts, rec, eps_np, eps_scale=0.1):
    R = oracle.bf16_round if w.dtype == "bf16" else (lambda v: v)
    w1, b1, w2, b2 = (a.astype(np.float64) for a in ws)
    M, n = w.layers, rec.shape[1]
    worst_y = 0.0
    for l in range(M):
        for b in range(w.batch):
            for d in range(w.channels):
                y_ref = oracle.causal_conv(h64[l, d, :n], acts[l][:n, b, d].astype(np.float64))
                worst_y = max(worst_y, oracle.stream_error(rec[l, :, b, d].astype(np.float64), y_ref))
    assert worst_y <= TOL[w.dtype], worst_y
    rel = 2e-2 if w.dtype == "bf16" else 1e-5
    for l in range(M):
        out = oracle.mlp_block(rec[l].astype(np.float64), w1[l], b1[l], w2[l], b2[l])   # [n][B][D]
        if l + 1 < M:
            got, want = acts[l + 1][:n].astype(np.float64), R(out)
        else:
            got = acts[0][1:n].astype(np.float64)
            want = R(out[: n - 1] + eps_scale * eps_np[: n - 1].astype(np.float64))
        assert np.max(np.abs(got - want)) <= rel * max(1.0, np.max(np.abs(want))), l
    return worst_y


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_generate_with_mlp_block_teacher_forced(fi, dtype):
    # fast-decaying filters and small block weights keep the loop bounded (the
    # MLP block, unlike tanh, does not clip)
    w = synth.Workload(f"mlp-3x16-L256-{dtype}", 3, 16, 256, 2, dtype, 1e-1, 5e-1)
    inp = gpu_inputs(w, 31)
    ws = _weights(w.layers, w.channels, 24, 32)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    _set(ctx, ws)
    n = w.length
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rec = torch.empty((w.layers, n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y, 0.1, rec)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, n)]
    ctx.close()
    rec = rec.cpu().numpy()
    assert np.array_equal(y.cpu().numpy(), rec[-1])
    _check_teacher_forced(w, oracle_filters(inp["h_np"], dtype), ws, acts, rec, inp["eps_np"])


def test_closed_loop_matches_oracle_with_contractive_block(fi):
    # Small block weights and decaying filters keep the loop contractive, so the
    # device's closed loop stays on the oracle's over the whole sequence.
    w = synth.Workload("mlp-2x8-L128", 2, 8, 128, 2, "f32", 2e-1, 5e-1)
    inp = gpu_inputs(w, 41)
    h = inp["h_np"].astype(np.float64) * 0.1
    ws = _weights(w.layers, w.channels, 12, 42, scale=0.2)
    ctx = fi.Context(torch.from_numpy(h.astype(np.float32)).cuda(), w.batch, w.dtype)
    _set(ctx, ws)
    n = w.length
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y, 0.1)
    ctx.sync()
    ctx.close()
    h32 = h.astype(np.float32).astype(np.float64)
    y_ref, _ = oracle.online_lcsm_mlp(h32, *(a.astype(np.float64) for a in ws), inp["x0_np"].astype(np.float64),
                                      inp["eps_np"][:n].astype(np.float64), 0.1)
    got = y.cpu().numpy().transpose(1, 2, 0)   # [B][D][n]
    err = max(oracle.stream_error(got[b, d], y_ref[-1, b, d]) for b in range(w.batch) for d in range(w.channels))
    assert err <= TOL["f32"], err


def test_step_api_with_mlp_block(fi):
    # fi_step on given tokens, then fi_generate continues: teacher-forced over the whole sequence.
    w = synth.Workload("mlp-2x8-L128-step", 2, 8, 128, 3, "f32", 1e-1, 5e-1)
    inp = gpu_inputs(w, 51)
    ws = _weights(w.layers, w.channels, 16, 52)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    _set(ctx, ws)
    toks = torch.from_numpy(synth.token_stream(w, 51)).cuda()
    n_step = 45
    ys = torch.empty((n_step, w.batch, w.channels), dtype=torch.float32, device="cuda")
    for t in range(n_step):
        ctx.step(toks[t].contiguous(), ys[t])
    n_gen = w.length - n_step
    yg = torch.empty((n_gen, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n_gen, toks[n_step].contiguous(), inp["eps"][:n_gen].contiguous(), yg, 0.1)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, w.length)]
    ctx.close()
    h64 = oracle_filters(inp["h_np"], "f32")
    y_all = np.concatenate([ys.cpu().numpy(), yg.cpu().numpy()])
    w1, b1, w2, b2 = (a.astype(np.float64) for a in ws)
    for b in range(w.batch):
        for d in range(w.channels):
            ref = oracle.causal_conv(h64[-1, d], acts[-1][:, b, d].astype(np.float64))
            assert oracle.stream_error(y_all[:, b, d], ref) <= TOL["f32"]
    # the block rule between the recorded layers (y^1 from its own convolution)
    y1 = np.stack([[oracle.causal_conv(h64[0, d], acts[0][:, b, d].astype(np.float64)) for d in range(w.channels)]
                   for b in range(w.batch)]).transpose(2, 0, 1)   # [n][B][D]
    want = oracle.mlp_block(y1, w1[0], b1[0], w2[0], b2[0])
    assert np.max(np.abs(acts[1].astype(np.float64) - want)) <= 1e-5 * max(1.0, np.max(np.abs(want)))
    # the generated tokens follow the sampler rule from the last layer's outputs
    out = oracle.mlp_block(y_all[n_step:-1].astype(np.float64), w1[-1], b1[-1], w2[-1], b2[-1])
    want_x = out + 0.1 * inp["eps_np"][: n_gen - 1].astype(np.float64)
    assert np.max(np.abs(acts[0][n_step + 1:].astype(np.float64) - want_x)) <= 1e-5 * max(1.0, np.max(np.abs(want_x)))


def test_mlp_block_state_rules(fi):
    w = synth.Workload("mlp-1x4-L64", 1, 4, 64, 1, "f32", 1e-3, 1e-1)
    inp = gpu_inputs(w, 61)
    ws = _weights(1, 4, 8, 62)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    y = torch.empty((8, 1, 4), dtype=torch.float32, device="cuda")
    ctx.generate(8, inp["x0"], inp["eps"][:8].contiguous(), y, 0.1)
    with pytest.raises(fi.FiError):
        _set(ctx, ws)                        # only at position 0
    ctx.reset()
    _set(ctx, ws)
    with pytest.raises(fi.FiError):
        ctx.prefill(4, torch.zeros((4, 1, 4), device="cuda"))
    with pytest.raises(fi.FiError):
        ctx.generate_lazy(8, inp["x0"], inp["eps"][:8].contiguous(), y, 0.1)
    # back to the elementwise block: the same outputs as a context that never had the MLP
    ctx.set_mlp_block()
    ctx.generate(8, inp["x0"], inp["eps"][:8].contiguous(), y, 0.1)
    ref = fi.Context(inp["h"], w.batch, w.dtype)
    y2 = torch.empty_like(y)
    ref.generate(8, inp["x0"], inp["eps"][:8].contiguous(), y2, 0.1)
    ctx.sync()
    ref.sync()
    assert torch.equal(y, y2)
    ctx.close()
    ref.close()


@pytest.mark.parametrize("M,D,Dh,B,dtype", [
    (1, 8, 10, 3, "f32"),      # one layer: the small-block launch records y^M itself
    (2, 12, 16, 9, "bf16"),    # two CTA groups (8 + 1) in a bf16 context
    (3, 8, 10, 2, "f32"),      # W1 rows float4 (D = 8), W2 rows scalar (Dh = 10)
])
def test_mlp_block_shapes_teacher_forced(fi, M, D, Dh, B, dtype):
    w = synth.Workload(f"mlp-{M}x{D}-L256-B{B}-{dtype}", M, D, 256, B, dtype, 1e-1, 5e-1)
    inp = gpu_inputs(w, 100 + M + D)
    ws = _weights(M, D, Dh, 200 + Dh)
    ctx = fi.Context(inp["h"], B, dtype)
    _set(ctx, ws)
    n = 200                                   # a ragged stop inside the sequence
    y = torch.empty((n, B, D), dtype=torch.float32, device="cuda")
    rec = torch.empty((M, n, B, D), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y, 0.1, rec)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, n)]
    ctx.close()
    rec = rec.cpu().numpy()
    assert np.array_equal(y.cpu().numpy(), rec[-1])
    _check_teacher_forced(w, oracle_filters(inp["h_np"], dtype), ws, acts, rec, inp["eps_np"])


def test_mlp_block_groups_and_scalar_rows(fi):
    # B = 10 sequences: two CTA groups (8 + 2); D = 6 and Dh = 10 are not
    # multiples of 4, so both products take the scalar row path.
    w = synth.Workload("mlp-2x6-L128-B10", 2, 6, 128, 10, "f32", 1e-1, 5e-1)
    inp = gpu_inputs(w, 71)
    ws = _weights(w.layers, w.channels, 10, 72)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    _set(ctx, ws)
    n = 96                                   # a ragged stop inside the sequence
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rec = torch.empty((w.layers, n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], inp["eps"][:n].contiguous(), y, 0.1, rec)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, n)]
    ctx.close()
    rec = rec.cpu().numpy()
    assert np.array_equal(y.cpu().numpy(), rec[-1])
    _check_teacher_forced(w, oracle_filters(inp["h_np"], "f32"), ws, acts, rec, inp["eps_np"])


def test_captured_positions_equal_direct_launches(fi):
    # fi_generate replays the captured layers (position read on the device);
    # fi_step launches them directly. Fed the tokens fi_generate produced,
    # fi_step must give the same outputs bit for bit. The generation runs in
    # two calls, so the second call's record (new base, buffers) is used too.
    w = synth.Workload("mlp-3x12-L256", 3, 12, 256, 3, "f32", 1e-1, 5e-1)
    inp = gpu_inputs(w, 81)
    ws = _weights(w.layers, w.channels, 20, 82)
    gen = fi.Context(inp["h"], w.batch, w.dtype)
    _set(gen, ws)
    n1, n = 57, 160
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    eps = inp["eps"][:n].contiguous()
    gen.generate(n1, inp["x0"], eps[:n1].contiguous(), y[:n1], 0.1)
    y2 = torch.empty((n - n1, w.batch, w.channels), dtype=torch.float32, device="cuda")
    gen.generate(n - n1, None, eps[n1:].contiguous(), y2, 0.1)
    gen.sync()
    toks = read_all_activations(gen, n)[0]     # [n][B][D] tokens x_t
    gen.close()
    step = fi.Context(inp["h"], w.batch, w.dtype)
    _set(step, ws)
    ys = torch.empty_like(y)
    for t in range(n):
        step.step(toks[t].contiguous().cuda(), ys[t])
    step.sync()
    step.close()
    assert torch.equal(torch.cat([y[:n1], y2]), ys)


def test_second_context_does_not_lower_the_shared_memory_cap(fi):
    # The block's kernels take min(B, 8) x D floats of shared memory (128 KB at
    # D = 4096). A second context that needs less (64 KB at D = 2048) must not
    # lower the per-kernel cap under the first, whose next positions still run
    # and repeat its first generation bit for bit.
    def make(D, seed):
        w = synth.Workload(f"mlp-1x{D}-L64-B8", 1, D, 64, 8, "f32", 1e-1, 5e-1)
        inp = gpu_inputs(w, seed)
        ctx = fi.Context(inp["h"], 8, "f32")
        _set(ctx, _weights(1, D, 256, seed + 1, scale=0.2))
        return w, inp, ctx

    w1, inp1, big = make(4096, 111)
    n = 16
    y = torch.empty((n, 8, 4096), dtype=torch.float32, device="cuda")
    big.generate(n, inp1["x0"], inp1["eps"][:n].contiguous(), y, 0.1)
    big.sync()
    _, _, small = make(2048, 121)
    big.reset()
    y2 = torch.empty_like(y)
    big.generate(n, inp1["x0"], inp1["eps"][:n].contiguous(), y2, 0.1)
    big.sync()
    assert torch.equal(y, y2)
    small.close()
    big.close()

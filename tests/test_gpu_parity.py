"""GPU parity of the library against the float64 oracle, through the C-ABI.

Small and medium cases compare every position of every stream; the tolerances
are the ones stated for the method's hot path: stream-normwise relative error
1e-4 for fp32 and 2e-2 for bf16-input / fp32-accumulate.
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import (TOL, gpu_inputs, oracle_filters, read_all_activations, sampler_error,
                        teacher_forced_errors)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _workload(M, D, L, B, dtype="f32", lam=(1e-3, 1e-1)):
    return synth.Workload(f"t{M}x{D}x{L}x{B}{dtype}", M, D, L, B, dtype, *lam)


def _run_generate(fi, w, seed=0, n=None, chunk=0, fft_from=0, split=None):
    """Generate n positions (optionally as several calls, `split` = call lengths)."""
    n = w.length if n is None else n
    inp = gpu_inputs(w, seed, n)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, chunk=chunk, fft_from=fft_from)
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rec = torch.empty((w.layers, n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    parts = split or [n]
    p = 0
    for k, m in enumerate(parts):
        if k == 0:
            x0 = inp["x0"]
        else:
            # continuing call: its first token is the one the sampler produced
            x0_f = torch.tanh(y[p - 1].double()) + 0.1 * inp["eps"][p - 1].double()
            x0 = x0_f.to(inp["x0"].dtype)
        yk = torch.empty((m, w.batch, w.channels), dtype=torch.float32, device="cuda")
        rk = torch.empty((w.layers, m, w.batch, w.channels), dtype=torch.float32, device="cuda")
        ctx.generate(m, x0, inp["eps"][p:p + m].contiguous(), yk, 0.1, rk)
        y[p:p + m] = yk
        rec[:, p:p + m] = rk
        p += m
    torch.cuda.synchronize()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, n)]
    return ctx, inp, y.cpu().numpy(), rec.cpu().numpy(), acts


def _check_teacher_forced(w, inp, rec, acts, streams=None, positions=None):
    h64 = oracle_filters(inp["h_np"], w.dtype)
    if streams is None:
        streams = [(b, d) for b in range(w.batch) for d in range(w.channels)]
    r = teacher_forced_errors(h64, acts, rec, streams, w.dtype, positions)
    tol = TOL[w.dtype]
    assert r["y"] <= tol, r["y"]
    assert r["block"] <= (2e-2 if w.dtype == "bf16" else 1e-6), r["block"]
    return r


# --------------------------------------------------------------------------- FFT
@pytest.mark.parametrize("log2n", list(range(6, 15)))
def test_device_fft_matches_dft(fi, log2n):
    N = 1 << log2n
    count = 3
    r = np.random.default_rng(log2n)
    x = (r.standard_normal((count, N)) + 1j * r.standard_normal((count, N))).astype(np.complex64)
    xt = torch.from_numpy(x).cuda()
    for inverse in (False, True):
        out = torch.empty_like(xt)
        fi.debug_fft(log2n, xt, out, inverse)
        got = out.cpu().numpy().astype(np.complex128)
        ref = oracle.dft(x.astype(np.complex128), inverse=inverse)
        err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
        assert err < 2e-6, (N, inverse, err)


# --------------------------------------------------------------------------- small exhaustive cases
def test_tiny_workload_closed_loop_and_teacher_forced(fi):
    w = synth.WORKLOADS["tiny-1x16-L1K"]
    ctx, inp, y, rec, acts = _run_generate(fi, w)
    _check_teacher_forced(w, inp, rec, acts)
    # closed loop: the oracle generates its own trajectory from the same x0 and noise
    h64 = oracle_filters(inp["h_np"], w.dtype)
    S = w.streams
    d_of = np.arange(S) % w.channels
    y_ref, _ = oracle.online_lcsm(h64[:, d_of, :], inp["x0_np"].reshape(-1), inp["eps_np"].reshape(w.length, S))
    y_gpu = rec.reshape(w.layers, w.length, S).transpose(0, 2, 1)
    assert oracle.stream_error(y_gpu, y_ref) <= TOL["f32"]
    assert sampler_error(acts[0], rec[-1], inp["eps_np"], w.dtype) < 1e-6


@pytest.mark.parametrize("M,D,L,B,chunk,fft_from", [
    (3, 5, 256, 3, 8, 64),      # FFT blocks 64, 128 and direct blocks from HBM 8..32
    (2, 7, 512, 2, 32, 128),    # default-like plan
    (4, 3, 128, 1, 2, 64),      # tiny chunk: almost everything from HBM
    (2, 4, 1024, 2, 64, 64),    # largest chunk
    (1, 33, 256, 1, 16, 1 << 20),  # direct-only (FFT disabled)
])
def test_generate_exhaustive(fi, M, D, L, B, chunk, fft_from):
    w = _workload(M, D, L, B)
    ctx, inp, y, rec, acts = _run_generate(fi, w, seed=M * 100 + D, chunk=chunk, fft_from=fft_from)
    _check_teacher_forced(w, inp, rec, acts)
    assert np.array_equal(y, rec[-1])
    assert sampler_error(acts[0], rec[-1], inp["eps_np"], w.dtype) < 1e-6


@pytest.mark.parametrize("L", [2, 4, 8, 16, 32])
def test_short_sequences(fi, L):
    w = _workload(2, 3, L, 2)
    ctx, inp, y, rec, acts = _run_generate(fi, w, seed=L)
    _check_teacher_forced(w, inp, rec, acts)


def test_ragged_calls_continue_exactly(fi):
    # Calls that stop inside a chunk, then continue: same state as one call.
    w = _workload(3, 6, 512, 2)
    ctx, inp, y, rec, acts = _run_generate(fi, w, seed=5, chunk=32, fft_from=64,
                                           split=[1, 36, 100, 3, 116, 256])
    assert ctx.position == 512
    _check_teacher_forced(w, inp, rec, acts)


def test_step_api_teacher_forced(fi):
    # fi_step with caller-provided tokens (open loop), then generate continues.
    w = _workload(3, 4, 256, 2)
    inp = gpu_inputs(w, 11)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, chunk=16, fft_from=64)
    toks = synth.token_stream(w, 11)
    n_step = 77
    ys = torch.empty((n_step, w.batch, w.channels), dtype=torch.float32, device="cuda")
    tt = torch.from_numpy(toks).cuda()
    for t in range(n_step):
        ctx.step(tt[t].contiguous(), ys[t])
    n_gen = w.length - n_step
    yg = torch.empty((n_gen, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rg = torch.empty((w.layers, n_gen, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n_gen, tt[n_step].contiguous(), inp["eps"][:n_gen].contiguous(), yg, 0.1, rg)
    torch.cuda.synchronize()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, w.length)]
    assert np.array_equal(acts[0][:n_step + 1], toks[:n_step + 1])
    h64 = oracle_filters(inp["h_np"], w.dtype)
    # layer M against the returned outputs, earlier layers through their recorded blocks
    y_all = np.concatenate([ys.cpu().numpy(), yg.cpu().numpy()])
    for (b, d) in [(b, d) for b in range(w.batch) for d in range(w.channels)]:
        ref = oracle.causal_conv(h64[-1, d], acts[-1][:, b, d])
        assert oracle.stream_error(y_all[:, b, d], ref) <= TOL["f32"]
        for l in range(1, w.layers):
            yl = oracle.causal_conv(h64[l - 1, d], acts[l - 1][:, b, d])
            assert np.max(np.abs(acts[l][:, b, d] - np.tanh(yl))) <= 1e-4 * max(1.0, np.max(np.abs(yl)))
    # after generate, stepping past the end is refused
    with pytest.raises(fi.FiError):
        ctx.step(tt[0].contiguous(), ys[0])


@pytest.mark.parametrize("M,D,L,B,dtype", [(1, 8, 256, 1, "f32"), (3, 6, 1024, 2, "f32"), (18, 4, 512, 3, "f32"),
                                           (2, 8, 512, 2, "bf16"), (33, 2, 128, 1, "f32")])
def test_step_api_every_position(fi, M, D, L, B, dtype):
    # fi_step for every position on given tokens: the red cells with the small
    # direct blocks fused into the same launch (M <= 32; M = 33 takes the
    # one-thread-per-stream kernel and separate block launches), every layer
    # checked against the oracle's causal convolution of the recorded inputs.
    w = synth.Workload(f"step-{M}x{D}-L{L}", M, D, L, B, dtype, 1e-3, 1e-1)
    inp = gpu_inputs(w, 21)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    toks = synth.token_stream(w, 21)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    tt = torch.from_numpy(toks).cuda().to(td)
    ys = torch.empty((L, B, D), dtype=torch.float32, device="cuda")
    for t in range(L):
        ctx.step(tt[t].contiguous(), ys[t])
    torch.cuda.synchronize()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, L)]
    ctx.close()
    h64 = oracle_filters(inp["h_np"], dtype)
    R = oracle.bf16_round if dtype == "bf16" else (lambda v: v)
    tol = TOL[dtype]
    y_np = ys.cpu().numpy()
    for b in range(B):
        for d in range(D):
            for l in range(M):
                yl = oracle.causal_conv(h64[l, d], acts[l][:, b, d].astype(np.float64))
                if l + 1 < M:
                    want = R(np.tanh(yl))
                    assert np.max(np.abs(acts[l + 1][:, b, d] - want)) <= (2e-2 if dtype == "bf16" else 1e-5)
                else:
                    assert oracle.stream_error(y_np[:, b, d], yl) <= tol


def test_bf16_small(fi):
    w = _workload(3, 8, 512, 2, dtype="bf16", lam=(1e-5, 1e-3))
    ctx, inp, y, rec, acts = _run_generate(fi, w, seed=3, chunk=16, fft_from=64)
    for a in acts:
        assert np.all(a.view(np.uint32) & 0xFFFF == 0)          # activations are bf16 values
    _check_teacher_forced(w, inp, rec, acts)
    assert sampler_error(acts[0], rec[-1], inp["eps_np"], w.dtype) <= 2e-2


def test_lazy_method_matches_oracle(fi):
    w = _workload(2, 6, 256, 2)
    inp = gpu_inputs(w, 21)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate_lazy(w.length, inp["x0"], inp["eps"], y, 0.1)
    torch.cuda.synchronize()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, w.length)]
    h64 = oracle_filters(inp["h_np"], w.dtype)
    for b in range(w.batch):
        for d in range(w.channels):
            ref = oracle.causal_conv(h64[-1, d], acts[-1][:, b, d])
            assert oracle.stream_error(y.cpu().numpy()[:, b, d], ref) <= TOL["f32"]
    # relaxed calls are refused until reset; after reset the relaxed run matches the lazy one
    with pytest.raises(fi.FiError):
        ctx.generate(1, inp["x0"], inp["eps"], y, 0.1)
    ctx.reset()
    y2 = torch.empty_like(y)
    ctx.generate(w.length, inp["x0"], inp["eps"], y2, 0.1)
    torch.cuda.synchronize()
    # the same closed loop through two summation orders: agree until chaos separates them
    e = np.abs(y2.cpu().numpy() - y.cpu().numpy())[:64]
    assert np.max(e) <= 1e-4 * np.max(np.abs(y.cpu().numpy()[:64]))


def test_generate_host_matches_device(fi):
    w = _workload(2, 8, 256, 2)
    inp = gpu_inputs(w, 4)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1)
    ctx.reset()
    yh = np.empty((w.length, w.batch, w.channels), dtype=np.float32)
    ctx.generate_host(w.length, inp["x0_np"], inp["eps_np"], yh, 0.1)
    assert np.array_equal(yh, y.cpu().numpy())


def test_generate_host_in_segments_matches_device(fi):
    # 20000 positions: 16 segments of 1280 (the last one 800), copies on their
    # own streams from pinned buffers; the outputs equal one device call's.
    # (Segments are at least 256 positions: a call of 4096 or fewer is one.)
    w = _workload(2, 4, 32768, 2)
    inp = gpu_inputs(w, 6)
    n = 20000
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    eps = inp["eps"][:n].contiguous()
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], eps, y, 0.1)
    ctx.reset()
    x0_h = inp["x0"].cpu().pin_memory()
    eps_h = eps.cpu().pin_memory()
    y_h = torch.empty((n, w.batch, w.channels), dtype=torch.float32).pin_memory()
    ctx.generate_host_ptr(n, x0_h.data_ptr(), eps_h.data_ptr(), y_h.data_ptr(), 0.1)
    assert torch.equal(y_h, y.cpu())
    ctx.close()


def test_reset_replays_identically(fi):
    w = _workload(2, 5, 512, 1)
    inp = gpu_inputs(w, 8)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, chunk=32, fft_from=64)
    y1 = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    ctx.generate(w.length, inp["x0"], inp["eps"], y1, 0.1)
    ctx.reset()
    ctx.generate(w.length, inp["x0"], inp["eps"], y2, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_state_errors(fi):
    w = _workload(1, 2, 16, 1)
    inp = gpu_inputs(w, 0)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    y = torch.empty((32, 1, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(fi.FiError) as e:
        ctx.generate(17, inp["x0"], torch.zeros((17, 1, 2), device="cuda"), y)
    assert e.value.status == fi.FI_E_STATE
    with pytest.raises(fi.FiError) as e:
        ctx.read_activations(1, y)
    assert e.value.status == fi.FI_E_INVALID
    ctx.generate(0, inp["x0"], inp["eps"], y)   # n = 0 is a no-op
    assert ctx.position == 0


def test_bounded_wait_reports_timeout(fi):
    # With a wait limit of 0 every device-side wait that is not already satisfied
    # gives up at once: the kernels finish, and fi_sync reports FI_E_TIMEOUT.
    w = _workload(3, 8, 256, 2)
    inp = gpu_inputs(w, 2)
    ctx = fi.Context(inp["h"], w.batch, w.dtype)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.set_wait_limit(0)
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1)
    with pytest.raises(fi.FiError) as e:
        ctx.sync()
    assert e.value.status == fi.FI_E_TIMEOUT
    # the flag was cleared; with the default limit the context works again
    ctx.set_wait_limit(-1)
    ctx.reset()
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1)
    ctx.sync()
    assert torch.isfinite(y).all()

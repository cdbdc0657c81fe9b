"""Blocks on the tensor cores (tcgen05 Toeplitz products) against the float64 oracle.

Each case forces block sides 64..tc_max onto the tensor cores and checks, for
every position of every stream, the teacher-forced outputs (the recorded inputs
of each layer convolved by the oracle) and the block rule. bf16 contexts hold
bf16-exact filters and activations, so their tensor-core products are exact and
only fp32 accumulation order separates them from the oracle: they are held to
1e-5 rather than the bf16 tolerance. fp32 contexts use three bf16 products of
split operands (relative error per product below 2^-16) and are held to the
fp32 tolerance. Batches cover the plan's shapes: 64-row tiles with several
target tiles per product (B < 16, including odd B and B = 1), 128-row tiles
(B a multiple of 16), and wide products (B = 64).
"""
import numpy as np
import pytest

import oracle
import synth
from fi_testlib import TOL, gpu_inputs, oracle_filters, read_all_activations, sampler_error, teacher_forced_errors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_convolution_sequence_online_b200 import fi as _fi
    return _fi


def _run(fi, w, seed, tc_max, fft_from=0, chunk=0):
    inp = gpu_inputs(w, seed)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, chunk=chunk, fft_from=fft_from, tc_max=tc_max)
    n = w.length
    y = torch.empty((n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    rec = torch.empty((w.layers, n, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(n, inp["x0"], inp["eps"], y, 0.1, rec)
    torch.cuda.synchronize()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, n)]
    plan = ctx.plan()
    ctx.close()
    return inp, rec.cpu().numpy(), acts, plan


@pytest.mark.parametrize("M,D,L,B,dtype,tc_max", [
    (3, 4, 2048, 8, "bf16", 512),     # 64-row tiles, two target tiles per product from side 128
    (2, 3, 1024, 16, "bf16", 512),    # 128-row tiles from side 128
    (2, 2, 1024, 64, "bf16", 256),    # wide products (N = 64)
    (2, 5, 1024, 4, "f32", 512),      # split products, four target tiles per product
    (3, 3, 1024, 3, "f32", 512),      # odd batch: padded operand rows
    (2, 6, 1024, 1, "f32", 256),      # one sequence: up to four target tiles per product
])
def test_tensor_core_blocks_teacher_forced(fi, M, D, L, B, dtype, tc_max):
    lam = (1e-5, 1e-3) if dtype == "bf16" else (1e-3, 1e-1)
    w = synth.Workload(f"tc{M}x{D}x{L}x{B}{dtype}", M, D, L, B, dtype, *lam)
    inp, rec, acts, plan = _run(fi, w, seed=7 * M + B, tc_max=tc_max)
    assert plan[2] == min(tc_max, L // 2)
    h64 = oracle_filters(inp["h_np"], w.dtype)
    streams = [(b, d) for b in range(B) for d in range(D)]
    r = teacher_forced_errors(h64, acts, rec, streams, w.dtype)
    tol = 1e-5 if dtype == "bf16" else TOL["f32"]
    assert r["y"] <= tol, r["y"]
    assert r["block"] <= (2e-2 if dtype == "bf16" else 1e-6), r["block"]
    assert sampler_error(acts[0], rec[-1], inp["eps_np"], w.dtype) <= (1e-2 if dtype == "bf16" else 1e-6)


def test_tensor_core_blocks_above_fft_range(fi):
    # tensor cores up to 128, FFT from 256 up, direct nowhere
    w = synth.Workload("tc-mixed", 2, 4, 2048, 8, "bf16", 1e-5, 1e-3)
    inp, rec, acts, plan = _run(fi, w, seed=3, tc_max=128, fft_from=256)
    assert plan[1:] == (256, 128)
    h64 = oracle_filters(inp["h_np"], w.dtype)
    r = teacher_forced_errors(h64, acts, rec, [(b, d) for b in range(8) for d in range(4)], w.dtype)
    assert r["y"] <= 1e-5, r["y"]


def test_tensor_core_bounded_waits_report_timeout(fi):
    # With a wait limit of 0 the tensor-core kernel's pipeline waits give up at
    # once: the MMA warp issues nothing, every role leaves its loop, the
    # accumulator columns are released and fi_sync reports FI_E_TIMEOUT. With
    # the default limit the same context then generates correctly.
    w = synth.Workload("tc-timeout", 2, 4, 1024, 8, "bf16", 1e-5, 1e-3)
    inp = gpu_inputs(w, 5)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, tc_max=256)
    y = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.set_wait_limit(0)
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1)
    with pytest.raises(fi.FiError) as e:
        ctx.sync()
    assert e.value.status == fi.FI_E_TIMEOUT
    ctx.set_wait_limit(-1)
    ctx.reset()
    rec = torch.empty((w.layers, w.length, w.batch, w.channels), dtype=torch.float32, device="cuda")
    ctx.generate(w.length, inp["x0"], inp["eps"], y, 0.1, rec)
    ctx.sync()
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, w.length)]
    h64 = oracle_filters(inp["h_np"], w.dtype)
    r = teacher_forced_errors(h64, acts, rec.cpu().numpy(), [(b, d) for b in range(8) for d in range(4)], w.dtype)
    assert r["y"] <= 1e-5, r["y"]


def test_tensor_core_blocks_with_steps_and_ragged_calls(fi):
    # fi_step (one position per call, blocks launched per position) for the
    # first 70 positions, then generation in calls that stop inside chunks: the
    # tensor-core blocks of sides 64..256 run from both paths on one state.
    w = synth.Workload("tc-mixed-calls", 2, 4, 1024, 8, "bf16", 1e-5, 1e-3)
    inp = gpu_inputs(w, 9)
    ctx = fi.Context(inp["h"], w.batch, w.dtype, tc_max=256)
    toks = synth.token_stream(w, 9)
    n_step = 70
    ys = torch.empty((n_step, w.batch, w.channels), dtype=torch.float32, device="cuda")
    tt = torch.from_numpy(toks).cuda().to(torch.bfloat16)
    for t in range(n_step):
        ctx.step(tt[t].contiguous(), ys[t])
    rest = w.length - n_step
    y = torch.empty((rest, w.batch, w.channels), dtype=torch.float32, device="cuda")
    p = 0
    x0 = tt[n_step].contiguous()
    for m in (58, 1, 200, 3, rest - 262):
        yk = torch.empty((m, w.batch, w.channels), dtype=torch.float32, device="cuda")
        ctx.generate(m, x0, inp["eps"][n_step + p:n_step + p + m].contiguous(), yk, 0.1)
        y[p:p + m] = yk
        p += m
        x0 = (torch.tanh(yk[-1].double()) + 0.1 * inp["eps"][n_step + p - 1].double()).to(torch.bfloat16)
    ctx.sync()
    assert ctx.position == w.length
    acts = [a.cpu().numpy() for a in read_all_activations(ctx, w.length)]
    h64 = oracle_filters(inp["h_np"], w.dtype)
    # last layer's outputs: the steps' y and the generated y, against the oracle
    # convolution of the recorded last-layer inputs
    y_all = np.concatenate([ys.cpu().numpy(), y.cpu().numpy()])
    worst = 0.0
    for b in range(w.batch):
        for d in range(w.channels):
            ref = oracle.causal_conv(h64[-1, d], acts[-1][:, b, d].astype(np.float64))
            worst = max(worst, oracle.stream_error(y_all[:, b, d], ref))
    assert worst <= 1e-5, worst

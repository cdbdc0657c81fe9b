"""Pins for the float64 oracle: each check compares it with something other than itself.

Sources of truth used here: numpy/scipy library routines (np.convolve, numpy.fft,
scipy.signal.fftconvolve, torch's bfloat16 conversion), closed forms (delta and
all-ones filters, the geometric filter's recurrence, the recurrent view of an
SSM-shaped filter), invariants (linearity, online equals offline), brute force on
tiny inputs and the schedule facts the Flash Inference summary page prints
(tests/golden/schedule_facts.json).
"""
import json
import os

import numpy as np
import pytest
import scipy.signal

import oracle
from oracle import (bf16_round, causal_conv, causal_conv_at, dft, lowbit, online_lcsm,
                    relaxed_online, relaxed_tiles, stream_error, tau)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "schedule_facts.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- causal_conv
@pytest.mark.parametrize("L", [1, 2, 7, 64, 333])
def test_causal_conv_matches_numpy_convolve(L):
    r = _rng(L)
    h, a = r.standard_normal(L), r.standard_normal(L)
    ref = np.convolve(h, a)[:L]
    assert np.allclose(causal_conv(h, a), ref, rtol=1e-12, atol=1e-12)


def test_causal_conv_matches_fft_convolution_batched():
    r = _rng(1)
    h, a = r.standard_normal((3, 5, 200)), r.standard_normal((3, 5, 200))
    ref = scipy.signal.fftconvolve(h, a, axes=-1)[..., :200]
    assert np.allclose(causal_conv(h, a), ref, rtol=1e-10, atol=1e-10)


def test_delta_input_returns_filter():
    r = _rng(2)
    h = r.standard_normal((4, 128))
    x = np.zeros(128)
    x[0] = 1.0
    assert np.array_equal(causal_conv(h, x), h)


def test_all_ones_filter_gives_prefix_sums():
    r = _rng(3)
    a = r.standard_normal((6, 300))
    assert np.allclose(causal_conv(np.ones(300), a), np.cumsum(a, axis=-1), rtol=1e-12, atol=1e-11)


@pytest.mark.parametrize("rate", [0.5, 0.97, -0.8])
def test_geometric_filter_recurrence(rate):
    # h_t = c r^t  =>  y_t = r y_{t-1} + c x_t  (the recurrent view of a 1-state filter)
    r_ = _rng(4)
    L, c = 400, 1.7
    x = r_.standard_normal(L)
    h = c * rate ** np.arange(L)
    y = causal_conv(h, x)
    rec = np.empty(L)
    acc = 0.0
    for t in range(L):
        acc = rate * acc + c * x[t]
        rec[t] = acc
    assert np.allclose(y, rec, rtol=1e-10, atol=1e-10)


def test_linearity():
    r = _rng(5)
    h1, h2, a1, a2 = (r.standard_normal(150) for _ in range(4))
    al, be = 0.3, -2.1
    assert np.allclose(causal_conv(h1, al * a1 + be * a2),
                       al * causal_conv(h1, a1) + be * causal_conv(h1, a2), atol=1e-11)
    assert np.allclose(causal_conv(al * h1 + be * h2, a1),
                       al * causal_conv(h1, a1) + be * causal_conv(h2, a1), atol=1e-11)


def test_brute_force_tiny_exact_integers():
    # Integer inputs: every sum is exact in float64, so compare bit for bit with
    # polynomial multiplication done in Python integers.
    r = _rng(6)
    for L in range(1, 17):
        h = r.integers(-9, 10, L)
        a = r.integers(-9, 10, L)
        prod = [0] * (2 * L - 1)
        for i in range(L):
            for j in range(L):
                prod[i + j] += int(h[i]) * int(a[j])
        assert np.array_equal(causal_conv(h, a), np.array(prod[:L], dtype=np.float64))


def test_causal_conv_at_matches_full():
    r = _rng(7)
    h, a = r.standard_normal((2, 512)), r.standard_normal((2, 512))
    ts = [0, 1, 17, 255, 511]
    ref = scipy.signal.fftconvolve(h, a, axes=-1)[:, ts]
    assert np.allclose(causal_conv_at(h, a, ts), ref, atol=1e-10)


# ----------------------------------------------------------------------------- tau / schedule
def test_tau_matches_convolution_slice():
    r = _rng(8)
    y, rho = r.standard_normal(64), r.standard_normal(64)
    l, rr, lp, rp = 8, 15, 16, 23
    yy = np.zeros(64)
    yy[l:rr + 1] = y[l:rr + 1]
    ref = np.convolve(yy, rho)[lp:rp + 1]
    assert np.allclose(tau(y, l, rr, rho, lp, rp), ref, atol=1e-12)


@pytest.mark.parametrize("L", [2, 16, 128, 1024])
def test_schedule_covers_every_pair_exactly_once(L):
    cover = np.zeros((L, L), dtype=np.int64)      # cover[s, t]
    for (i, U, s0, s1, t0, t1) in relaxed_tiles(L):
        assert U == lowbit(i)
        assert i + U <= L                            # targets never leave the sequence
        cover[s0:s1, t0:t1] += 1
    cover[np.arange(L), np.arange(L)] += 1          # red cells
    expect = np.triu(np.ones((L, L), dtype=np.int64))  # every s <= t once, nothing else
    assert np.array_equal(cover, expect)


def _facts():
    with open(GOLDEN) as f:
        return {x["name"]: x for x in json.load(f)["facts"]}


@pytest.mark.parametrize("P", [4, 10, 15, 17])
def test_schedule_counts_match_page(P):
    facts = _facts()
    L = 2 ** P
    sizes = np.array([lowbit(i) for i in range(1, L)])
    # Proposition 1: 2^(P-1-q) blocks of side 2^q.
    for q in range(P):
        assert np.sum(sizes == 2 ** q) == 2 ** (P - 1 - q)
    # Theorem 2: L-1 calls per layer.
    assert facts["tiles_total"]["value"] == "L-1" and len(sizes) == L - 1
    # 87.5% of blocks of side <= 4 and 93.75% of tokens on blocks <= 8 (limits as L grows).
    if P >= 10:
        assert abs(np.mean(sizes <= 4) - facts["frac_tiles_le_4"]["value"]) < 2e-3
        assert abs(np.mean(sizes <= 8) - facts["frac_tokens_le_8"]["value"]) < 2e-3


@pytest.mark.parametrize("U", [1, 2, 8, 64])
def test_circular_trick_window_is_linear(U):
    # Length-2U circular convolution of [x || 0] with h[0:2U]: outputs [U, 2U) equal
    # the block contribution (page: "Trucco di Convoluzione Circolare").
    r = _rng(U)
    L = 4 * U
    a = r.standard_normal(L)
    h = r.standard_normal(L)
    i = 2 * U                               # a step whose lowbit is >= U; use block side U
    xx = np.concatenate([a[i - U:i], np.zeros(U)])
    hh = h[:2 * U]
    circ = np.fft.irfft(np.fft.rfft(xx) * np.fft.rfft(hh), n=2 * U)
    ref = tau(a, i - U, i - 1, h, i, i + U - 1)
    assert np.allclose(circ[U:], ref, atol=1e-10)
    assert _facts()["circular_window"]["value"] == "[U, 2U-1]"


# ----------------------------------------------------------------------------- bf16
def test_bf16_round_hand_values():
    e = 2.0 ** -8
    cases = {1.0: 1.0, 1 + e: 1.0,                      # halfway -> even (1.0)
             1 + 3 * e: 1 + 4 * e,                      # halfway -> even (1 + 2^-6)
             1 + 1.5 * e: 1 + 2 * e, -1 - 3 * e: -1 - 4 * e,
             0.0: 0.0, 3.0: 3.0, 2 ** -100: 2 ** -100, 255.0: 255.0, 257.0: 256.0,
             259.0: 260.0}
    for x, want in cases.items():
        assert bf16_round(x) == want, (x, bf16_round(x), want)


def test_bf16_round_matches_torch_on_fp32_values():
    torch = pytest.importorskip("torch")
    r = _rng(9)
    x = (r.standard_normal(200000) * np.exp(r.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_idempotent_and_representable():
    r = _rng(10)
    x = bf16_round(r.standard_normal(10000))
    assert np.array_equal(bf16_round(x), x)
    bits = x.astype(np.float32).view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)


# ----------------------------------------------------------------------------- online model
def _small_stack(M=3, S=4, L=64, seed=11, lam=0.05):
    r = _rng(seed)
    t = np.arange(L)
    h = r.standard_normal((M, S, L)) * np.exp(-lam * t)
    x0 = r.standard_normal(S)
    eps = r.standard_normal((L, S))
    return h, x0, eps


@pytest.mark.parametrize("bf16", [False, True])
def test_online_equals_offline_of_final_sequence(bf16):
    h, x0, eps = _small_stack()
    if bf16:
        h = bf16_round(h)
    y, a = online_lcsm(h, x0, eps, bf16=bf16)
    M = h.shape[0]
    for l in range(M):
        off = scipy.signal.fftconvolve(h[l], a[l], axes=-1)[..., : a.shape[-1]]
        assert stream_error(y[l], off) < 1e-12
        if l + 1 < M:
            want = np.tanh(y[l])
            if bf16:
                want = bf16_round(want)
            assert np.allclose(a[l + 1], want, atol=0, rtol=0)
    # sampler rule
    want = np.tanh(y[-1][:, :-1]) + 0.1 * eps[:-1].T
    if bf16:
        want = bf16_round(want)
    assert np.array_equal(a[0][:, 1:], want)


def test_identity_filter_reduces_to_tanh_map():
    # One layer with h = delta_0: y_t = x_t and x_{t+1} = tanh(x_t) + 0.1 eps_t.
    L, S = 50, 3
    h = np.zeros((1, S, L))
    h[:, :, 0] = 1.0
    r = _rng(12)
    x0, eps = r.standard_normal(S), r.standard_normal((L, S))
    y, a = online_lcsm(h, x0, eps)
    x = x0.copy()
    for t in range(L):
        assert np.array_equal(y[0][:, t], x)
        x = np.tanh(x) + 0.1 * eps[t]


def test_pure_delay_filter():
    # h = delta_1: y_t = x_{t-1}, so x_{t+1} = tanh(x_{t-1}) + 0.1 eps_t.
    L, S = 40, 2
    h = np.zeros((1, S, L))
    h[:, :, 1] = 1.0
    r = _rng(13)
    x0, eps = r.standard_normal(S), r.standard_normal((L, S))
    y, a = online_lcsm(h, x0, eps)
    xs = [x0]
    for t in range(L - 1):
        prev = xs[t - 1] if t >= 1 else np.zeros(S)
        assert np.array_equal(y[0][:, t], prev)
        xs.append(np.tanh(prev) + 0.1 * eps[t])


def test_geometric_filters_match_recurrent_view():
    # With h^l_t = c_l r_l^t every layer is a one-state linear recurrence.
    M, S, L = 3, 5, 120
    r = _rng(14)
    c = r.uniform(0.5, 1.5, (M, S))
    rate = r.uniform(0.5, 0.95, (M, S))
    h = c[..., None] * rate[..., None] ** np.arange(L)
    x0, eps = r.standard_normal(S), r.standard_normal((L, S))
    y, a = online_lcsm(h, x0, eps)
    state = np.zeros((M, S))
    x = x0.copy()
    for t in range(L):
        inp = x
        for l in range(M):
            state[l] = rate[l] * state[l] + c[l] * inp
            assert np.allclose(y[l][:, t], state[l], rtol=1e-10, atol=1e-10)
            inp = np.tanh(state[l])
        x = np.tanh(state[-1]) + 0.1 * eps[t]


@pytest.mark.parametrize("bf16", [False, True])
def test_relaxed_schedule_reproduces_lazy(bf16):
    h, x0, eps = _small_stack(M=2, S=3, L=64)
    if bf16:
        h = bf16_round(h)
    y1, a1 = online_lcsm(h, x0, eps, bf16=bf16)
    y2, a2 = relaxed_online(h, x0, eps, bf16=bf16)
    if bf16:
        # bf16 rounding of the same real value agrees except at exact ties between
        # two summation orders; with random data the trajectories agree to 1e-9.
        assert stream_error(y2, y1) < 1e-9
    else:
        assert stream_error(y2, y1) < 1e-12
        assert np.allclose(a1, a2, atol=1e-12)


def test_partial_length_generation():
    h, x0, eps = _small_stack(L=64)
    y_full, _ = online_lcsm(h, x0, eps)
    y_part, _ = online_lcsm(h, x0, eps, n=20)
    assert np.array_equal(y_full[..., :20], y_part)


# ----------------------------------------------------------------------------- DFT
@pytest.mark.parametrize("N", [1, 2, 8, 60, 256, 4096])
def test_dft_matches_numpy_fft(N):
    r = _rng(N)
    x = r.standard_normal(N) + 1j * r.standard_normal(N)
    assert np.allclose(dft(x), np.fft.fft(x), atol=1e-9 * max(1, N))
    assert np.allclose(dft(x, inverse=True), np.fft.ifft(x) * N, atol=1e-9 * max(1, N))


def test_dft_special_cases():
    N = 64
    d = np.zeros(N)
    d[0] = 1.0
    assert np.allclose(dft(d), np.ones(N), atol=1e-14)                 # delta -> flat
    k0 = 5
    c = np.cos(2 * np.pi * k0 * np.arange(N) / N)
    X = dft(c)
    spikes = np.zeros(N)
    spikes[k0] = spikes[N - k0] = N / 2
    assert np.allclose(X, spikes, atol=1e-11)                          # cosine -> two spikes
    r = _rng(15)
    x = r.standard_normal(N) + 1j * r.standard_normal(N)
    assert np.isclose(np.sum(np.abs(x) ** 2), np.sum(np.abs(dft(x)) ** 2) / N)   # Parseval


def test_stream_error_definition():
    ref = np.array([[1.0, -4.0, 2.0], [0.5, 0.5, 0.5]])
    y = ref + np.array([[0.4, 0.0, 0.0], [0.0, 0.0, 0.05]])
    assert np.isclose(stream_error(y, ref), 0.1)


def test_oracle_header_marks_test_infrastructure():
    assert "TEST INFRASTRUCTURE ONLY" in oracle.__doc__


# --------------------------------------------------------------------------- prompt (prefill)
def test_prompt_single_layer_matches_numpy_convolve():
    r = np.random.default_rng(31)
    h = r.standard_normal((1, 3, 40))
    x = r.standard_normal((3, 25))
    y, a = oracle.prompt_lcsm(h, x)
    for s in range(3):
        assert np.allclose(y[0, s], np.convolve(h[0, s, :25], x[s])[:25], rtol=1e-12, atol=1e-12)
    assert np.array_equal(a[0], x)


def test_prompt_of_closed_loop_tokens_reproduces_the_closed_loop():
    # Feeding a closed-loop trajectory's own tokens as a prompt gives back its
    # outputs and activations (the online model is the prompt model on the
    # tokens it generates).
    r = np.random.default_rng(32)
    M, S, L = 3, 4, 48
    h = r.standard_normal((M, S, L)) * np.exp(-0.05 * np.arange(L))
    x0 = r.standard_normal(S)
    eps = r.standard_normal((L, S))
    for bf16 in (False, True):
        hh = oracle.bf16_round(h) if bf16 else h
        y_ref, a_ref = oracle.online_lcsm(hh, x0, eps, 0.1, bf16)
        y, a = oracle.prompt_lcsm(hh, a_ref[0], bf16)
        assert np.allclose(y, y_ref, rtol=0, atol=1e-12)
        assert np.allclose(a, a_ref, rtol=0, atol=1e-12)


def test_prompt_identity_filter_is_iterated_tanh():
    # h = delta: every layer's output is its own input, so y^l = tanh^(l-1)(x).
    M, S, p = 4, 2, 10
    h = np.zeros((M, S, 16))
    h[:, :, 0] = 1.0
    x = np.linspace(-2, 2, S * p).reshape(S, p)
    y, _ = oracle.prompt_lcsm(h, x)
    want = x.copy()
    for l in range(M):
        assert np.allclose(y[l], want, atol=1e-15)
        want = np.tanh(want)


# ---------------------------------------------------------------------------- channel-mixing block
def test_gelu_is_x_times_normal_cdf():
    # GELU(x) = x Phi(x), Phi from scipy's normal distribution (an independent
    # implementation), and the identity GELU(x) - GELU(-x) = x (Phi(x) + Phi(-x) = 1)
    import scipy.stats
    x = np.linspace(-8, 8, 2001)
    ref = x * scipy.stats.norm.cdf(x)
    assert np.max(np.abs(oracle.gelu(x) - ref)) <= 1e-15 * 8
    assert np.max(np.abs(oracle.gelu(x) - oracle.gelu(-x) - x)) <= 1e-14
    assert oracle.gelu(0.0) == 0.0


def test_mlp_block_matches_index_loops():
    rng = np.random.default_rng(3)
    B, D, Dh = 2, 5, 7
    y = rng.standard_normal((B, D))
    w1, b1 = rng.standard_normal((Dh, D)), rng.standard_normal(Dh)
    w2, b2 = rng.standard_normal((D, Dh)), rng.standard_normal(D)
    out = oracle.mlp_block(y, w1, b1, w2, b2)
    import math
    for b in range(B):
        z = []
        for k in range(Dh):
            u = b1[k] + sum(w1[k, d] * y[b, d] for d in range(D))
            z.append(0.5 * u * (1 + math.erf(u / math.sqrt(2))))
        for d in range(D):
            want = b2[d] + sum(w2[d, k] * z[k] for k in range(Dh))
            assert abs(out[b, d] - want) <= 1e-12 * max(1.0, abs(want))


def _mlp_setup(M, B, D, Dh, L, seed):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((M, D, L)) * np.exp(-0.05 * np.arange(L))
    w1 = rng.standard_normal((M, Dh, D)) / np.sqrt(D)
    b1 = 0.1 * rng.standard_normal((M, Dh))
    w2 = rng.standard_normal((M, D, Dh)) / np.sqrt(Dh)
    b2 = 0.1 * rng.standard_normal((M, D))
    x0 = rng.standard_normal((B, D))
    eps = rng.standard_normal((L, B, D))
    return h, w1, b1, w2, b2, x0, eps


def test_mlp_constant_block_closed_form():
    # W2 = 0: every block outputs b2, so layers 2..M see a constant input and
    # y^l_t = b2^{l-1}_d * sum_{k <= t} h^l_k (prefix sums of the filter), and the
    # sampler's tokens are x_{t+1} = b2^M + eps_scale eps_t.
    M, B, D, Dh, L = 3, 2, 4, 3, 24
    h, w1, b1, w2, b2, x0, eps = _mlp_setup(M, B, D, Dh, L, 5)
    w2 = np.zeros_like(w2)
    y, a = oracle.online_lcsm_mlp(h, w1, b1, w2, b2, x0, eps, 0.25)
    for l in range(1, M):
        want = b2[l - 1][None, :, None] * np.cumsum(h[l], axis=-1)[None, :, :]
        assert np.max(np.abs(y[l] - want)) <= 1e-12
    toks = np.concatenate([x0[:, :, None], (b2[M - 1][None, :, None] + 0.25 * eps[:-1].transpose(1, 2, 0))], axis=-1)
    assert np.max(np.abs(a[0] - toks)) <= 1e-12
    assert np.max(np.abs(y[0] - np.stack([[causal_conv(h[0, d], toks[b, d]) for d in range(D)] for b in range(B)]))) <= 1e-12


@pytest.mark.parametrize("bf16", [False, True])
def test_mlp_online_equals_offline_of_final_sequence(bf16):
    # Each layer's outputs are the causal convolutions of its recorded inputs,
    # and each recorded input is the block of the layer below at the same position.
    M, B, D, Dh, L = 3, 2, 4, 6, 32
    h, w1, b1, w2, b2, x0, eps = _mlp_setup(M, B, D, Dh, L, 7)
    if bf16:
        h = bf16_round(h)
    R = bf16_round if bf16 else (lambda v: v)
    y, a = oracle.online_lcsm_mlp(h, w1, b1, w2, b2, x0, eps, 0.1, bf16=bf16)
    for l in range(M):
        for b in range(B):
            for d in range(D):
                assert np.max(np.abs(y[l, b, d] - causal_conv(h[l, d], a[l, b, d]))) <= 1e-10
    for l in range(1, M):
        for t in range(L):
            want = R(oracle.mlp_block(y[l - 1, :, :, t], w1[l - 1], b1[l - 1], w2[l - 1], b2[l - 1]))
            assert np.max(np.abs(a[l, :, :, t] - want)) <= 1e-12
    for t in range(L - 1):
        want = R(oracle.mlp_block(y[M - 1, :, :, t], w1[M - 1], b1[M - 1], w2[M - 1], b2[M - 1]) + 0.1 * eps[t])
        assert np.max(np.abs(a[0, :, :, t + 1] - want)) <= 1e-12

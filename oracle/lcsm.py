"""Plain float64 definitions of the online long-convolution mixer stack.

TEST INFRASTRUCTURE ONLY (see the package docstring): a slow, obviously correct
CPU statement of what the CUDA library computes. No blocking, no fusion, no
reordering beyond what the definitions below state.

Notation (0-indexed positions t = 0..L-1, layers l = 1..M, streams s = (b, d)):

* mixer of one layer (Flash Inference summary page, "Architettura del Modello",
  LCSM definition): y^l_t = sum_{s <= t} a^{l-1}_s * h^l_{t-s}, elementwise
  (Hadamard) over channels, so every channel is an independent 1-D sequence;
* block: a^l_t = R(tanh(y^l_t)) (the synthetic workloads' elementwise block),
  or the channel-mixing MLP + GELU block (online_lcsm_mlp);
* sampler: x_{t+1} = a^0_{t+1} = R(tanh(y^M_t) + 0.1 * eps_t);
* R is the identity for fp32 workloads and round-to-nearest-even to bfloat16
  for bf16 workloads.

Parity unpinned: none. Every function is pinned in tests/test_oracle.py.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# Schedule (Flash Inference summary page, "Algoritmo Principale", Strategia di
# Tiling / Algoritmo 1 and Proposizione 1).
# ----------------------------------------------------------------------------
def lowbit(i: int) -> int:
    """Largest power of two dividing i (i >= 1): the block side U at step i."""
    if i <= 0:
        raise ValueError("lowbit is defined for i >= 1")
    return i & -i


def relaxed_tiles(L: int):
    """Gray blocks of the relaxed schedule for a sequence of L positions.

    0-indexed reading of Algorithm 1: at step i (1 <= i <= L-1) with
    U = lowbit(i), the block adds the contribution of inputs at positions
    [i-U, i) to outputs at positions [i, i+U). Returned as tuples
    (i, U, src_lo, src_hi, dst_lo, dst_hi) with half-open ranges, dst clipped to L.
    """
    out = []
    for i in range(1, L):
        U = lowbit(i)
        out.append((i, U, i - U, i, i, min(i + U, L)))
    return out


# ----------------------------------------------------------------------------
# Contribution aggregate (summary page, "Definizione di Aggregazione di
# Contribuzione"): tau(y, [l, r], rho, [l', r'])_t = sum_{i=l}^{r} y_i rho_{t-i}.
# ----------------------------------------------------------------------------
def tau(y: np.ndarray, l: int, r: int, rho: np.ndarray, lp: int, rp: int) -> np.ndarray:
    """Contribution of y[l..r] to outputs t in [lp, rp] (inclusive ranges, as on the page).

    rho_k for k < 0 is taken as 0 (the filter is causal). Works on the last axis;
    leading axes are independent streams. Returns shape (..., rp - lp + 1).
    """
    y = np.asarray(y, dtype=np.float64)
    rho = np.asarray(rho, dtype=np.float64)
    out = np.zeros(y.shape[:-1] + (rp - lp + 1,), dtype=np.float64)
    for t in range(lp, rp + 1):
        acc = np.zeros(y.shape[:-1], dtype=np.float64)
        for i in range(l, r + 1):
            if t - i >= 0:
                acc = acc + y[..., i] * rho[..., t - i]
        out[..., t - lp] = acc
    return out


# ----------------------------------------------------------------------------
# The mixer: causal long convolution (summary page, "Definizione del Compito":
# z_t = sum_{i <= t} y_i rho_{t-i}; "Architettura del Modello": the LCSM mixer).
# ----------------------------------------------------------------------------
def causal_conv(h: np.ndarray, a: np.ndarray) -> np.ndarray:
    """y[..., t] = sum_{s=0}^{t} h[..., t-s] * a[..., s], in float64.

    h and a broadcast over leading axes; the last axis is time (length L).
    """
    h = np.asarray(h, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    L = a.shape[-1]
    shape = np.broadcast_shapes(h.shape[:-1], a.shape[:-1]) + (L,)
    y = np.empty(shape, dtype=np.float64)
    for t in range(L):
        y[..., t] = np.sum(h[..., t::-1] * a[..., : t + 1], axis=-1)
    return y


def causal_conv_at(h: np.ndarray, a: np.ndarray, ts) -> np.ndarray:
    """The same sum as causal_conv, evaluated only at positions ts (O(L) each)."""
    h = np.asarray(h, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    shape = np.broadcast_shapes(h.shape[:-1], a.shape[:-1])
    out = np.empty(shape + (len(ts),), dtype=np.float64)
    for j, t in enumerate(ts):
        out[..., j] = np.sum(h[..., t::-1] * a[..., : t + 1], axis=-1)
    return out


# ----------------------------------------------------------------------------
# bfloat16 rounding, from the format's definition: 8 significant bits
# (1 implicit + 7 stored), 8 exponent bits like fp32, round to nearest, ties to even.
# ----------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even), as float64.

    Exact for every finite value in bfloat16's normal range (which is fp32's);
    subnormals, infinities and NaNs are outside the workloads and not handled.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    k = np.rint(np.ldexp(m, 8))              # 8 significant bits; rint ties to even
    return np.ldexp(k, e - 8)


def _identity(x):
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# The online model (summary page, "Definizione del Compito": autoregressive
# generation; the activations a^l_i = block^l(mixer^l(a^{l-1})_i) and the
# sampler x_{i+1} from a^M_i). Lazy evaluation ("Tre Strategie di Calcolo":
# z_t computed on demand, O(t) per position, O(L^2) in total).
# ----------------------------------------------------------------------------
def online_lcsm(h: np.ndarray, x0: np.ndarray, eps: np.ndarray, eps_scale: float = 0.1,
                bf16: bool = False, n: int | None = None):
    """Closed-loop generation of n positions through an M-layer mixer stack.

    h:   [M][S][L] filters (per stream; already rounded by the caller in bf16 mode)
    x0:  [S] first token
    eps: [n][S] sampler noise (unscaled)
    Returns (y, a): y[l-1] = y^l, shape [M][S][n] (mixer outputs before the block),
    a[l] = a^l for l = 0..M-1, shape [M][S][n] (a^0 = x, the tokens).
    """
    h = np.asarray(h, dtype=np.float64)
    M, S, L = h.shape
    n = L if n is None else n
    R = bf16_round if bf16 else _identity
    eps = np.asarray(eps, dtype=np.float64)
    a = np.zeros((M, S, n), dtype=np.float64)
    y = np.zeros((M, S, n), dtype=np.float64)
    a[0, :, 0] = R(x0)
    for t in range(n):
        below = a[0, :, : t + 1]
        for l in range(M):
            # y^{l+1}_t = sum_{s <= t} h^{l+1}_{t-s} a^l_s
            y[l, :, t] = np.sum(h[l, :, t::-1] * below, axis=-1)
            if l + 1 < M:
                a[l + 1, :, t] = R(np.tanh(y[l, :, t]))
                below = a[l + 1, :, : t + 1]
        if t + 1 < n:
            a[0, :, t + 1] = R(np.tanh(y[M - 1, :, t]) + eps_scale * eps[t])
    return y, a


# ----------------------------------------------------------------------------
# Channel-mixing block (summary page, "Architettura del Modello": block^l maps
# R^D to R^D and includes an MLP; "Configurazione Sperimentale", synthetic
# setting: the blocks are MLP + GELU and the sampler adds noise). Reading: one
# hidden layer of width Dh, block^l(y) = W2^l GELU(W1^l y + b1^l) + b2^l per
# sequence, GELU in its exact form x * Phi(x) (Phi the standard normal CDF).
# ----------------------------------------------------------------------------
_erf = np.vectorize(__import__("math").erf, otypes=[np.float64])


def gelu(x) -> np.ndarray:
    """GELU(x) = x Phi(x) = x (1 + erf(x / sqrt 2)) / 2, float64."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / np.sqrt(2.0)))


def mlp_block(y: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray, b2: np.ndarray) -> np.ndarray:
    """block(y) = w2 @ gelu(w1 @ y + b1) + b2 along the channel axis.

    y: [..., D]; w1: [Dh][D]; b1: [Dh]; w2: [D][Dh]; b2: [D]. Returns [..., D].
    """
    y = np.asarray(y, dtype=np.float64)
    z = gelu(y @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64))
    return z @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)


def online_lcsm_mlp(h: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray, b2: np.ndarray,
                    x0: np.ndarray, eps: np.ndarray, eps_scale: float = 0.1, bf16: bool = False,
                    n: int | None = None):
    """Closed-loop generation with the channel-mixing block after every layer.

    h: [M][D][L] filters (rounded by the caller in bf16 mode); w1: [M][Dh][D];
    b1: [M][Dh]; w2: [M][D][Dh]; b2: [M][D]; x0: [B][D]; eps: [n][B][D].
    Per position t, layer by layer: y^l_t = sum_{s <= t} h^l_{t-s} a^{l-1}_s
    (per channel), a^l_t = R(block^l(y^l_t)) (across channels, per sequence);
    then x_{t+1} = R(a^M_t + eps_scale eps_t), with a^M_t the last layer's
    block output before rounding.
    Returns (y, a): y[l-1] = y^l, shape [M][B][D][n]; a[l] = a^l for l = 0..M-1.
    """
    h = np.asarray(h, dtype=np.float64)
    M, D, L = h.shape
    B = np.asarray(x0).shape[0]
    n = L if n is None else n
    R = bf16_round if bf16 else _identity
    eps = np.asarray(eps, dtype=np.float64)
    a = np.zeros((M, B, D, n), dtype=np.float64)
    y = np.zeros((M, B, D, n), dtype=np.float64)
    a[0, :, :, 0] = R(x0)
    for t in range(n):
        for l in range(M):
            # y^{l+1}_t = sum_{s <= t} h^{l+1}_{t-s} a^l_s, per (b, d)
            y[l, :, :, t] = np.sum(h[l][None, :, t::-1] * a[l, :, :, : t + 1], axis=-1)
            out = mlp_block(y[l, :, :, t], w1[l], b1[l], w2[l], b2[l])
            if l + 1 < M:
                a[l + 1, :, :, t] = R(out)
            elif t + 1 < n:
                a[0, :, :, t + 1] = R(out + eps_scale * eps[t])
    return y, a


def prompt_lcsm(h: np.ndarray, x: np.ndarray, bf16: bool = False):
    """The stack on a prompt whose tokens are all given (summary page,
    "Limitazioni" 4, Fase di Prompt: every prompt position is known up front).

    a^0 = R(x); for each layer y^l = causal convolution of a^{l-1} with h^l over
    the prompt, a^l = R(tanh(y^l)). No sampler: the tokens are the prompt's.
    h: [M][S][L] filters (per stream), x: [S][p] tokens.
    Returns (y, a) with y[l-1] = y^l and a[l] = a^l, each [M][S][p].
    """
    h = np.asarray(h, dtype=np.float64)
    M, S, L = h.shape
    x = np.asarray(x, dtype=np.float64)
    p = x.shape[-1]
    R = bf16_round if bf16 else _identity
    a = np.zeros((M, S, p), dtype=np.float64)
    y = np.zeros((M, S, p), dtype=np.float64)
    a[0] = R(x)
    for l in range(M):
        y[l] = causal_conv(h[l, :, :p], a[l])
        if l + 1 < M:
            a[l + 1] = R(np.tanh(y[l]))
    return y, a


def relaxed_online(h: np.ndarray, x0: np.ndarray, eps: np.ndarray, eps_scale: float = 0.1,
                   bf16: bool = False, n: int | None = None):
    """The same generation, computed in the order of the page's Algorithm 2.

    Per position p: for each layer the red cell b^l_p += a^{l-1}_p rho^l_0, the
    block a^l_p = R(tanh(b^l_p)), and the gray block that adds
    tau(a^{l-1}, [p+1-U, p], rho^l, [p+1, p+U]) with U = lowbit(p+1); then the
    sampler. Used to pin that the tiling reproduces the lazy definition.
    Returns (y, a) like online_lcsm.
    """
    h = np.asarray(h, dtype=np.float64)
    M, S, L = h.shape
    n = L if n is None else n
    R = bf16_round if bf16 else _identity
    eps = np.asarray(eps, dtype=np.float64)
    a = np.zeros((M, S, n), dtype=np.float64)
    b = np.zeros((M, S, n), dtype=np.float64)   # accumulators b^l, l = 1..M
    a[0, :, 0] = R(x0)
    for p in range(n):
        last = None
        for l in range(M):
            src = a[l]
            b[l, :, p] += src[:, p] * h[l, :, 0]
            if l + 1 < M:
                a[l + 1, :, p] = R(np.tanh(b[l, :, p]))
            else:
                last = b[l, :, p]
            if p + 1 < n:
                U = lowbit(p + 1)
                hi = min(p + U, n - 1)
                b[l, :, p + 1: hi + 1] += tau(src, p + 1 - U, p, h[l], p + 1, hi)
        if p + 1 < n:
            a[0, :, p + 1] = R(np.tanh(last) + eps_scale * eps[p])
    return b, a


# ----------------------------------------------------------------------------
# Discrete Fourier transform, written out (used to pin the FFT device code;
# Lemma 1 of the summary page computes tau through it).
# ----------------------------------------------------------------------------
def dft(x: np.ndarray, inverse: bool = False) -> np.ndarray:
    """X[k] = sum_n x[n] exp(-+2 pi i k n / N) over the last axis, unnormalised.

    The exponent uses (k n mod N) so the angle is exact before the float64 cos/sin.
    """
    x = np.asarray(x, dtype=np.complex128)
    N = x.shape[-1]
    sign = 1.0 if inverse else -1.0
    n = np.arange(N)
    out = np.empty_like(x)
    for k0 in range(0, N, 256):
        k = np.arange(k0, min(N, k0 + 256))
        ang = sign * 2.0 * np.pi * ((np.outer(k, n) % N) / N)
        w = np.cos(ang) + 1j * np.sin(ang)
        out[..., k0: k0 + len(k)] = x @ w.T
    return out


# ----------------------------------------------------------------------------
# Error metric: stream-normwise relative error (max over streams of
# max_t |y - y_ref| / max_t |y_ref|).
# ----------------------------------------------------------------------------
def stream_error(y: np.ndarray, y_ref: np.ndarray) -> float:
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    num = np.max(np.abs(y - y_ref), axis=-1)
    den = np.max(np.abs(y_ref), axis=-1)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(num / den)) if num.size else 0.0

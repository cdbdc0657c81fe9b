"""Seeded synthetic workloads for the online long-convolution mixer stack.

This module only draws random inputs; it holds none of the method's arithmetic.
Both the CUDA path (through the Python binding) and the float64 oracle receive
the arrays it returns, so the two sides see identical inputs.

Workload recipe (the five shapes studied for the Flash Inference hot path, on the
Hyena-style synthetic LCSM of the paper's "Configurazione Sperimentale" section):

* filters  h[l][d][t] = g[l][d][t] * exp(-lam[l][d] * t), g ~ N(0,1) i.i.d.,
  lam[l][d] ~ Uniform[lam_lo, lam_hi], one decay rate per (layer, channel);
* first token x_0[b][d] ~ N(0,1);
* sampler noise eps[t][b][d] ~ N(0,1), scaled by 0.1 inside the feedback rule.

Every array has its own numpy PCG64 stream keyed by (seed, kind, layer), so a
layer can be drawn without drawing the others, and drawing is parallel over
layers.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

KIND_TAPS = 1
KIND_LAMBDA = 2
KIND_X0 = 3
KIND_EPS = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input law of one synthetic workload."""

    name: str
    layers: int      # M
    channels: int    # D
    length: int      # L (power of two)
    batch: int       # B
    dtype: str       # "f32" or "bf16" (bf16 inputs and filters, fp32 accumulate)
    lam_lo: float
    lam_hi: float
    eps_scale: float = 0.1

    def with_batch(self, b: int) -> "Workload":
        return dataclasses.replace(self, batch=b, name=f"{self.name.split('-B')[0]}-B{b}")

    @property
    def streams(self) -> int:
        return self.batch * self.channels


# The five workloads: a tiny single-layer case, three Hyena-shaped stacks and a batch sweep.
WORKLOADS = {
    "tiny-1x16-L1K": Workload("tiny-1x16-L1K", 1, 16, 1024, 1, "f32", 1e-3, 1e-1),
    "hyena-8x768-L8K": Workload("hyena-8x768-L8K", 8, 768, 8192, 1, "f32", 1e-3, 1e-1),
    "hyena-18x864-L32K-B4": Workload("hyena-18x864-L32K-B4", 18, 864, 32768, 4, "f32", 1e-3, 1e-1),
    "longrange-4x1024-L128K-bf16": Workload("longrange-4x1024-L128K-bf16", 4, 1024, 131072, 1, "bf16",
                                            1e-5, 1e-3),
    "sweep-8x2048-L16K-bf16-B1": Workload("sweep-8x2048-L16K-bf16-B1", 8, 2048, 16384, 1, "bf16", 1e-3, 1e-1),
}
for _b in (8, 32, 64):
    _w = WORKLOADS["sweep-8x2048-L16K-bf16-B1"]
    WORKLOADS[f"sweep-8x2048-L16K-bf16-B{_b}"] = dataclasses.replace(
        _w, batch=_b, name=f"sweep-8x2048-L16K-bf16-B{_b}")

# Reduced-footprint shapes of the headline stack for profiler captures (about 1 GB
# on the device): the full layer/channel/batch shape at L = 2048, and a 64-channel
# slice at the full length L = 32768 (which reaches the largest FFT blocks).
WORKLOADS["hyena-18x864-L2K-B4"] = Workload("hyena-18x864-L2K-B4", 18, 864, 2048, 4, "f32", 1e-3, 1e-1)
WORKLOADS["hyena-18x64-L32K-B4"] = Workload("hyena-18x64-L32K-B4", 18, 64, 32768, 4, "f32", 1e-3, 1e-1)
# ... and of the batched bf16 stack (8 layers, B = 64): 128 channels at L = 4096.
WORKLOADS["sweep-8x128-L4K-bf16-B64"] = Workload("sweep-8x128-L4K-bf16-B64", 8, 128, 4096, 64, "bf16", 1e-3, 1e-1)
# ... and of the long-range stack: 64 channels at the full L = 131072 (which reaches the
# partitioned blocks of sides 32768 and 65536; 0.2 GB of state).
WORKLOADS["longrange-4x64-L128K-bf16"] = Workload("longrange-4x64-L128K-bf16", 4, 64, 131072, 1, "bf16", 1e-5, 1e-3)

HEADLINE = "hyena-18x864-L32K-B4"


def _rng(seed: int, kind: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, kind, *key])))


def decay_rates(w: Workload, seed: int) -> np.ndarray:
    """lam[l][d] ~ U[lam_lo, lam_hi] (float64)."""
    return _rng(seed, KIND_LAMBDA).uniform(w.lam_lo, w.lam_hi, size=(w.layers, w.channels))


def filter_layer(w: Workload, seed: int, layer: int, lam: np.ndarray | None = None,
                 channels: np.ndarray | slice | None = None) -> np.ndarray:
    """Filter taps of one layer, float32 [D][L] (or the selected channels)."""
    if lam is None:
        lam = decay_rates(w, seed)
    g = _rng(seed, KIND_TAPS, layer).standard_normal((w.channels, w.length), dtype=np.float32)
    lam_l = lam[layer]
    if channels is not None:
        g = g[channels]
        lam_l = lam_l[channels]
    t = np.arange(w.length, dtype=np.float64)
    out = np.empty(g.shape, dtype=np.float32)
    step = 64
    for d0 in range(0, g.shape[0], step):
        env = np.exp(-np.outer(lam_l[d0:d0 + step], t))
        out[d0:d0 + step] = (g[d0:d0 + step].astype(np.float64) * env).astype(np.float32)
    return out


def filters(w: Workload, seed: int, threads: int | None = None) -> np.ndarray:
    """All filters, float32 [M][D][L]."""
    lam = decay_rates(w, seed)
    out = np.empty((w.layers, w.channels, w.length), dtype=np.float32)
    threads = threads or min(w.layers, os.cpu_count() or 1, 16)

    def one(layer):
        out[layer] = filter_layer(w, seed, layer, lam)

    if threads <= 1 or w.layers == 1:
        for layer in range(w.layers):
            one(layer)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(w.layers)))
    return out


def first_token(w: Workload, seed: int) -> np.ndarray:
    """x_0, float32 [B][D]."""
    return _rng(seed, KIND_X0).standard_normal((w.batch, w.channels), dtype=np.float32)


def noise(w: Workload, seed: int, n: int | None = None, threads: int | None = None) -> np.ndarray:
    """Sampler noise eps, float32 [n][B][D] (unscaled N(0,1)); one stream per sequence."""
    n = w.length if n is None else n
    out = np.empty((n, w.batch, w.channels), dtype=np.float32)

    def one(b):
        out[:, b, :] = _rng(seed, KIND_EPS, b).standard_normal((n, w.channels), dtype=np.float32)

    threads = threads or min(w.batch, os.cpu_count() or 1, 16)
    if threads <= 1:
        for b in range(w.batch):
            one(b)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(w.batch)))
    return out


def token_stream(w: Workload, seed: int, n: int | None = None) -> np.ndarray:
    """An arbitrary input sequence x[t][b][d] ~ N(0,1) for open-loop (teacher-forced) runs."""
    n = w.length if n is None else n
    return _rng(seed, KIND_X0, 1).standard_normal((n, w.batch, w.channels), dtype=np.float32)

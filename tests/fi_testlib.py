"""Shared helpers for the GPU parity tests: inputs on both sides, and the checks.

Parity reading (closed-loop generation is chaotic, so two correct programs that
round differently drift apart): pass/fail is TEACHER-FORCED. The library records
every layer's input a^{l-1} (fi_read_activations) and output y^l (the rec buffer
of fi_generate); the float64 oracle recomputes y^l from the recorded inputs by
the plain causal convolution and checks the block and sampler rules pointwise.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}


def gpu_inputs(w: synth.Workload, seed: int, n: int | None = None, device="cuda"):
    """Draw a workload's inputs and place them on the device in the library's dtypes."""
    import torch
    n = w.length if n is None else n
    h = synth.filters(w, seed)
    x0 = synth.first_token(w, seed)
    eps = synth.noise(w, seed, n)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return dict(
        h_np=h, x0_np=x0, eps_np=eps,
        h=torch.from_numpy(h).to(device).to(td).contiguous(),
        x0=torch.from_numpy(x0).to(device).to(td).contiguous(),
        eps=torch.from_numpy(eps).to(device).contiguous(),
    )


def oracle_filters(h32: np.ndarray, dtype: str) -> np.ndarray:
    """The filter values the device computes with, in float64 (bf16 rounding done by the oracle)."""
    h = h32.astype(np.float64)
    return oracle.bf16_round(h) if dtype == "bf16" else h


def read_all_activations(ctx, n_pos: int):
    import torch
    out = []
    for layer in range(ctx.M):
        dst = torch.empty((n_pos, ctx.B, ctx.D), dtype=torch.float32, device="cuda")
        ctx.read_activations(layer, dst)
        out.append(dst)
    return out


def teacher_forced_errors(h64, acts, rec, streams, dtype, positions=None, t0=0):
    """Per-layer stream-normwise errors of the recorded outputs.

    h64: [M][D][L] float64 filters; acts[l]: [n][B][D] recorded a^l (numpy, l < M);
    rec: [M][n][B][D] recorded y^l (numpy); streams: list of (b, d); positions:
    None for every position (full causal conv), or a list of positions (each
    evaluated by its own O(t) sum). Positions are relative to t0 = 0 only.
    Returns dict with 'y' (max error over layers), 'block' (max |a^l - R(tanh y^l)|
    relative to max|a^l|, layers 1..M-1) and 'per_layer'.
    """
    M = h64.shape[0]
    R = oracle.bf16_round if dtype == "bf16" else (lambda v: v)
    per_layer = []
    block_err = 0.0
    for l in range(M):
        for (b, d) in streams:
            a_in = acts[l][:, b, d].astype(np.float64)
            y_gpu = rec[l][:, b, d].astype(np.float64)
            if positions is None:
                y_ref = oracle.causal_conv(h64[l, d, : len(a_in)], a_in)
                y_cmp = y_gpu
            else:
                y_ref = oracle.causal_conv_at(h64[l, d, : len(a_in)], a_in, positions)
                y_cmp = y_gpu[positions]
            per_layer.append((l, b, d, oracle.stream_error(y_cmp, y_ref)))
            if l + 1 < M:
                a_out = acts[l + 1][:, b, d].astype(np.float64)
                want = R(np.tanh(y_gpu))
                den = max(np.max(np.abs(want)), 1e-30)
                block_err = max(block_err, float(np.max(np.abs(a_out - want)) / den))
    return {"y": max(e for *_, e in per_layer), "block": block_err, "per_layer": per_layer}


def sampler_error(acts0, rec_last, eps, dtype, eps_scale=0.1):
    """max |x_{t+1} - R(tanh(y^M_t) + 0.1 eps_t)| over the recorded positions."""
    R = oracle.bf16_round if dtype == "bf16" else (lambda v: v)
    want = R(np.tanh(rec_last[:-1].astype(np.float64)) + eps_scale * eps[:-1].astype(np.float64))
    got = acts0[1:].astype(np.float64)
    return float(np.max(np.abs(got - want)))

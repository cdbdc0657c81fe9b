"""The tensor-core block's operand layout, emulated on CPU.

k_tile_tc reads its A operand (the filter) from a table of 16-byte entries,
entry s = h[s+1 .. s+8], through a K-major, no-swizzle shared-memory descriptor
whose row-group and K-half strides are both 128 bytes, and its B operand (the
sources, reversed, one row per (target tile j, sequence b)) from core matrices
laid out at ((k/8)*(R/8) + n/8)*128 + (n%8)*16 + (k%8)*2. This test reads both
operands the way such a descriptor addresses shared memory, multiplies them K
step by K step, and checks the result against the block's definition (the
oracle's tau) for every plan shape the library can choose; it also checks that
no read leaves the operand buffers.
"""
import numpy as np
import pytest

import oracle


def _plan(U, B):
    # the library's choice of tile rows, tiles per product and operand rows
    MT = 128 if (U >= 128 and B % 16 == 0) else 64
    NT = U // MT
    J = 1
    while J < NT and B * J < 16:
        J *= 2
    mult = 16 if MT == 128 else 8
    NR = (B * J + mult - 1) // mult * mult
    return MT, J, NR, U + (J - 1) * MT


def _read_operand(mem, start, rows, lbo, sbo):
    """rows x 16 K-major operand from a byte-addressed buffer of 2-byte elements."""
    r = np.arange(rows)[:, None]
    k = np.arange(16)[None, :]
    addr = start + (r // 8) * sbo + (k // 8) * lbo + (r % 8) * 16 + (k % 8) * 2
    assert addr.min() >= 0 and addr.max() + 2 <= 2 * len(mem)
    return mem[addr // 2]


@pytest.mark.parametrize("U,B", [(64, 1), (64, 4), (128, 3), (128, 16), (256, 4), (256, 8), (256, 64), (512, 4)])
def test_descriptor_reads_give_the_block(U, B):
    rng = np.random.default_rng(U + B)
    L = 4 * U
    i = 3 * U                                     # a step whose lowest set bit is U
    h = rng.standard_normal(L)
    x = rng.standard_normal((B, L))
    MT, J, NR, K = _plan(U, B)
    assert K % 16 == 0
    # table: 2U entries of 8 taps
    table = np.zeros(2 * U * 8)
    for s in range(2 * U):
        for e in range(8):
            table[8 * s + e] = h[s + 1 + e] if s + 1 + e < L else 0.0
    # B operand: row n = j*B + b holds x[b][i-1-kappa+j*MT] at kappa in [j*MT, j*MT+U)
    xs = np.zeros(NR * K)
    for j in range(J):
        for b in range(B):
            n = j * B + b
            for kap in range(j * MT, j * MT + U):
                addr = ((kap // 8) * (NR // 8) + n // 8) * 128 + (n % 8) * 16 + (kap % 8) * 2
                xs[addr // 2] = x[b, i - 1 - kap + j * MT]
    lbo_b = (NR // 8) * 128
    out = np.zeros((U, B))
    for gi in range(U // MT // J):
        D = np.zeros((MT, NR))
        for ks in range(K // 16):
            A = _read_operand(table, (gi * J * MT + 16 * ks) * 16, MT, 128, 128)
            Bm = _read_operand(xs, 2 * ks * lbo_b, NR, lbo_b, 128)
            D += A @ Bm.T
        for j in range(J):
            for b in range(B):
                out[(gi * J + j) * MT:(gi * J + j + 1) * MT, b] = D[:, j * B + b]
    for b in range(B):
        ref = oracle.tau(x[b], i - U, i - 1, h, i, i + U - 1)
        assert np.allclose(out[:, b], ref, rtol=1e-12, atol=1e-12)

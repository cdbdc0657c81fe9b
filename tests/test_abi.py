"""The C-ABI library loads on a machine without a GPU, exports every symbol that
include/fi.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fi.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FI_API\s+[\w\s\*]+?\b(fi_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for must in ("fi_init", "fi_step", "fi_generate", "fi_reset", "fi_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol():
    from long_convolution_sequence_online_b200 import fi
    lib = ctypes.CDLL(fi.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(fi.EXPORTED) == declared_symbols()


def test_status_strings():
    from long_convolution_sequence_online_b200 import fi
    assert fi.status_str(0) == "ok"
    assert fi.status_str(fi.FI_E_STATE) == "invalid state"
    assert fi.status_str(99) == "unknown status"


def _init(cfg, h=ctypes.c_void_p(16)):
    from long_convolution_sequence_online_b200 import fi
    out = ctypes.c_void_p(1)
    s = fi.lib.fi_init(ctypes.byref(out), ctypes.byref(cfg), h, None)
    return s, out


@pytest.mark.parametrize("fields,why", [
    (dict(layers=0, channels=4, max_len=64, batch=1), "layers"),
    (dict(layers=1, channels=0, max_len=64, batch=1), "channels"),
    (dict(layers=1, channels=4, max_len=48, batch=1), "power of two"),
    (dict(layers=1, channels=4, max_len=1, batch=1), "power of two"),
    (dict(layers=1, channels=4, max_len=1 << 18, batch=1), "power of two"),
    (dict(layers=1, channels=4, max_len=64, batch=0), "batch"),
    (dict(layers=1, channels=4, max_len=64, batch=1, dtype=7), "dtype"),
    (dict(layers=1, channels=4, max_len=64, batch=1, chunk=3), "chunk"),
    (dict(layers=1, channels=4, max_len=64, batch=1, chunk=128), "chunk"),
    (dict(layers=1, channels=4, max_len=64, batch=1, fft_from=32), "fft_from"),
    (dict(layers=1, channels=4, max_len=64, batch=1, tc_max=32), "tc_max"),
    (dict(layers=1, channels=4, max_len=64, batch=1, tc_max=-2), "tc_max"),
    (dict(layers=1, channels=4, max_len=64, batch=1, tc_max=96), "tc_max"),
])
def test_init_rejects_bad_config_without_gpu(fields, why):
    from long_convolution_sequence_online_b200 import fi
    cfg = fi.Config(**fields)
    s, out = _init(cfg)
    assert s == fi.FI_E_INVALID
    assert out.value is None
    assert why in fi.lib.fi_last_error().decode()


def test_init_rejects_reserved_and_nulls():
    from long_convolution_sequence_online_b200 import fi
    cfg = fi.Config(1, 4, 64, 1)
    cfg.reserved[2] = 1
    assert _init(cfg)[0] == fi.FI_E_INVALID
    cfg = fi.Config(1, 4, 64, 1)
    assert _init(cfg, h=None)[0] == fi.FI_E_INVALID
    assert fi.lib.fi_init(None, ctypes.byref(cfg), ctypes.c_void_p(16), None) == fi.FI_E_INVALID


def test_calls_on_null_context_are_rejected():
    from long_convolution_sequence_online_b200 import fi
    L = fi.lib
    assert L.fi_destroy(None) == fi.FI_OK
    assert L.fi_reset(None) == fi.FI_E_INVALID
    assert L.fi_step(None, None, None) == fi.FI_E_INVALID
    assert L.fi_generate(None, 4, None, None, 0.1, None, None) == fi.FI_E_INVALID
    assert L.fi_generate_lazy(None, 4, None, None, 0.1, None) == fi.FI_E_INVALID
    assert L.fi_generate_host(None, 4, None, None, 0.1, None) == fi.FI_E_INVALID
    p = ctypes.c_int32()
    assert L.fi_position(None, ctypes.byref(p)) == fi.FI_E_INVALID
    assert L.fi_read_activations(None, 0, None) == fi.FI_E_INVALID
    assert L.fi_profile(None, 1) == fi.FI_E_INVALID
    assert L.fi_debug_fft(5, 1, ctypes.c_void_p(16), ctypes.c_void_p(16), 0, None) == fi.FI_E_INVALID
    assert L.fi_debug_fft(15, 1, ctypes.c_void_p(16), ctypes.c_void_p(16), 0, None) == fi.FI_E_INVALID


def test_python_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    from long_convolution_sequence_online_b200 import fi
    with pytest.raises(ValueError):
        fi._ptr(torch.zeros(4))


@pytest.mark.parametrize("chunk", [2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("retimed,coarse", [(False, False), (True, False), (True, True)])
def test_chunk_piece_table_covers_every_pair_once_in_time(chunk, retimed, coarse):
    """The on-chip pieces of a chunk and the chain together sum every (source s,
    target t) pair with s < t inside the chunk exactly once.

    Page's tiling (retimed=False): one square block of side lowbit(r) per step r,
    sources [r-U, r), targets [r, r+U); a piece at step r reads sources below r
    (final once position r-1 is done) and writes targets >= r (the chain reads
    target t after the pieces of step t).
    Re-timed (the whole chunk in one launch): the chain adds the pairs of lags
    1 and 2 itself, and the pieces cover every pair with t - s >= 3 with the
    page's tiling shifted by two targets (the chain reads target t after the
    pieces of step t-2, so a piece at step r writes targets >= r+2); a piece may
    also reach the window's spare positions t = chunk, chunk+1 (never read).
    Lags stay below chunk+2 (taps from `chunk` up are held as zero); the
    re-timed pieces hold at most 64 products per row each and are spread so that
    no step carries more than 96 (the coarse cut for short stacks: 16 x 16 pieces,
    at most 256 and 320)."""
    from long_convolution_sequence_online_b200 import fi
    sh, tab = fi.chunk_schedule(chunk, retimed, coarse)
    assert sh == (2 if retimed else 0)
    count = {}
    per_step = {}
    for step, s_lo, ns, t_lo, nd in tab:
        assert 1 <= step < chunk
        assert s_lo >= 0 and s_lo + ns <= step, (step, s_lo, ns)
        assert t_lo >= step + sh and t_lo < chunk and t_lo + nd <= chunk + sh, (step, t_lo, nd)
        assert t_lo - (s_lo + ns - 1) >= 1 + sh and (t_lo + nd - 1) - s_lo <= chunk + sh - 1
        per_step.setdefault(step, []).append((s_lo, ns, t_lo, nd))
        for s in range(s_lo, s_lo + ns):
            for t in range(t_lo, min(t_lo + nd, chunk)):
                count[(s, t)] = count.get((s, t), 0) + 1
    want = {(s, t) for t in range(chunk) for s in range(t) if t - s >= 1 + sh}
    assert set(count) == want
    assert all(v == 1 for v in count.values())
    assert [step for step, *_ in tab] == sorted(step for step, *_ in tab)
    for r in range(1, chunk - sh):
        U = r & -r
        pieces = per_step.get(r, [])
        if not retimed:
            assert pieces == [(r - U, U, r, U)]
        else:
            if U <= 8 and r + sh < chunk:
                assert (r - U, U, r + sh, U) in pieces
            assert max(ns * nd for _, ns, _, nd in pieces) <= (256 if coarse else 64)
            assert sum(ns * nd for _, ns, _, nd in pieces) <= (320 if coarse else 96)

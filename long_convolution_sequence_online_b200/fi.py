"""Thin ctypes binding of libfi.so (include/fi.h): argument marshalling only.

Every computation runs in the library's CUDA kernels. PyTorch supplies device
memory (tensors' data pointers) and the current CUDA stream. If libfi.so is
missing or fails to load, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfi.so")

FI_OK, FI_E_INVALID, FI_E_OOM, FI_E_CUDA, FI_E_STATE, FI_E_TIMEOUT, FI_E_UNSUPPORTED = range(7)
FI_F32, FI_BF16 = 0, 1
NUM_KERNEL_CLASSES = 6
KERNEL_CLASSES = ("chunk", "direct", "fft", "token", "lazy", "tc")

EXPORTED = ("fi_init", "fi_step", "fi_generate", "fi_generate_host", "fi_generate_lazy", "fi_sync", "fi_reset",
            "fi_position", "fi_read_activations", "fi_set_stream", "fi_get_plan", "fi_profile",
            "fi_profile_read", "fi_destroy", "fi_status_str", "fi_last_error", "fi_debug_fft",
            "fi_generate_noalloc", "fi_debug_set_wait_limit", "fi_debug_chunk_schedule", "fi_prefill", "fi_profile_read_sides",
            "fi_set_mlp_block")


class FiError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status}: {message}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("channels", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("batch", ctypes.c_int32), ("dtype", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("fft_from", ctypes.c_int32), ("tc_max", ctypes.c_int32), ("reserved", ctypes.c_int32 * 4)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m long_convolution_sequence_online_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    sig = {
        "fi_init": [ctypes.POINTER(vp), ctypes.POINTER(Config), vp, vp],
        "fi_step": [vp, vp, vp],
        "fi_generate": [vp, i32, vp, vp, f32, vp, vp],
        "fi_generate_host": [vp, i32, vp, vp, f32, vp],
        "fi_generate_lazy": [vp, i32, vp, vp, f32, vp],
        "fi_reset": [vp],
        "fi_sync": [vp],
        "fi_position": [vp, ctypes.POINTER(i32)],
        "fi_read_activations": [vp, i32, vp],
        "fi_set_stream": [vp, vp],
        "fi_get_plan": [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "fi_profile": [vp, i32],
        "fi_profile_read": [vp, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double)],
        "fi_destroy": [vp],
        "fi_debug_fft": [i32, i32, vp, vp, i32, vp],
        "fi_generate_noalloc": [ctypes.POINTER(Config), vp, i32, vp, vp, f32, vp, vp],
        "fi_debug_set_wait_limit": [vp, i32],
        "fi_debug_chunk_schedule": [i32, i32, vp, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "fi_prefill": [vp, i32, vp, vp, vp],
        "fi_set_mlp_block": [vp, i32, vp, vp, vp, vp],
        "fi_profile_read_sides": [vp, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i32),
                                  ctypes.POINTER(ctypes.c_double)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.fi_status_str.argtypes = [ctypes.c_int]
    lib.fi_status_str.restype = ctypes.c_char_p
    lib.fi_last_error.argtypes = []
    lib.fi_last_error.restype = ctypes.c_char_p
    return lib


lib = _load()


def _check(status: int, where: str):
    if status != FI_OK:
        raise FiError(status, where, (lib.fi_last_error() or b"").decode())


def _ptr(t) -> int | None:
    """Device address of a contiguous CUDA tensor (None passes through as NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream) if not hasattr(stream, "cuda_stream") else stream.cuda_stream


class Context:
    """One fi_ctx: filters, spectra and state of an M-layer online mixer stack."""

    def __init__(self, h, batch: int, dtype: str = "f32", chunk: int = 0, fft_from: int = 0, stream=None,
                 tc_max: int = 0):
        import torch
        if h.dim() != 3:
            raise ValueError("h must be [M][D][L]")
        want = torch.bfloat16 if dtype == "bf16" else torch.float32
        if h.dtype != want:
            raise ValueError(f"h must be {want} for dtype {dtype}")
        M, D, L = h.shape
        self.M, self.D, self.L, self.B = int(M), int(D), int(L), int(batch)
        self.dtype = dtype
        self.torch_dtype = want
        cfg = Config(self.M, self.D, self.L, self.B, FI_BF16 if dtype == "bf16" else FI_F32, chunk, fft_from, tc_max)
        self._cfg = cfg
        self._h = ctypes.c_void_p()
        _check(lib.fi_init(ctypes.byref(self._h), ctypes.byref(cfg), _ptr(h), _stream(stream)), "fi_init")

    # -- lifetime
    def close(self):
        if self._h:
            _check(lib.fi_destroy(self._h), "fi_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- calls
    def set_stream(self, stream):
        _check(lib.fi_set_stream(self._h, _stream(stream)), "fi_set_stream")

    def step(self, x_t, y_t):
        _check(lib.fi_step(self._h, _ptr(x_t), _ptr(y_t)), "fi_step")

    def step_ptr(self, x_ptr: int, y_ptr: int):
        """fi_step on raw device addresses (a loop over positions without tensor views)."""
        _check(lib.fi_step(self._h, x_ptr, y_ptr), "fi_step")

    def generate(self, n: int, x0, eps, y_out, eps_scale: float = 0.1, rec=None):
        _check(lib.fi_generate(self._h, n, _ptr(x0), _ptr(eps), eps_scale, _ptr(y_out), _ptr(rec)), "fi_generate")

    def prefill(self, p: int, x, y_out=None, rec=None):
        _check(lib.fi_prefill(self._h, p, _ptr(x), _ptr(y_out), _ptr(rec)), "fi_prefill")

    def set_mlp_block(self, w1=None, b1=None, w2=None, b2=None):
        """Channel-mixing block W2 GELU(W1 y + b1) + b2 after every layer (fp32 CUDA
        tensors w1 [M][Dh][D], b1 [M][Dh], w2 [M][D][Dh], b2 [M][D]); no arguments
        return to the elementwise tanh block."""
        hidden = 0 if w1 is None else int(w1.shape[1])
        _check(lib.fi_set_mlp_block(self._h, hidden, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2)), "fi_set_mlp_block")

    def generate_host(self, n: int, x0: np.ndarray, eps: np.ndarray, y_out: np.ndarray, eps_scale: float = 0.1):
        for a in (x0, eps, y_out):
            if not a.flags["C_CONTIGUOUS"]:
                raise ValueError("host arrays must be C-contiguous")
        _check(lib.fi_generate_host(self._h, n, x0.ctypes.data, eps.ctypes.data, eps_scale, y_out.ctypes.data),
               "fi_generate_host")

    def generate_host_ptr(self, n: int, x0_ptr: int, eps_ptr: int, y_ptr: int, eps_scale: float = 0.1):
        _check(lib.fi_generate_host(self._h, n, x0_ptr, eps_ptr, eps_scale, y_ptr), "fi_generate_host")

    def generate_lazy(self, n: int, x0, eps, y_out, eps_scale: float = 0.1):
        _check(lib.fi_generate_lazy(self._h, n, _ptr(x0), _ptr(eps), eps_scale, _ptr(y_out)), "fi_generate_lazy")

    def sync(self):
        _check(lib.fi_sync(self._h), "fi_sync")

    def reset(self):
        _check(lib.fi_reset(self._h), "fi_reset")

    def set_wait_limit(self, limit: int):
        _check(lib.fi_debug_set_wait_limit(self._h, limit), "fi_debug_set_wait_limit")

    @property
    def position(self) -> int:
        p = ctypes.c_int32()
        _check(lib.fi_position(self._h, ctypes.byref(p)), "fi_position")
        return p.value

    def read_activations(self, layer: int, dst):
        _check(lib.fi_read_activations(self._h, layer, _ptr(dst)), "fi_read_activations")

    def plan(self):
        """(chunk, fft_from, tc_max) after automatic selection; 0 = that kind of block is not used."""
        c, f, t = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.fi_get_plan(self._h, ctypes.byref(c), ctypes.byref(f), ctypes.byref(t)), "fi_get_plan")
        return c.value, f.value, t.value

    def profile(self, enable: bool):
        _check(lib.fi_profile(self._h, 1 if enable else 0), "fi_profile")

    def profile_read(self):
        counts = (ctypes.c_int32 * NUM_KERNEL_CLASSES)()
        ms = (ctypes.c_double * NUM_KERNEL_CLASSES)()
        _check(lib.fi_profile_read(self._h, counts, ms), "fi_profile_read")
        return {KERNEL_CLASSES[k]: (counts[k], ms[k]) for k in range(NUM_KERNEL_CLASSES)}

    def profile_read_sides(self):
        """(per-class dict as profile_read, {block side: (launches, ms)})."""
        counts = (ctypes.c_int32 * NUM_KERNEL_CLASSES)()
        ms = (ctypes.c_double * NUM_KERNEL_CLASSES)()
        sc = (ctypes.c_int32 * 32)()
        sm = (ctypes.c_double * 32)()
        _check(lib.fi_profile_read_sides(self._h, counts, ms, sc, sm), "fi_profile_read_sides")
        return ({KERNEL_CLASSES[k]: (counts[k], ms[k]) for k in range(NUM_KERNEL_CLASSES)},
                {1 << q: (sc[q], sm[q]) for q in range(32) if sc[q]})


def debug_fft(log2n: int, x, out, inverse: bool = False, stream=None):
    """The library's device FFT on x (complex64 CUDA tensor [count][2^log2n]) into out."""
    count = x.numel() >> log2n
    _check(lib.fi_debug_fft(log2n, count, _ptr(x), _ptr(out), 1 if inverse else 0, _stream(stream)), "fi_debug_fft")


def generate_noalloc(h, batch: int, n: int, x0, eps, y_out, dtype: str = "f32", eps_scale: float = 0.1,
                     chunk: int = 0, stream=None):
    """fi_generate_noalloc: one generation from position 0 with no device allocation."""
    M, D, L = (int(v) for v in h.shape)
    cfg = Config(M, D, L, int(batch), FI_BF16 if dtype == "bf16" else FI_F32, chunk, 0)
    _check(lib.fi_generate_noalloc(ctypes.byref(cfg), _ptr(h), n, _ptr(x0), _ptr(eps), eps_scale, _ptr(y_out),
                                   _stream(stream)), "fi_generate_noalloc")


def chunk_schedule(chunk: int, retimed: bool, coarse: bool = False):
    """The chunk kernel's table of on-chip block pieces (host only): (lags the
    chain adds itself, [(step, first source, sources, first target, targets)]),
    chunk-relative. coarse: the cut used for stacks of at most 8 layers."""
    cap = 4 * chunk
    out = (ctypes.c_int32 * (5 * cap))()
    n, lags = ctypes.c_int32(), ctypes.c_int32()
    mode = (2 if coarse else 1) if retimed else 0
    _check(lib.fi_debug_chunk_schedule(chunk, mode, ctypes.cast(out, ctypes.c_void_p), cap,
                                       ctypes.byref(n), ctypes.byref(lags)), "fi_debug_chunk_schedule")
    return lags.value, [tuple(out[5 * j: 5 * j + 5]) for j in range(min(n.value, cap))]


def status_str(s: int) -> str:
    return lib.fi_status_str(s).decode()

"""Python binding of libfi.so, the B200 Flash Inference mixer (see include/fi.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libfi.so.  Arrays may be torch tensors (host or CUDA) or numpy arrays;
they must be contiguous float32.  If libfi.so has not been built, the first use
of the library raises ImportError -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_LIB_PATH = Path(__file__).resolve().parent / "libfi.so"

FI_OK, FI_EINVAL, FI_ECAPACITY, FI_ENOMEM, FI_ECUDA, FI_ESTATE = 0, -1, -2, -3, -4, -5
FI_TAU_AUTO, FI_TAU_DIRECT, FI_TAU_FFT = 0, 1, 2
FI_PATH_WINDOW, FI_PATH_TOKEN, FI_PATH_LAZY, FI_PATH_EAGER, FI_PATH_LAZY_NP, FI_PATH_EAGER_NP = range(6)


class FiError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("fi error %d: %s" % (code, msg))
        self.code = code


class fi_info(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int), ("B", ctypes.c_int), ("D", ctypes.c_int), ("L", ctypes.c_int),
                ("t", ctypes.c_int), ("window", ctypes.c_int), ("chains_per_cta", ctypes.c_int),
                ("path", ctypes.c_int), ("graphs", ctypes.c_int), ("tau", ctypes.c_int * 32),
                ("tau_us", (ctypes.c_float * 2) * 32), ("device_bytes", ctypes.c_size_t),
                ("sm_count", ctypes.c_int), ("launches", ctypes.c_longlong)]


FI_K_WINDOW, FI_K_TOKEN_STEP, FI_K_BLOCK_DIRECT, FI_K_BLOCK_FFT, FI_K_BLOCK_CLUSTER = range(5)
FI_K_CLASSES = 5
KERNEL_CLASS_NAMES = ("window", "token_step", "block_direct", "block_fft", "block_cluster")


class fi_trace(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int * FI_K_CLASSES), ("total_us", ctypes.c_double * FI_K_CLASSES),
                ("max_us", ctypes.c_double * FI_K_CLASSES),
                ("block_launches", ctypes.c_int * 32), ("block_us", ctypes.c_double * 32)]


# Every entry point declared in include/fi.h, with its C signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "fi_create": (_P, [_I, _I, _I, _I, _P]),
    "fi_destroy": (None, [_P]),
    "fi_step": (_I, [_P, _P, _P]),
    "fi_generate": (_I, [_P, _P, _I, _P]),
    "fi_forward": (_I, [_P, _P, _I, _P]),
    "fi_prefill": (_I, [_P, _P, _I, _P]),
    "fi_reset": (_I, [_P]),
    "fi_read_layer": (_I, [_P, _I, _I, _I, _P]),
    "fi_set_stream": (_I, [_P, _P]),
    "fi_set_path": (_I, [_P, _I]),
    "fi_set_graphs": (_I, [_P, _I]),
    "fi_set_tau": (_I, [_P, _I, _I]),
    "fi_get_info": (_I, [_P, ctypes.POINTER(fi_info)]),
    "fi_set_trace": (_I, [_P, _I]),
    "fi_trace_read": (_I, [_P, ctypes.POINTER(fi_trace)]),
    "fi_debug_schedule": (_I, [_P, _I] + [ctypes.POINTER(_I)] * 5),
    "fi_trace_launches": (_I, [_P, _I, _P, _P, _P]),
    "fi_tau": (_I, [_I, _I, _I, _P, _P, _I, _P, _I]),
    "fi_tau_fft_noalloc": (_I, [_I, _I, _P, _P, _I, _P, _I]),
    "fi_lm_create": (_P, [_I, _I, _I, _I, _I] + [_P] * 7),
    "fi_lm_destroy": (None, [_P]),
    "fi_lm_reset": (_I, [_P]),
    "fi_lm_forward": (_I, [_P, _P, _I, _P, _P]),
    "fi_lm_generate": (_I, [_P, _P, _I, _P]),
    "fi_lm_set_trace": (_I, [_P, _I]),
    "fi_lm_set_graphs": (_I, [_P, _I]),
    "fi_lm_split": (_I, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "fi_dd_create": (_P, [_I, _I]),
    "fi_dd_destroy": (None, [_P]),
    "fi_dd_reset": (_I, [_P]),
    "fi_dd_forward": (_I, [_P, _P, _P, _I, _P]),
    "fi_dd_set_tau": (_I, [_P, _I, _I]),
    "fi_last_error": (ctypes.c_char_p, []),
    "fi_version": (ctypes.c_char_p, []),
}


def _load():
    if not _LIB_PATH.exists():
        raise ImportError("libfi.so is not built (run __graft_entry__.build() or "
                          "python -m long_convolution_sequence_b200.build); no fallback exists")
    lib = ctypes.CDLL(str(_LIB_PATH))
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = None


def get_lib():
    """The loaded libfi.so (raises ImportError if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def __getattr__(name):
    if name == "lib":
        return get_lib()
    raise AttributeError(name)


def last_error() -> str:
    return get_lib().fi_last_error().decode()


def _check(rc):
    if rc != FI_OK:
        raise FiError(rc, last_error())


def _ptr(a):
    """Address of a contiguous float32 torch tensor / numpy array (None -> NULL)."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):  # torch
        assert a.is_contiguous(), "tensor must be contiguous"
        assert str(a.dtype) == "torch.float32", "tensor must be float32"
        return a.data_ptr()
    import numpy as np
    assert isinstance(a, np.ndarray) and a.dtype == np.float32 and a.flags.c_contiguous
    return a.ctypes.data


class FlashInference:
    """One context (fi_create .. fi_destroy)."""

    def __init__(self, layers: int, B: int, D: int, L: int, filters):
        self.layers, self.B, self.D, self.L = layers, B, D, L
        lib = get_lib()
        h = lib.fi_create(layers, B, D, L, _ptr(filters))
        if not h:
            raise FiError(FI_EINVAL, last_error())
        self._h = h
        self._lib = lib  # kept for close(), which may run during interpreter shutdown

    def close(self):
        if getattr(self, "_h", None):
            self._lib.fi_destroy(self._h)
            self._h = None

    __del__ = close

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def step(self, x_t, y_t):
        _check(get_lib().fi_step(self._h, _ptr(x_t), _ptr(y_t)))

    def generate(self, x0, steps: int, out):
        _check(get_lib().fi_generate(self._h, _ptr(x0), steps, _ptr(out)))

    def forward(self, x, steps: int, y):
        _check(get_lib().fi_forward(self._h, _ptr(x), steps, _ptr(y)))

    def prefill(self, x, p: int, y):
        """Fold a p-token prompt in with one FFT convolution per layer: see fi_prefill."""
        _check(get_lib().fi_prefill(self._h, _ptr(x), p, _ptr(y)))

    def reset(self):
        _check(get_lib().fi_reset(self._h))

    def read_layer(self, layer: int, t0: int, t1: int, dst):
        _check(get_lib().fi_read_layer(self._h, layer, t0, t1, _ptr(dst)))

    def set_stream(self, stream_handle: int):
        _check(get_lib().fi_set_stream(self._h, stream_handle))

    def set_path(self, path: int):
        _check(get_lib().fi_set_path(self._h, path))

    def set_graphs(self, on: bool):
        _check(get_lib().fi_set_graphs(self._h, int(bool(on))))

    def set_tau(self, q: int, impl: int):
        _check(get_lib().fi_set_tau(self._h, q, impl))

    def set_trace(self, on: bool):
        _check(get_lib().fi_set_trace(self._h, int(bool(on))))

    def trace(self, per_block_size: bool = False):
        """{class name: (launches, total_us, max_us)} of the last traced run; with
        per_block_size also {q: (launches, total_us)} of the block launches."""
        tr = fi_trace()
        _check(get_lib().fi_trace_read(self._h, ctypes.byref(tr)))
        cls = {KERNEL_CLASS_NAMES[k]: (tr.launches[k], tr.total_us[k], tr.max_us[k])
               for k in range(FI_K_CLASSES) if tr.launches[k]}
        if not per_block_size:
            return cls
        return cls, {q: (tr.block_launches[q], tr.block_us[q]) for q in range(32) if tr.block_launches[q]}

    def trace_launches(self):
        """(cls, q, us) numpy arrays of every launch of the last traced run, in issue order."""
        import numpy as np
        lib = get_lib()
        n = lib.fi_trace_launches(self._h, 0, None, None, None)
        if n < 0:
            _check(n)
        cls = np.empty(max(n, 1), np.int32)
        q = np.empty(max(n, 1), np.int32)
        us = np.empty(max(n, 1), np.float32)
        got = lib.fi_trace_launches(self._h, n, cls.ctypes.data, q.ctypes.data, us.ctypes.data)
        if got < 0:
            _check(got)
        return cls[:n], q[:n], us[:n]

    def info(self) -> fi_info:
        inf = fi_info()
        _check(get_lib().fi_get_info(self._h, ctypes.byref(inf)))
        return inf

    def schedule(self, n: int):
        vals = [ctypes.c_int() for _ in range(5)]
        _check(get_lib().fi_debug_schedule(self._h, n, *[ctypes.byref(v) for v in vals]))
        U, impl, src_lo, dst_lo, dst_hi = (v.value for v in vals)
        return dict(U=U, impl=impl, src_lo=src_lo, dst_lo=dst_lo, dst_hi=dst_hi)


def _iptr(a):
    """Address of a contiguous int32 torch tensor / numpy array (None -> NULL)."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        assert a.is_contiguous() and str(a.dtype) == "torch.int32", "int32 contiguous tensor expected"
        return a.data_ptr()
    import numpy as np
    assert isinstance(a, np.ndarray) and a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data


class LanguageModel:
    """The Hyena-like model around the mixer (fi_lm_create .. fi_lm_destroy); weights as
    float32 arrays (bf16 values for the GEMM weights), per layer stacked: see fi.h."""

    def __init__(self, layers, B, D, L, V, E, W_lm, W_in, conv, W1, W2, filters):
        self.layers, self.B, self.D, self.L, self.V = layers, B, D, L, V
        lib = get_lib()
        h = lib.fi_lm_create(layers, B, D, L, V, *(_ptr(a) for a in (E, W_lm, W_in, conv, W1, W2, filters)))
        if not h:
            raise FiError(FI_EINVAL, last_error())
        self._h = h
        self._lib = lib

    def close(self):
        if getattr(self, "_h", None):
            self._lib.fi_lm_destroy(self._h)
            self._h = None

    __del__ = close

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def reset(self):
        _check(get_lib().fi_lm_reset(self._h))

    def forward(self, tokens, steps, logits, next_tokens):
        _check(get_lib().fi_lm_forward(self._h, _iptr(tokens), steps, _ptr(logits), _iptr(next_tokens)))

    def generate(self, tok0, steps, next_tokens):
        _check(get_lib().fi_lm_generate(self._h, _iptr(tok0), steps, _iptr(next_tokens)))

    def set_trace(self, on: bool):
        _check(get_lib().fi_lm_set_trace(self._h, int(bool(on))))

    def set_graphs(self, on: bool):
        _check(get_lib().fi_lm_set_graphs(self._h, int(bool(on))))

    def split(self):
        """(mixer_us, total_us) of the last traced call."""
        a, b = ctypes.c_double(), ctypes.c_double()
        _check(get_lib().fi_lm_split(self._h, ctypes.byref(a), ctypes.byref(b)))
        return a.value, b.value


class DataDependentConvolution:
    """The long convolution with a filter that arrives online with the data
    (fi_dd_create .. fi_dd_destroy): G channels, y_t = sum_{i+j=t} rho_i x_j, both x_t
    and rho_t given at step t.  Arrays are float32 [steps][G], host or device."""

    def __init__(self, G: int, L: int):
        self.G, self.L = G, L
        lib = get_lib()
        h = lib.fi_dd_create(G, L)
        if not h:
            raise FiError(FI_EINVAL, last_error())
        self._h = h
        self._lib = lib

    def close(self):
        if getattr(self, "_h", None):
            self._lib.fi_dd_destroy(self._h)
            self._h = None

    __del__ = close

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def reset(self):
        _check(get_lib().fi_dd_reset(self._h))

    def set_tau(self, q: int, impl: int):
        _check(get_lib().fi_dd_set_tau(self._h, q, impl))

    def forward(self, x, rho, steps, y):
        _check(get_lib().fi_dd_forward(self._h, _ptr(x), _ptr(rho), steps, _ptr(y)))


def tau(impl: int, U: int, blocks, taps, out, accumulate: bool = False):
    """Stand-alone tau over independent blocks (device arrays): see fi_tau in fi.h."""
    count = blocks.shape[0]
    ldt = taps.shape[1]
    _check(get_lib().fi_tau(impl, U, count, _ptr(blocks), _ptr(taps), ldt, _ptr(out), int(bool(accumulate))))


def tau_fft_noalloc(U: int, blocks, taps, out, accumulate: bool = False):
    """FFT tau without device allocations (fixed library scratch): see
    fi_tau_fft_noalloc in fi.h."""
    count = blocks.shape[0]
    ldt = taps.shape[1]
    _check(get_lib().fi_tau_fft_noalloc(U, count, _ptr(blocks), _ptr(taps), ldt, _ptr(out),
                                        int(bool(accumulate))))

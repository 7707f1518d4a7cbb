"""Plain fp64 CPU oracle for the Flash Inference mixer stack (ctypes over oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path (the
CUDA library ``long_convolution_sequence_b200``) never imports it, and this
package never imports the product path: the two share no code.  The only thing
both sides consume is the seeded input generator module
``long_convolution_sequence_b200.synth``, which holds none of the method's
arithmetic.

Every function cites the section of the web summary of arXiv 2410.12982
("Flash Inference: Near Linear Time Inference for Long Convolution Sequence
Models and Beyond") that it follows; see ``oracle.c`` for the readings taken
where the pages are silent.

Parity status: every function here is pinned by a CPU test against numpy /
closed forms / brute force (tests/test_oracle_pins.py, tests/test_schedule.py);
none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB = _HERE / "liboracle.so"

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> Path:
    """Compile oracle.c into liboracle.so with gcc (OpenMP, -O2, no fast-math)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(".so.tmp%d" % os.getpid())
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-ffp-contract=off", str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(_LIB)
    return _lib


def load(path):
    """Open a compiled oracle library and declare its C signatures."""
    L = ctypes.CDLL(str(path))
    i64 = ctypes.c_int64
    L.orc_num_threads.restype = ctypes.c_int
    L.orc_causal_conv.argtypes = [i64, _f64p, _f64p, _f64p]
    L.orc_causal_conv_batch.argtypes = [i64, i64, i64, _f32p, _f32p, _f64p]
    L.orc_conv_at.argtypes = [i64, ctypes.c_void_p, ctypes.c_void_p, i64]
    L.orc_conv_at.restype = ctypes.c_double
    L.orc_stack.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, i64, i64, _f32p,
                            ctypes.c_int, _f32p, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_int]
    L.orc_stack.restype = ctypes.c_int
    L.orc_schedule.argtypes = [i64] + [_i64p] * 6
    L.orc_schedule.restype = i64
    L.orc_tau.argtypes = [i64, i64, _f32p, i64, _f32p, _f64p]
    L.orc_relaxed_stack.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, i64, i64,
                                    _f32p, ctypes.c_int, _f32p, ctypes.c_void_p]
    L.orc_relaxed_stack.restype = ctypes.c_int
    L.orc_fft.argtypes = [i64, _f64p, _f64p, ctypes.c_int]
    L.orc_fft.restype = ctypes.c_int
    L.orc_fft_conv.argtypes = [i64, _f64p, _f64p, _f64p]
    L.orc_fft_conv.restype = ctypes.c_int
    L.orc_filter_spectrum.argtypes = [i64, i64, _f32p, i64, _f64p, _f64p]
    L.orc_filter_spectrum.restype = ctypes.c_int
    return L


def num_threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS or all cores)."""
    return int(lib().orc_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# -- [Aufgabendefinition] / [Drei Berechnungsstrategien]: lazy causal convolution --
def causal_conv(h, y):
    """z_t = sum_{s<=t} h[t-s] y[s] for one sequence (fp64, lazy)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    h = np.ascontiguousarray(h[: len(y)], dtype=np.float64)
    z = np.empty_like(y)
    lib().orc_causal_conv(len(y), h, y, z)
    return z


def causal_conv_batch(h, y):
    """Rows of y [C][T] convolved with rows of h [C][>=T]; returns fp64 [C][T]."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    h = np.ascontiguousarray(h, dtype=np.float32)
    C, T = y.shape
    assert h.shape[0] == C and h.shape[1] >= T
    z = np.empty((C, T), dtype=np.float64)
    lib().orc_causal_conv_batch(C, T, h.shape[1], h, y, z)
    return z


def conv_at(t, h_row, y_col):
    """One sampled output z_t = sum_{s<=t} h[t-s] y[s]; y_col may be strided float32."""
    h_row = np.asarray(h_row)
    assert h_row.dtype == np.float32 and h_row.flags.c_contiguous and len(h_row) > t
    assert y_col.dtype == np.float32 and y_col.strides[0] % 4 == 0 and len(y_col) > t
    return float(lib().orc_conv_at(int(t), h_row.ctypes.data, y_col.ctypes.data,
                                   y_col.strides[0] // 4))


# -- [LCSM-Inferenz-Algorithmus (Algorithmus 2)], evaluated lazily ----------------
def stack(h, x, T=None, closed_loop=False, want=("y_last",), fp32=False):
    """The mixer stack with tanh blocks and tanh sampler, by its plain definition.

    h: float32 [M][D][>=T].  Teacher-forced: x float32 [T][B][D].  Closed loop:
    x float32 [B][D] (= x_0) and T given.  Returns a dict with the requested keys:
    "y_last" [T][B][D], "y_all" [M][T][B][D], "a_all" [M+1][T][B][D] (fp64).
    """
    h = np.ascontiguousarray(h, dtype=np.float32)
    M, D, ldh = h.shape
    x = np.ascontiguousarray(x, dtype=np.float32)
    if closed_loop:
        B = x.shape[0]
        assert x.shape == (B, D) and T is not None
    else:
        T = x.shape[0] if T is None else T
        B = x.shape[1]
        assert x.shape == (T, B, D)
    out = {}
    if "y_last" in want:
        out["y_last"] = np.empty((T, B, D), np.float64)
    if "y_all" in want:
        out["y_all"] = np.empty((M, T, B, D), np.float64)
    if "a_all" in want:
        out["a_all"] = np.empty((M + 1, T, B, D), np.float64)
    rc = lib().orc_stack(M, B, D, T, ldh, h, int(bool(closed_loop)), x,
                         _ptr(out.get("y_all")), _ptr(out.get("y_last")),
                         _ptr(out.get("a_all")), int(bool(fp32)))
    if rc != 0:
        raise RuntimeError("orc_stack failed: %d" % rc)
    return out


def relaxed_stack(h, x, T=None, closed_loop=False):
    """Algorithm 2 simulated on the CPU with direct tau; returns y_all [M][T][B][D]."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    M, D, ldh = h.shape
    x = np.ascontiguousarray(x, dtype=np.float32)
    if closed_loop:
        B = x.shape[0]
    else:
        T = x.shape[0]
        B = x.shape[1]
    y = np.empty((M, T, B, D), np.float64)
    rc = lib().orc_relaxed_stack(M, B, D, T, ldh, h, int(bool(closed_loop)), x, _ptr(y))
    if rc != 0:
        raise RuntimeError("orc_relaxed_stack failed: %d" % rc)
    return y


# -- [Kachelung-Strategie (Algorithmus 1)] schedule -------------------------------
def schedule(L):
    """Rows (n, U, src_lo, src_hi, dst_lo, dst_hi) for n = 1..L-1, int64 [L-1][6]."""
    k = max(L - 1, 0)
    cols = [np.zeros(max(k, 1), np.int64) for _ in range(6)]
    got = lib().orc_schedule(L, *cols)
    assert got == k
    return np.stack([c[:k] for c in cols], axis=1)


# -- [Beitrags-Aggregations-Definition] tau, directly ------------------------------
def tau(blocks, taps):
    """blocks [count][U], taps [count][>=2U] -> out[count][U] (fp64),
    out[i][r] = sum_j blocks[i][j] * taps[i][U + r - j]."""
    blocks = np.ascontiguousarray(blocks, dtype=np.float32)
    taps = np.ascontiguousarray(taps, dtype=np.float32)
    count, U = blocks.shape
    assert taps.shape[0] == count and taps.shape[1] >= 2 * U
    out = np.empty((count, U), np.float64)
    lib().orc_tau(U, count, blocks, taps.shape[1], taps, out)
    return out


# -- own fp64 FFT and the Lemma 1 route ---------------------------------------------
def fft(x, inverse=False):
    """Own radix-2 fp64 DFT (unnormalised in both directions)."""
    x = np.asarray(x, dtype=np.complex128)
    re = np.ascontiguousarray(x.real)
    im = np.ascontiguousarray(x.imag)
    rc = lib().orc_fft(len(x), re, im, 1 if inverse else -1)
    if rc != 0:
        raise ValueError("length must be a power of two")
    return re + 1j * im


def fft_conv(h, y):
    """Causal convolution via a zero-padded FFT of the whole sequence (fp64)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    h = np.ascontiguousarray(h[: len(y)], dtype=np.float64)
    z = np.empty_like(y)
    lib().orc_fft_conv(len(y), h, y, z)
    return z


def filter_spectrum(taps, U):
    """[Speicheroptimierung] FFT precompute: DFT_{2U} of taps[:, :2U], bins 0..U."""
    taps = np.ascontiguousarray(taps, dtype=np.float32)
    count = taps.shape[0]
    assert taps.shape[1] >= 2 * U
    re = np.empty((count, U + 1), np.float64)
    im = np.empty((count, U + 1), np.float64)
    lib().orc_filter_spectrum(U, count, taps, taps.shape[1], re, im)
    return re + 1j * im

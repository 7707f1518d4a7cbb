"""CPU-side checks of the C-ABI library: it loads without a GPU, exports every
entry point include/fi.h declares, the binding declares the same set, and the
host-side argument validation answers before any device work."""
import ctypes
import re
from pathlib import Path

import pytest

import long_convolution_sequence_b200 as fi
from long_convolution_sequence_b200 import build as fibuild

HEADER = Path(__file__).resolve().parent.parent / "include" / "fi.h"


@pytest.fixture(scope="module")
def lib():
    fibuild.build()
    return fi.get_lib()


def declared():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(fi_[a-z_]+)\s*\(", text))


def test_header_declares_the_boundary():
    names = declared()
    for core in ("fi_create", "fi_step", "fi_generate", "fi_destroy"):
        assert core in names
    assert names == set(fi.SIGNATURES), names ^ set(fi.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    for name in declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_error_strings(lib):
    assert b"sm_100a" in lib.fi_version()
    assert isinstance(lib.fi_last_error(), bytes)


@pytest.mark.parametrize("args", [
    (0, 1, 1, 8), (1, 0, 1, 8), (1, 1, 0, 8), (1, 1, 1, 12), (1, 1, 1, 1), (1, 1, 1, 0),
])
def test_create_rejects_bad_shapes_before_device_work(lib, args):
    dummy = (ctypes.c_float * 16)()
    assert not lib.fi_create(*args, ctypes.addressof(dummy))
    assert b"L a power of two" in lib.fi_last_error()


def test_create_rejects_null_filters(lib):
    assert not lib.fi_create(1, 1, 1, 8, None)
    assert fi.last_error()


def test_calls_on_null_context_report_state_error(lib):
    buf = (ctypes.c_float * 4)()
    p = ctypes.addressof(buf)
    assert lib.fi_step(None, p, p) == fi.FI_ESTATE
    assert lib.fi_generate(None, p, 1, p) == fi.FI_ESTATE
    assert lib.fi_forward(None, p, 1, p) == fi.FI_ESTATE
    assert lib.fi_prefill(None, p, 8, p) == fi.FI_ESTATE
    assert lib.fi_reset(None) == fi.FI_ESTATE
    assert lib.fi_read_layer(None, 0, 0, 0, p) == fi.FI_ESTATE
    assert lib.fi_set_path(None, 0) == fi.FI_ESTATE
    assert lib.fi_set_path(None, fi.FI_PATH_LAZY) == fi.FI_ESTATE
    assert lib.fi_set_tau(None, 0, 1) == fi.FI_ESTATE
    assert lib.fi_get_info(None, ctypes.byref(fi.fi_info())) == fi.FI_ESTATE
    assert b"context" in lib.fi_last_error()
    lib.fi_destroy(None)  # accepted


def test_tau_rejects_bad_arguments(lib):
    buf = (ctypes.c_float * 64)()
    p = ctypes.addressof(buf)
    assert lib.fi_tau(fi.FI_TAU_DIRECT, 3, 1, p, p, 8, p, 0) == fi.FI_EINVAL   # U not a power of two
    assert lib.fi_tau(fi.FI_TAU_DIRECT, 4, 1, p, p, 7, p, 0) == fi.FI_EINVAL   # ldt < 2U
    assert lib.fi_tau(fi.FI_TAU_FFT, 4, 1, p, p, 8, p, 0) == fi.FI_EINVAL      # FFT needs U >= 8
    assert lib.fi_tau(7, 8, 1, p, p, 16, p, 0) == fi.FI_EINVAL                 # unknown impl
    assert lib.fi_tau(fi.FI_TAU_DIRECT, 8, 0, p, p, 16, p, 0) == fi.FI_EINVAL  # empty


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(fi, "_LIB_PATH", tmp_path / "missing.so")
    monkeypatch.setattr(fi, "_lib", None)
    with pytest.raises(ImportError):
        fi.get_lib()

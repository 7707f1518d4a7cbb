"""Pins for the CPU oracle: each check ties it to something other than itself
(numpy library routines, closed forms, brute force), chosen so that a dropped
term, a wrong index or sign, or a transposed operand in the oracle fails one.

Definitions followed (web summary of arXiv 2410.12982, "Flash Inference"):
sections "Aufgabendefinition", "LCSM-spezifische Definition",
"Beitrags-Aggregations-Definition", "LCSM-Inferenz-Algorithmus (Algorithmus 2)",
"Zirkulaere Faltungs-Trick", "Speicheroptimierung" (FFT precompute).
"""
import math

import numpy as np
import pytest

import oracle


class _Rng:
    """Per-test deterministic draws (independent of test order)."""

    def __getattr__(self, name):
        import os
        import zlib
        key = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        if key != self.__dict__.get("_key"):
            self.__dict__["_key"] = key
            self.__dict__["_g"] = np.random.default_rng(zlib.crc32(key.encode()))
        return getattr(self.__dict__["_g"], name)


RNG = _Rng()


# ---------------------------------------------------------------- single conv
@pytest.mark.parametrize("T", [1, 2, 3, 7, 64, 100])
def test_causal_conv_equals_numpy_convolve(T):
    h = RNG.standard_normal(T + 5)
    y = RNG.standard_normal(T)
    ref = np.convolve(y, h[:T])[:T]
    np.testing.assert_allclose(oracle.causal_conv(h, y), ref, rtol=0, atol=1e-12)


def test_conv_is_not_symmetric_in_lag():
    # a transposed operand (h[s] * y[t-s] vs h[t-s] * y[s] is symmetric, but a
    # reversed filter h[s-t] is not): a decaying filter must weight recent inputs most
    T = 16
    h = 0.5 ** np.arange(T)
    y = np.zeros(T)
    y[3] = 1.0
    z = oracle.causal_conv(h, y)
    assert np.all(z[:3] == 0)
    np.testing.assert_allclose(z[3:], 0.5 ** np.arange(T - 3), atol=0)


@pytest.mark.parametrize("N", [1, 2, 4, 8, 64, 1024])
def test_own_fft_equals_numpy_fft(N):
    x = RNG.standard_normal(N) + 1j * RNG.standard_normal(N)
    np.testing.assert_allclose(oracle.fft(x), np.fft.fft(x), rtol=0, atol=1e-10 * N)
    np.testing.assert_allclose(oracle.fft(x, inverse=True), np.fft.ifft(x) * N,
                               rtol=0, atol=1e-10 * N)


@pytest.mark.parametrize("T", [1, 5, 33, 128, 300])
def test_fft_conv_equals_lazy_and_numpy(T):
    h = RNG.standard_normal(T)
    y = RNG.standard_normal(T)
    ref = np.convolve(y, h)[:T]
    np.testing.assert_allclose(oracle.fft_conv(h, y), ref, atol=1e-10)
    np.testing.assert_allclose(oracle.causal_conv(h, y), ref, atol=1e-11)


def test_closed_form_delta_and_shift():
    T = 50
    y = RNG.standard_normal(T)
    d0 = np.zeros(T); d0[0] = 1.0
    np.testing.assert_array_equal(oracle.causal_conv(d0, y), y)
    for k in (1, 7, 49):
        dk = np.zeros(T); dk[k] = 1.0
        want = np.concatenate([np.zeros(k), y[: T - k]])
        np.testing.assert_array_equal(oracle.causal_conv(dk, y), want)


def test_closed_form_geometric_filter_is_first_order_recurrence():
    # h_k = g r^k  =>  z_t = r z_{t-1} + g y_t (the LTI-SSM view of a filter)
    T, r, g = 400, 0.97, 0.3
    h = g * r ** np.arange(T)
    y = RNG.standard_normal(T)
    z = np.empty(T)
    prev = 0.0
    for t in range(T):
        prev = r * prev + g * y[t]
        z[t] = prev
    np.testing.assert_allclose(oracle.causal_conv(h, y), z, atol=1e-11)


def test_closed_form_constant_filter_is_prefix_sum():
    T = 257
    y = RNG.standard_normal(T)
    np.testing.assert_allclose(oracle.causal_conv(np.ones(T), y), np.cumsum(y), atol=1e-11)


def test_batch_conv_and_sampled_conv_agree_with_numpy():
    C, T = 5, 70
    h = RNG.standard_normal((C, T + 3)).astype(np.float32)
    y = RNG.standard_normal((C, T)).astype(np.float32)
    z = oracle.causal_conv_batch(h, y)
    for c in range(C):
        ref = np.convolve(y[c].astype(np.float64), h[c, :T].astype(np.float64))[:T]
        np.testing.assert_allclose(z[c], ref, atol=1e-11)
        for t in (0, 1, T // 2, T - 1):
            assert abs(oracle.conv_at(t, h[c], y[c]) - ref[t]) < 1e-11
    # strided column access (time-major [T][C] layout)
    yt = np.ascontiguousarray(y.T)
    for c in range(C):
        assert abs(oracle.conv_at(T - 1, h[c], yt[:, c]) - z[c, T - 1]) < 1e-11


# ---------------------------------------------------------------- the stack
def _np_stack(h, x, closed_loop, T=None):
    """Independent restatement with numpy.convolve, layer by layer (teacher) or
    token by token (closed loop)."""
    M, D, _ = h.shape
    h = h.astype(np.float64)
    if not closed_loop:
        T, B, _ = x.shape
        a = x.astype(np.float64)
        ys = []
        for l in range(M):
            y = np.empty((T, B, D))
            for b in range(B):
                for c in range(D):
                    y[:, b, c] = np.convolve(a[:, b, c], h[l, c, :T])[:T]
            ys.append(y)
            a = np.tanh(y)
        return np.stack(ys)
    B = x.shape[0]
    seq = np.zeros((M + 1, T, B, D))
    ys = np.zeros((M, T, B, D))
    for t in range(T):
        seq[0, t] = x if t == 0 else seq[M, t - 1]
        for l in range(M):
            # y_t = sum_s h[t-s] a_s, via a reversed-filter dot product
            y = np.einsum("sbc,cs->bc", seq[l, : t + 1], h[l, :, t::-1])
            ys[l, t] = y
            seq[l + 1, t] = np.tanh(y)
    return ys


@pytest.mark.parametrize("closed", [False, True])
def test_stack_equals_numpy_restatement(closed):
    M, B, D, T = 3, 2, 3, 40
    h = (RNG.standard_normal((M, D, T + 2)) * 0.4).astype(np.float32)
    if closed:
        x = RNG.standard_normal((B, D)).astype(np.float32)
        got = oracle.stack(h, x, T=T, closed_loop=True, want=("y_all", "y_last"))
        ref = _np_stack(h, x, True, T)
    else:
        x = RNG.standard_normal((T, B, D)).astype(np.float32)
        got = oracle.stack(h, x, want=("y_all", "y_last"))
        ref = _np_stack(h, x, False)
    np.testing.assert_allclose(got["y_all"], ref, atol=1e-11)
    np.testing.assert_array_equal(got["y_last"], got["y_all"][-1])


def test_stack_delta_filters_closed_form():
    # h^l = g_l * delta_0  =>  y^1_t = g_1 a^0_t, a^l = tanh(y^l): a scalar map per channel
    M, B, D, T = 4, 2, 3, 30
    g = np.array([1.3, -0.7, 2.1, 0.9], np.float32)
    h = np.zeros((M, D, T), np.float32)
    h[:, :, 0] = g[:, None]
    x0 = RNG.standard_normal((B, D)).astype(np.float32)
    got = oracle.stack(h, x0, T=T, closed_loop=True, want=("y_all",))["y_all"]
    for b in range(B):
        for c in range(D):
            a = float(x0[b, c])
            for t in range(T):
                for l in range(M):
                    y = float(g[l]) * a
                    assert abs(got[l, t, b, c] - y) < 1e-12
                    a = math.tanh(y)


def test_stack_geometric_filters_recurrence_teacher_and_closed():
    # h^l_c[k] = g r^k  =>  y^l_t = r y^l_{t-1} + g a^{l-1}_t for every layer
    M, B, D, T = 3, 1, 4, 300
    r = RNG.uniform(0.5, 0.999, size=(M, D))
    gain = RNG.uniform(-1.5, 1.5, size=(M, D))
    k = np.arange(T)
    h = (gain[:, :, None] * r[:, :, None] ** k).astype(np.float32)
    hd = h.astype(np.float64)
    # the recurrence holds exactly for the real-valued filter g r^k; the float32
    # taps the oracle receives differ from it by at most 2^-24 |h_k| each
    for closed in (False, True):
        if closed:
            x0 = RNG.standard_normal((B, D)).astype(np.float32)
            got = oracle.stack(h, x0, T=T, closed_loop=True, want=("y_all",))["y_all"]
        else:
            x = RNG.standard_normal((T, B, D)).astype(np.float32)
            got = oracle.stack(h, x, want=("y_all",))["y_all"]
        for c in range(D):
            state = np.zeros(M)
            a_prev_last = None
            for t in range(T):
                a = (float(x0[0, c]) if t == 0 else a_prev_last) if closed else float(x[t, 0, c])
                for l in range(M):
                    state[l] = r[l, c] * state[l] + gain[l, c] * a
                    bound = 2.0 ** -24 * np.abs(hd[l, c, : t + 1]).sum() * 1.01 + 1e-12
                    assert abs(got[l, t, 0, c] - state[l]) < bound
                    a = math.tanh(got[l, t, 0, c])
                a_prev_last = a


@pytest.mark.parametrize("closed", [False, True])
def test_relaxed_tiling_equals_lazy(closed):
    # Algorithm 2 (relaxed tiling, direct tau) reproduces the lazy definition
    M, B, D, T = 3, 2, 2, 64
    h = (RNG.standard_normal((M, D, T)) * 0.3).astype(np.float32)
    if closed:
        x = RNG.standard_normal((B, D)).astype(np.float32)
        lazy = oracle.stack(h, x, T=T, closed_loop=True, want=("y_all",))["y_all"]
        rel = oracle.relaxed_stack(h, x, T=T, closed_loop=True)
    else:
        x = RNG.standard_normal((T, B, D)).astype(np.float32)
        lazy = oracle.stack(h, x, want=("y_all",))["y_all"]
        rel = oracle.relaxed_stack(h, x)
    np.testing.assert_allclose(rel, lazy, atol=1e-11)


def test_fp32_variant_tracks_fp64_on_short_runs():
    M, B, D, T = 2, 1, 3, 50
    h = (RNG.standard_normal((M, D, T)) * 0.2).astype(np.float32)
    x = RNG.standard_normal((T, B, D)).astype(np.float32)
    a = oracle.stack(h, x, want=("y_all",))["y_all"]
    b = oracle.stack(h, x, want=("y_all",), fp32=True)["y_all"]
    np.testing.assert_allclose(a, b, atol=1e-5)
    assert np.any(a != b)  # it really is a float evaluation


# ---------------------------------------------------------------- tau and spectra
@pytest.mark.parametrize("U", [1, 2, 4, 8, 32, 64])
def test_tau_is_the_window_of_a_2U_circular_convolution(U):
    # "Zirkulaere Faltungs-Trick": outputs [U, 2U-1] of the 2U-point circular
    # convolution of [block, 0^U] with rho_0..rho_{2U-1} are the gray block.
    cnt = 3
    blocks = RNG.standard_normal((cnt, U)).astype(np.float32)
    taps = RNG.standard_normal((cnt, 2 * U + 3)).astype(np.float32)
    got = oracle.tau(blocks, taps)
    pad = np.concatenate([blocks.astype(np.float64), np.zeros((cnt, U))], axis=1)
    circ = np.fft.ifft(np.fft.fft(pad, axis=1) * np.fft.fft(taps[:, : 2 * U].astype(np.float64), axis=1), axis=1).real
    np.testing.assert_allclose(got, circ[:, U:], atol=1e-10)


def test_tau_is_the_definition_on_the_sequence():
    # tau(y, [n-U, n-1], rho, [n, n+U-1]) equals the contribution of that block of a
    # full sequence to later outputs (numpy.convolve of the masked sequence)
    T, U, n = 64, 8, 24
    y = RNG.standard_normal(T)
    rho = RNG.standard_normal(T)
    masked = np.zeros(T); masked[n - U:n] = y[n - U:n]
    full = np.convolve(masked, rho)[:T]
    got = oracle.tau(y[None, n - U:n].astype(np.float32), rho[None].astype(np.float32))
    np.testing.assert_allclose(got[0], np.convolve(masked.astype(np.float32).astype(np.float64),
                                                   rho.astype(np.float32).astype(np.float64))[n:n + U],
                               atol=1e-11)
    np.testing.assert_allclose(got[0], full[n:n + U], atol=1e-5)


@pytest.mark.parametrize("U", [1, 2, 16, 128])
def test_filter_spectrum_equals_numpy_rfft(U):
    taps = RNG.standard_normal((4, 2 * U + 1)).astype(np.float32)
    got = oracle.filter_spectrum(taps, U)
    ref = np.fft.rfft(taps[:, : 2 * U].astype(np.float64), axis=1)
    np.testing.assert_allclose(got, ref, atol=1e-10 * U)

"""The data-dependent filter's window evaluation, restated on the CPU and checked by
brute force against the tiling (oracle/dd.py).

The window kernel relies on two facts about an aligned window [kW, kW + W) with
kW >= W: (1) the blocks released inside it (kW < n < kW + W) read and write only the
window, and together add, for every pair of window positions j < t,
x_j rho_{t-j} + rho_j x_{t-j}, with lags t - j < W (prefix indices); (2) so their
running-sum updates can be skipped (they only feed positions of the same window),
and y_t = acc[t] + rho_0 x_t + rho_t x_0 + that sum, from the running sums of the
blocks released at or before kW.  Here the tiling's blocks are replayed with the
in-window ones left out for every window that is evaluated whole, and every output
must equal the causal convolution."""
import numpy as np
import pytest

import oracle
from oracle import dd


def window_run(x, rho, W, whole):
    """y by the tiling, except that a window at kW >= W with `whole(kW)` true is
    evaluated by the window formula and its in-window blocks are not applied."""
    T, G = x.shape
    acc = np.zeros((T, G))
    y = np.zeros((T, G))
    t = 0
    while t < T:
        kW = (t // W) * W
        if t == kW and kW >= W and kW + W <= T and whole(kW):
            for s in range(W):
                tt = kW + s
                v = acc[tt] + rho[0] * x[tt] + rho[tt] * x[0]
                for j in range(kW, tt):
                    v = v + x[j] * rho[tt - j] + rho[j] * x[tt - j]
                y[tt] = v
            t = kW + W
            n = t
        else:
            y[t] = acc[t] + rho[0] * x[t] + (rho[t] * x[0] if t > 0 else 0.0)
            n = t + 1
            t += 1
        if n >= T:
            continue
        # the blocks released after token n (the window's own only at its end)
        for kind in ("x", "rho"):
            if kind == "rho" and dd.is_pow2(n):
                continue
            for i, j in dd.block_pairs(n, kind, n & -n):
                if i + j < T:
                    acc[i + j] += rho[i] * x[j]
    return y


@pytest.mark.parametrize("T,W", [(64, 8), (128, 16), (96, 8), (256, 32)])
@pytest.mark.parametrize("pattern", ["all", "none", "alternate"])
def test_window_formula_equals_the_causal_convolution(T, W, pattern):
    rng = np.random.default_rng(T + W)
    G = 3
    x = rng.standard_normal((T, G))
    rho = rng.standard_normal((T, G)) / np.sqrt(np.arange(1, T + 1))[:, None]
    whole = {"all": lambda kW: True, "none": lambda kW: False,
             "alternate": lambda kW: (kW // W) % 2 == 1}[pattern]
    y = window_run(x, rho, W, whole)
    for g in range(G):
        ref = oracle.causal_conv(rho[:, g].copy(), x[:, g].copy())
        np.testing.assert_allclose(y[:, g], ref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("T,W", [(64, 8), (256, 32)])
def test_in_window_blocks_stay_in_their_window(T, W):
    # every block released strictly inside an aligned window at kW >= W reads and
    # writes only window positions (its input range) and prefix indices below W (its
    # taps), and adds exactly the pairs of window positions j < t with both kinds
    for kW in range(W, T - W + 1, W):
        pairs = set()
        for n in range(kW + 1, kW + W):
            U = n & -n
            assert U < W and n - U >= kW and n + U <= kW + W
            for kind in ("x", "rho"):
                assert not dd.is_pow2(n)
                for i, j in dd.block_pairs(n, kind, U):
                    inp, lag = (j, i) if kind == "x" else (i, j)
                    assert kW <= inp < kW + W and 1 <= lag < W
                    pairs.add((kind, inp, inp + lag))
        want = {(k, j, t) for k in ("x", "rho") for t in range(kW, kW + W) for j in range(kW, t)}
        assert pairs == want

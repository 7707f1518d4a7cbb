"""Pins of the data-dependent filter's oracle (oracle/dd.py), on the CPU.

The tiling is a reading (the pages state only its cost: two convolutions of the same
size per step, twice the work); it is pinned here by what the mathematics fixes:
every product rho_i x_j with i, j >= 1 is added exactly once, by a block released
when both factors are known and before its output is due, and the online evaluation
equals the causal convolution computed by its definition (the C oracle's
causal_conv, pinned on its own in test_oracle_pins.py)."""
import numpy as np
import pytest

import oracle
from oracle import dd


@pytest.mark.parametrize("L", [2, 3, 8, 33, 64, 256])
def test_every_product_added_exactly_once_when_both_factors_are_known(L):
    count = np.zeros((L, L), np.int64)
    for n, kind, U in dd.schedule(L):
        assert U == (n & -n)
        for i, j in dd.block_pairs(n, kind, U):
            assert i >= 1 and j >= 1
            assert i < n and j < n          # both factors known after the n-th token
            assert i + j >= n               # the output is still to come
            if i + j < L:
                count[i, j] += 1
    want = np.zeros((L, L), np.int64)
    for i in range(1, L):
        for j in range(1, L - i):
            want[i, j] = 1
    np.testing.assert_array_equal(count, want)


@pytest.mark.parametrize("P", [1, 2, 4, 8, 12])
def test_two_convolutions_of_the_same_size_per_step(P):
    # one size per step; two blocks at every step but the powers of two, so of each size
    # 2^q there are 2 L / 2^(q+1) - 1 convolutions against Algorithm 1's L / 2^(q+1)
    # (the pages' factor of two, in FFT convolutions)
    L = 1 << P
    s = dd.schedule(L)
    per_step = {}
    for n, kind, U in s:
        per_step.setdefault(n, []).append((kind, U))
    for n, blocks in per_step.items():
        assert {U for _, U in blocks} == {n & -n}
        assert sorted(k for k, _ in blocks) == (["x"] if dd.is_pow2(n) else ["rho", "x"])
    fi = oracle.schedule(L)
    for q in range(P):
        U = 1 << q
        n_fi = int(np.sum(fi[:, 1] == U))
        assert n_fi == L >> (q + 1)
        assert sum(1 for _, _, u in s if u == U) == 2 * n_fi - 1


@pytest.mark.parametrize("T,G", [(1, 3), (2, 1), (37, 4), (130, 2)])
def test_online_evaluation_is_the_causal_convolution(T, G):
    rng = np.random.default_rng(T * 31 + G)
    x = rng.standard_normal((T, G))
    rho = rng.standard_normal((T, G)) / np.sqrt(np.arange(1, T + 1))[:, None]
    y = dd.run(x, rho)
    assert np.isfinite(y).all()  # no block read a value before it was known
    for g in range(G):
        ref = oracle.causal_conv(rho[:, g].copy(), x[:, g].copy())
        np.testing.assert_allclose(y[:, g], ref, rtol=1e-12, atol=1e-12)


def test_roles_of_input_and_filter_are_symmetric():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 3))
    rho = rng.standard_normal((64, 3))
    np.testing.assert_allclose(dd.run(x, rho), dd.run(rho, x), rtol=1e-12, atol=1e-12)


def test_delta_filter_and_delta_input():
    T = 50
    x = np.random.default_rng(6).standard_normal((T, 2))
    delta = np.zeros((T, 2))
    delta[0] = 1.0
    np.testing.assert_array_equal(dd.run(x, delta), x)
    np.testing.assert_array_equal(dd.run(delta, x), x)
    # a delayed delta filter delays the input
    d3 = np.zeros((T, 2))
    d3[3] = 1.0
    y = dd.run(x, d3)
    np.testing.assert_array_equal(y[3:], x[:-3])
    np.testing.assert_array_equal(y[:3], 0.0)

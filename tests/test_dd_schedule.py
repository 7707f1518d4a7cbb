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


# ----------------------------------------------------------------- the pins can fail
# Each plausible mistake is planted in a copy of oracle/dd.py's source (loaded as a
# module of its own; the oracle itself is untouched) and must break at least one pin.
DD_MUTANTS = {
    "mirror_block_at_powers_of_two": ("        if not is_pow2(n):\n            out.append((n, \"rho\", U))",
                                      "        out.append((n, \"rho\", U))"),
    "reads_unknown_tail": ("            if is_pow2(n) and lag >= U:\n                continue           # rho[U, 2U)",
                           "            if False:\n                continue           # rho[U, 2U)"),
    "run_reads_unknown_tail": ("                    if is_pow2(n) and lag >= U:\n                        continue",
                               "                    if False:\n                        continue"),
    "run_lag_off_by_one": ("                    lag = n + r - s\n", "                    lag = n + r - s - 1\n"),
    "run_drops_red_cell": ("            y[t] += rb[t] * xb[0]", "            y[t] += 0.0"),
    "run_mirror_at_powers_of_two": ("            if kind == \"rho\" and is_pow2(n):\n                continue",
                                    "            if False:\n                continue"),
}


def _planted(name):
    import importlib.util
    import sys
    import types
    from pathlib import Path
    src = Path(dd.__file__).read_text()
    old, new = DD_MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("dd_mutant_" + name)
    exec(compile(src.replace(old, new), "dd_mutant_" + name, "exec"), mod.__dict__)
    return mod


def _pins_pass(mod):
    """True if every pin above holds for the module `mod` standing in for oracle.dd."""
    global dd
    real = dd
    dd = mod
    try:
        for L in (8, 33, 64):
            test_every_product_added_exactly_once_when_both_factors_are_known(L)
        for P in (4, 8):
            test_two_convolutions_of_the_same_size_per_step(P)
        for T, G in ((37, 4), (130, 2)):
            test_online_evaluation_is_the_causal_convolution(T, G)
        test_roles_of_input_and_filter_are_symmetric()
        test_delta_filter_and_delta_input()
        return True
    except AssertionError:
        return False
    finally:
        dd = real


def test_the_unmodified_oracle_passes_the_pins():
    assert _pins_pass(dd)


@pytest.mark.parametrize("name", sorted(DD_MUTANTS))
def test_every_planted_mistake_fails_a_pin(name):
    assert not _pins_pass(_planted(name)), name

"""Which (input j, output p) contributions each window launch applies.

The window kernel splits the relaxed tiling's in-window blocks (section
"Kachelung-Strategie (Algorithmus 1)" of the Flash Inference summary) between three
roles: the chain lanes add lags 1 .. K-1 of the current position (K = 3), the helper
pairs add the rows of every lag >= K, and a launch that stops inside the window completes the
blocks it released.  This restates those decisions (a chain lag is added when its
block was released after the launch began, by the closed forms of those blocks; the
helper rows' cover ranges; the completion step) as the kernel takes them and checks,
against brute force over the tiling, that after every launch of every split of a
window each pair of a block released so far has been applied exactly once and no
other pair has."""
import functools
import itertools
import random

import pytest


def lowbit(n):
    return n & -n


def block_of(j, p):
    # the released block n (j < n <= p) whose inputs hold j and whose outputs hold p
    for n in range(j + 1, p + 1):
        U = lowbit(n)
        if n - U <= j < n <= p < n + U:
            return n
    raise AssertionError((j, p))


def cover_range(T, s0, hi):
    # lowest input (and highest input) of the blocks released in (s0, hi] covering T
    lo, n, top = -1, T, -1
    while n > s0 and n > 0:
        lon = n - lowbit(n)
        if n <= hi:
            if top < 0:
                top = n - 1
            lo = lon
        n = lon
    return lo, top


def lag_block(s, d):
    # the block holding the pair (s - d, s), d = 1, 2, 3, in closed form
    if d == 1:
        return s
    if d == 2:
        return s - 1 if s & 1 else s
    return (s, s - 1, s - 2, s - 1)[s & 3]


def launch(W, s0, s1, K):
    added = []
    for s in range(s0, s1):
        for d in range(1, K):
            if s - d >= 0 and lag_block(s, d) > s0:
                added.append((s - d, s))
        T = s + 1
        if T < W:
            lo = 0 if s0 == 0 else cover_range(T, s0, T)[0]
            added += [(j, T) for j in range(lo, T - K + 1)]  # lags >= K
    if s0 < s1 < W:
        for d in range(1, K):
            if s1 - d >= 0 and lag_block(s1, d) > s0:
                added.append((s1 - d, s1))
        for T in range(s1 + 1, W):
            lo, top = cover_range(T, s0, s1)
            if lo >= 0:
                added += [(j, T) for j in range(lo, top + 1)]
    return added


@functools.lru_cache(maxsize=None)
def blocks(W):
    return {(j, p): block_of(j, p) for p in range(W) for j in range(p)}


def check(W, splits, K):
    applied = {}
    pts = [0] + list(splits) + [W]
    for s0, s1 in zip(pts[:-1], pts[1:]):
        for pr in launch(W, s0, s1, K):
            assert 0 <= pr[0] < pr[1] < W, pr
            applied[pr] = applied.get(pr, 0) + 1
        want = {pr for pr, n in blocks(W).items() if n <= s1}
        assert all(c == 1 for c in applied.values()), (splits, s0, s1)
        assert set(applied) == want, (splits, s0, s1)


def test_lag_blocks_closed_forms():
    for s in range(3, 2048):
        for d in (1, 2, 3):
            assert lag_block(s, d) == block_of(s - d, s)


@pytest.mark.parametrize("K", [3])
@pytest.mark.parametrize("W", [32, 64])
def test_whole_window_and_every_single_split(W, K):
    check(W, [], K)
    for a in range(1, W):
        check(W, [a], K)


@pytest.mark.parametrize("K", [3])
def test_every_two_way_split(K):
    W = 32
    for a, b in itertools.combinations(range(1, W), 2):
        check(W, [a, b], K)


@pytest.mark.parametrize("K", [3])
def test_random_splits_of_the_128_window(K):
    rng = random.Random(7)
    for _ in range(40):
        check(128, sorted(rng.sample(range(1, 128), rng.randint(1, 10))), K)


# ---------------------------------------------------------------- helper-row reads
# The helper pair of one (layer, chain) item computes row T over lags 3 .. T - lo in
# lag pairs (3 + 2k, 4 + 2k), pair k = part + 2m on lane `part`, one 8-byte load per
# pair at positions (T - 4 - 2k, T - 3 - 2k).  Rows whose blocks start at window
# position 0 run whole blocks of 8 pairs and rely on 36 zero floats before each row;
# the others mask per term.  These restate the kernel's index arithmetic and check
# that every lag is taken exactly once and no read leaves the row or its padding.
PAD = 36


def helper_terms(T, lo, padded, W):
    dmax = T - lo
    K = (dmax - 1) >> 1
    terms, low = [], 0
    for part in (0, 1):
        if padded:
            nblk = (((K + 1) >> 1) + 7) >> 3
            assert 8 * nblk <= ((W - 2) // 4 + 7) // 8 * 8  # register tap pairs
            for m in range(8 * nblk):
                k = part + 2 * m
                for d, pos in ((4 + 2 * k, T - 4 - 2 * k), (3 + 2 * k, T - 3 - 2 * k)):
                    low = min(low, pos)
                    if pos >= 0 and d < W:
                        terms.append((d, pos))
                    else:  # a zero from the padding, or a zero tap past the window
                        assert pos < 0 or d >= W
        else:
            nm_me = (K - part + 1) >> 1
            last_half = (dmax & 1) == 1 and ((K - 1) & 1) == part
            for m in range(nm_me):
                k = part + 2 * m
                if not (last_half and m == nm_me - 1):
                    terms.append((4 + 2 * k, T - 4 - 2 * k))
                terms.append((3 + 2 * k, T - 3 - 2 * k))
    if not padded:
        low = min((p for _, p in terms), default=lo)
    return terms, low


@pytest.mark.parametrize("W", [32, 64, 128, 256])
def test_helper_rows_take_every_lag_once_and_stay_in_bounds(W):
    for T in range(1, W):
        for lo in range(0, T):
            for padded in ((True, False) if lo == 0 else (False,)):
                terms, low = helper_terms(T, lo, padded, W)
                assert sorted(d for d, _ in terms) == list(range(3, T - lo + 1)), (T, lo, padded)
                assert all(T - d == p for d, p in terms)
                if padded:
                    assert low >= -31 and 31 < PAD, (T, low)
                else:
                    assert low >= lo, (T, lo, low)
            # the 8-byte load of pair 0 is aligned in the row (T even) or its shifted copy
            assert ((T - 4) % 2 == 0) == (T % 2 == 0)

"""The two facts the prompt prefill (fi_prefill) rests on, checked on the CPU.

1. The causal convolution of a p-token prompt is the block tau of Lemma 1
   (section "Beitrags-Aggregations-Definition") with U >= p, the prompt as the block
   (zero past p) and the taps shifted by U: taps[m] = 0 for m < U, h[m - U] above.
2. After p tokens the tiled paths hold, at every position >= p, exactly the pairs of
   the blocks released up to p (section "Kachelung-Strategie (Algorithmus 1)"); those
   are the blocks n <= p with n + lowbit(n) > p.  The largest power of two n0 <= p is
   one of them and its outputs [n0, 2 n0) hold every other's, and replaying them in
   decreasing n never writes a position another, later replayed block reads."""
import functools

import numpy as np
import pytest

import oracle


def lowbit(n):
    return n & -n


@functools.lru_cache(maxsize=None)
def block_of(j, p):
    for n in range(j + 1, p + 1):
        U = lowbit(n)
        if n - U <= j < n <= p < n + U:
            return n
    raise AssertionError((j, p))


@pytest.mark.parametrize("p,U", [(1, 8), (5, 8), (8, 8), (13, 16), (100, 128), (128, 128)])
def test_shifted_taps_tau_is_the_causal_convolution(p, U):
    rng = np.random.default_rng(p)
    x = rng.standard_normal(p).astype(np.float32)
    h = rng.standard_normal(U).astype(np.float32)
    blocks = np.zeros((1, U), np.float32)
    blocks[0, :p] = x
    taps = np.concatenate([np.zeros(U, np.float32), h])[None, :]
    got = oracle.tau(blocks, taps)[0, :p]
    want = oracle.causal_conv(h, x)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * max(1.0, float(np.abs(want).max())))


def open_blocks(p, L):
    return [n for n in range(1, min(p, L - 1) + 1) if n + lowbit(n) > p]


@pytest.mark.parametrize("L", [64, 256])
def test_open_blocks_rebuild_the_tiled_state_after_a_prompt(L):
    for p in range(1, L + 1):
        blocks = open_blocks(p, L)
        # pairs the replay adds at positions >= p
        added = {}
        for n in blocks:
            U = lowbit(n)
            for j in range(n - U, n):
                for q in range(max(n, p), min(n + U, L)):
                    added[(j, q)] = added.get((j, q), 0) + 1
        assert all(c == 1 for c in added.values())
        want = {(j, q) for q in range(p, L) for j in range(min(p, q)) if block_of(j, q) <= p}
        assert set(added) == want, p
        if blocks:
            n0 = 1 << (p.bit_length() - 1)
            assert min(blocks) == n0
            # every replayed block writes inside [n0, 2 n0), so the activations it
            # overwrites lie in [n0, p)
            assert all(n0 <= n and n + lowbit(n) <= 2 * n0 for n in blocks)
            # decreasing n: no replayed block writes a position that a block replayed
            # after it (smaller n) reads
            for a in blocks:
                for b in blocks:
                    if b < a:
                        writes = set(range(a, a + lowbit(a)))
                        reads = set(range(b - lowbit(b), b))
                        assert not writes & reads, (p, a, b)

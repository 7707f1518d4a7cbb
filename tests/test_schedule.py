"""The relaxed tiling's schedule (Algorithm 1 of the Flash Inference summary,
section "Kachelung-Strategie (Algorithmus 1)") pinned to the counts the pages
state (golden fixture tests/golden/schedule_counts.json) and to brute-force
coverage of the contribution space."""
import json
from pathlib import Path

import numpy as np
import pytest

import oracle

GOLD = json.loads((Path(__file__).parent / "golden" / "schedule_counts.json").read_text())


@pytest.mark.parametrize("P", list(range(1, 18)))
def test_tile_histogram_proposition_1(P):
    L = 1 << P
    s = oracle.schedule(L)
    assert len(s) == L - 1  # L-1 calls per layer (Theorem 2)
    U = s[:, 1]
    for q in range(P):
        assert int(np.sum(U == (1 << q))) == 1 << (P - 1 - q)
    assert int(U.max()) == (1 << (P - 1)) if P > 1 else True


def test_fractions_printed_on_the_pages():
    P = GOLD["check_length_P"]
    s = oracle.schedule(1 << P)
    U = s[:, 1]
    frac_blocks = np.mean(U <= 4)
    assert abs(frac_blocks - GOLD["fraction_blocks_le_4"]["value"]) < 1e-4
    # "tokens that use a block of size <= 8": one block is released per token
    frac_tokens = np.mean(U <= 8)
    assert abs(frac_tokens - GOLD["fraction_tokens_block_le_8"]["value"]) < 1e-4


@pytest.mark.parametrize("L", [2, 4, 8, 32, 256])
def test_every_pair_covered_exactly_once(L):
    s = oracle.schedule(L)
    cover = np.zeros((L, L), np.int32)  # cover[src, dst]
    for n, U, slo, shi, dlo, dhi in s:
        assert slo == n - U and shi == n - 1 and dlo == n
        assert 0 <= slo <= shi < dlo <= dhi <= L - 1
        cover[slo:shi + 1, dlo:dhi + 1] += 1
    for src in range(L):
        for dst in range(L):
            want = 1 if src < dst else 0  # the diagonal is the red cell
            assert cover[src, dst] == want, (src, dst)


def test_lowbit_values():
    s = oracle.schedule(64)
    for n, U, *_ in s:
        assert n % U == 0 and (n // U) % 2 == 1

"""Plain fp64 CPU oracle of the long convolution with a data-dependent filter.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it; the CUDA
path never imports it and it imports nothing of the CUDA path.

What the pages state.  The Flash Inference summary (section "Technische Innovationen",
item 4 "Datenabhaengige Filter-Erweiterung") says that a modified tiling supports a
filter rho that depends on the data, at twice the computation; the rebuttal (its answer
on data-dependent filters) adds that this tiling performs two FFT calls of the same
size at each step instead of one.  The tiling itself (the appendix that holds it) is
not on the pages.

Reading taken here.  Both sequences arrive online: at step t the input x_t and the
filter value rho_t become known together, and the output is the causal convolution

    y_t = sum_{i + j = t} rho_i x_j            (i, j >= 0),

which is the definition a fixed filter also has (``oracle.causal_conv(rho, x)``); only
what is known when differs.  Pairs (i, j) with i = 0 or j = 0 are red cells, added at
step t itself (rho_0 x_t + rho_t x_0).  The other pairs are tiled by blocks released
after the n-th token (indices < n known), U = lowbit(n):

  * n not a power of two (so n >= 3U): the block of Algorithm 1 with x as the input
    and rho as the taps, x[n - U, n) against rho[1, 2U), onto y[n, n + U); and the
    same block with the roles swapped, rho[n - U, n) against x[1, 2U).  rho[0, 2U)
    and x[0, 2U) are known since step 2U <= n.  These are the two convolutions of the
    same size per step.
  * n = U a power of two: the pairs with both indices below U and i + j >= U, which
    is Algorithm 1's block with x[0, U) as the input and rho[0, 2U) as the taps,
    rho[U, 2U) not yet known and taken as zero.

Every pair with i, j >= 1 is then covered exactly once (tests/test_dd_schedule.py
checks it by brute force, together with the knowledge constraint), and the work is
twice that of Algorithm 1 with a fixed filter.  For a block of size U the FFT form
needs the spectra of the prefixes x[0, 2U) and rho[0, 2U): they are final at step
2U, before the first block of size U that uses them (step 3U).
"""
from __future__ import annotations

import numpy as np


def lowbit(n: int) -> int:
    return n & -n


def is_pow2(n: int) -> bool:
    return n > 0 and (n & (n - 1)) == 0


def schedule(L: int):
    """Blocks released after the n-th token, n = 1 .. L-1: (n, kind, U) with kind
    "x" (x as the input, rho as the taps) or "rho" (roles swapped)."""
    out = []
    for n in range(1, L):
        U = lowbit(n)
        out.append((n, "x", U))
        if not is_pow2(n):
            out.append((n, "rho", U))
    return out


def block_pairs(n: int, kind: str, U: int):
    """The (i, j) pairs (i: index into rho, j: index into x) whose products a block
    adds, in the order of its outputs t = i + j in [n, n + U)."""
    pairs = []
    for r in range(U):
        t = n + r
        for s in range(n - U, n):  # the block's input positions
            lag = t - s            # its tap index, 1 .. 2U - 1
            if is_pow2(n) and lag >= U:
                continue           # rho[U, 2U) is not known yet at n = U
            pairs.append((lag, s) if kind == "x" else (s, lag))
    return pairs


def run(x, rho):
    """y [T][G] by the online schedule: at step t, x_t and rho_t join the known
    values, the red cells finish y_t, then the blocks released after token t + 1 are
    added to the running sums of later positions.  Values not yet known are NaN in
    the buffers, so a block that read one would poison its outputs.  x, rho: [T][G]."""
    x = np.asarray(x, dtype=np.float64)
    rho = np.asarray(rho, dtype=np.float64)
    T, G = x.shape
    xb = np.full((T, G), np.nan)
    rb = np.full((T, G), np.nan)
    acc = np.zeros((T, G))
    y = np.zeros((T, G))
    for t in range(T):
        xb[t] = x[t]
        rb[t] = rho[t]
        y[t] = acc[t] + rb[0] * xb[t]
        if t > 0:
            y[t] += rb[t] * xb[0]
        n = t + 1
        if n >= T:
            continue
        U = lowbit(n)
        for kind in ("x", "rho"):
            if kind == "rho" and is_pow2(n):
                continue
            inp, taps = (xb, rb) if kind == "x" else (rb, xb)
            for r in range(U):
                if n + r >= T:
                    break
                s_acc = np.zeros(G)
                for s in range(n - U, n):
                    lag = n + r - s
                    if is_pow2(n) and lag >= U:
                        continue
                    s_acc += inp[s] * taps[lag]
                acc[n + r] += s_acc
    return y

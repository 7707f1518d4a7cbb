"""Seeded synthetic inputs for the mixer stack.

This module holds no arithmetic of the method itself: it only draws filters and
input tokens.  Both the CUDA path's callers (tests, bench) and the CPU oracle are
fed the same arrays from here, so the choice of generator can never cause a
mismatch between the two.

Recipe (random-init weights, as in the experimental setup of the Flash Inference
paper summary, section "Experimentelle Einrichtung"):

* filter of layer l, channel c, tap k:
  ``h[l, c, k] = N(0,1) * exp(-a_c * k) / sqrt(32)`` with ``a_c ~ U(0.001, 0.05)``;
  every layer draws its own ``a`` and its own normals ("same law", not the same draw).
* inputs: ``x ~ N(0,1)`` i.i.d. over (t, b, c); closed loop starts from one
  ``x_0 ~ N(0,1)`` per (b, c).

Generator: numpy PCG64 seeded through ``SeedSequence([seed, stream, l])``, one
independent stream per layer (stream 1), one for teacher-forced inputs (stream 2),
one for the closed-loop start token (stream 3), the Hyena-like model's weights
(stream 4), its token ids (stream 5) and the data-dependent filter's inputs (stream 6).  Within a layer stream the
draw order is: ``a_c`` for all c, then the normals in [c][k] order.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

A_LO, A_HI = 0.001, 0.05
SCALE = 1.0 / math.sqrt(32.0)


def _rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, sub])))


def _layer(out: np.ndarray, seed: int, l: int, decay: bool, chunk: int = 64) -> None:
    D, L = out.shape
    g = _rng(seed, 1, l)
    a = g.uniform(A_LO, A_HI, size=D)
    if not decay:
        a[:] = 0.0
    k = np.arange(L, dtype=np.float64)
    for c0 in range(0, D, chunk):
        c1 = min(D, c0 + chunk)
        z = g.standard_normal((c1 - c0, L))
        z *= np.exp(-a[c0:c1, None] * k[None, :])
        z *= SCALE
        out[c0:c1] = z


def filters(M: int, D: int, L: int, seed: int = 0, decay: bool = True,
            threads: int | None = None, out: np.ndarray | None = None) -> np.ndarray:
    """float32 [M][D][L] decaying-exponential random filters (one stream per layer).

    ``decay=False`` keeps the same normals but sets every ``a_c`` to 0, giving
    non-decaying filters whose long lags are not negligible (used to exercise
    the large tiles numerically)."""
    h = np.empty((M, D, L), np.float32) if out is None else out
    assert h.shape == (M, D, L) and h.dtype == np.float32
    if threads is None:
        import os
        threads = min(M, max(1, len(os.sched_getaffinity(0))))
    if threads <= 1 or M == 1:
        for l in range(M):
            _layer(h[l], seed, l, decay)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda l: _layer(h[l], seed, l, decay), range(M)))
    return h


def filter_rows(M: int, D: int, L: int, chans, T: int, seed: int = 0, decay: bool = True) -> np.ndarray:
    """float32 [M][len(chans)][T]: ``filters(M, D, L, seed)[:, chans, :T]`` without
    materialising the whole array.  Each layer's stream is drawn in the same order
    and the same chunks as ``filters`` (every chunk is drawn whole and the rows asked
    for are kept), so the values are bit-identical."""
    chans = [int(c) for c in chans]
    out = np.empty((M, len(chans), T), np.float32)
    k = np.arange(L, dtype=np.float64)
    chunk = 64

    def layer(l):
        g = _rng(seed, 1, l)
        a = g.uniform(A_LO, A_HI, size=D)
        if not decay:
            a[:] = 0.0
        for c0 in range(0, D, chunk):
            c1 = min(D, c0 + chunk)
            z = g.standard_normal((c1 - c0, L))
            for i, c in enumerate(chans):
                if c0 <= c < c1:
                    row = z[c - c0] * np.exp(-a[c] * k)
                    row *= SCALE
                    out[l, i] = row[:T]

    import os
    threads = min(M, max(1, len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(layer, range(M)))
    return out


def device_filters(M: int, D: int, L: int, seed: int = 0):
    """float32 [M][D][L] torch CUDA tensor with the filter law of ``filters`` drawn on
    the device by torch's seeded CUDA generator (per layer ``manual_seed(1000003 *
    seed + l)``: ``a_c`` for all c, then the normals).  A different draw from
    ``filters``; used where host generation of long filters would take minutes (the
    configuration sweep).  Copy it to the host to give the oracle the same array."""
    import torch
    h = torch.empty((M, D, L), device="cuda", dtype=torch.float32)
    k = torch.arange(L, device="cuda", dtype=torch.float32)
    for l in range(M):
        g = torch.Generator(device="cuda")
        g.manual_seed(1_000_003 * seed + l)
        a = torch.empty(D, device="cuda").uniform_(A_LO, A_HI, generator=g)
        h[l].normal_(generator=g)
        h[l] *= torch.exp(-a[:, None] * k[None, :]) * SCALE
    return h


def inputs(T: int, B: int, D: int, seed: int = 0) -> np.ndarray:
    """float32 [T][B][D] teacher-forced tokens, N(0,1)."""
    return _rng(seed, 2).standard_normal((T, B, D)).astype(np.float32)


def start_token(B: int, D: int, seed: int = 0) -> np.ndarray:
    """float32 [B][D] closed-loop start token x_0, N(0,1)."""
    return _rng(seed, 3).standard_normal((B, D)).astype(np.float32)


def _bf16_values(a: np.ndarray) -> np.ndarray:
    """float32 array holding the nearest bfloat16 values (torch's conversion): the GEMM
    weights of the Hyena-like model are bf16 tensors."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def hyena_params(M: int, D: int, L: int, V: int, seed: int = 0) -> dict:
    """Random-init weights of the Hyena-like model (stream 4, one sub-stream per layer):
    embedding E [V][D] ~ N(0, 1); per layer W_in [3D][D] ~ N(0, 1/D), short-conv taps
    c [3][3D] ~ N(0, 1/3), W1 [4D][D] ~ N(0, 1/D), W2 [D][4D] ~ N(0, 1/(4D)); LM head
    W_lm [V][D] ~ N(0, 1/D); the GEMM weights (E, W_in, W1, W2, W_lm) rounded to bf16
    values.  The long-convolution filters h [M][D][L] follow the mixer's law
    (``filters``, same seed)."""
    g = _rng(seed, 4, 0)
    E = _bf16_values(g.standard_normal((V, D)))
    W_lm = _bf16_values(g.standard_normal((V, D)) / math.sqrt(D))
    W_in, c, W1, W2 = [], [], [], []
    for l in range(M):
        gl = _rng(seed, 4, 1 + l)
        W_in.append(_bf16_values(gl.standard_normal((3 * D, D)) / math.sqrt(D)))
        c.append((gl.standard_normal((3, 3 * D)) / math.sqrt(3.0)).astype(np.float32))
        W1.append(_bf16_values(gl.standard_normal((4 * D, D)) / math.sqrt(D)))
        W2.append(_bf16_values(gl.standard_normal((D, 4 * D)) / math.sqrt(4 * D)))
    h = filters(M, D, L, seed=seed)
    return {"E": E, "W_lm": W_lm, "W_in": W_in, "c": c, "W1": W1, "W2": W2, "h": list(h)}


def token_ids(T: int, B: int, V: int, seed: int = 0) -> np.ndarray:
    """int32 [T][B] synthetic token ids, uniform over the vocabulary (stream 5)."""
    return _rng(seed, 5).integers(0, V, size=(T, B)).astype(np.int32)


def dd_inputs(T: int, G: int, seed: int = 0):
    """The data-dependent filter's online inputs (stream 6): x [T][G] ~ N(0, 1) and
    rho [T][G] with the filter law of ``filters`` laid out by step, rho[t][g] =
    N(0, 1) * exp(-a_g t) / sqrt(32), a_g ~ U(0.001, 0.05) (a_g drawn first, then the
    normals of x, then those of rho, [t][g] order).  float32."""
    g = _rng(seed, 6)
    a = g.uniform(A_LO, A_HI, size=G)
    x = g.standard_normal((T, G)).astype(np.float32)
    z = g.standard_normal((T, G))
    rho = (z * np.exp(-np.outer(np.arange(T, dtype=np.float64), a)) * SCALE).astype(np.float32)
    return x, rho


def device_dd_inputs(T: int, G: int, seed: int = 0):
    """``dd_inputs``' law drawn on the device by torch's seeded CUDA generator
    (``manual_seed(1000003 * seed + 6)``: a, then x, then the normals of rho): a
    different draw, for sizes whose host generation would take minutes.  Torch CUDA
    tensors [T][G]."""
    import torch
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1_000_003 * seed + 6)
    a = torch.empty(G, device="cuda").uniform_(A_LO, A_HI, generator=gen)
    x = torch.empty((T, G), device="cuda").normal_(generator=gen)
    rho = torch.empty((T, G), device="cuda").normal_(generator=gen)
    t = torch.arange(T, device="cuda", dtype=torch.float32)
    for t0 in range(0, T, 4096):
        rho[t0:t0 + 4096] *= torch.exp(-t[t0:t0 + 4096, None] * a[None, :]) * SCALE
    return x, rho


# Workloads (layers, B, D, L) of the measured configurations.
CONFIGS = {
    "tiny": dict(M=1, B=1, D=16, L=1 << 10),
    "headline": dict(M=18, B=1, D=864, L=1 << 17),
    "hyena_shape": dict(M=18, B=4, D=768, L=1 << 15),
}

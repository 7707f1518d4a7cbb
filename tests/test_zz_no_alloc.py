"""fi_tau_fft_noalloc: the FFT tau for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: their device memory is reserved up front by
another allocator (a framework's caching pool, a serving engine that claims most
of HBM at start-up), or they cannot accept the device-wide synchronisation an
allocation may cost.  For them the library offers one entry point whose
temporaries live in a fixed array of device memory inside the library itself.
This file checks it through the C-ABI against fi_tau, the allocating entry point,
and against the CPU oracle's tau (the sum of Lemma 1, section
"Beitrags-Aggregations-Definition" of the Flash Inference paper summary): every
output for the small blocks, sampled outputs for the large ones.

The file is named so that pytest collects it last: if it fails, a run that stops
at the first failure has already run every other test.  It must pass both alone
in a fresh process and after the rest of the suite, since every call shares the
same fixed array.
"""
import ctypes
import math

import numpy as np
import pytest

import long_convolution_sequence_b200 as fi
import oracle

TOL = 1e-4  # max |err| / RMS, the tolerance of the other tau parity tests


def rel(got, ref):
    return float(np.abs(got - ref).max() / math.sqrt(float(np.mean(ref.astype(np.float64) ** 2))))


def oracle_tau(blocks, taps, rng, k=48):
    """The oracle's tau: (rows, reference) with every row r for U <= 4096, else k
    sampled rows per block (first, last and random), each by the plain sum
    sum_j blocks[i][j] taps[i][U + r - j] (a causal convolution sample at t = U + r
    of the block padded with zeros)."""
    count, U = blocks.shape
    if U <= 4096:
        return np.arange(U), oracle.tau(blocks, taps)
    rows = np.unique(np.concatenate([[0, 1, U // 2, U - 1], rng.integers(0, U, size=k)]))
    ref = np.empty((count, rows.size))
    for i in range(count):
        y = np.zeros(2 * U, np.float32)
        y[:U] = blocks[i]
        h = np.ascontiguousarray(taps[i])
        for j, r in enumerate(rows):
            ref[i, j] = oracle.conv_at(U + int(r), h, y)
    return rows, ref


def test_noalloc_rejects_blocks_beyond_its_scratch():
    # argument checks answer before any device work, so this runs without a GPU
    lib = fi.get_lib()
    buf = (ctypes.c_float * 64)()
    p = ctypes.addressof(buf)
    assert lib.fi_tau_fft_noalloc(1 << 17, 1, p, p, 1 << 18, p, 0) == fi.FI_EINVAL
    assert b"65536" in lib.fi_last_error()
    assert lib.fi_tau_fft_noalloc(4, 1, p, p, 8, p, 0) == fi.FI_EINVAL      # below the FFT sizes
    assert lib.fi_tau_fft_noalloc(48, 1, p, p, 96, p, 0) == fi.FI_EINVAL    # not a power of two
    assert lib.fi_tau_fft_noalloc(8, 1, p, p, 17, p, 0) == fi.FI_EINVAL     # odd row length
    assert lib.fi_tau_fft_noalloc(8, 0, p, p, 16, p, 0) == fi.FI_EINVAL     # nothing to do


# (U, count): counts above what one chunk of the fixed array holds at the largest
# sizes (12 blocks at U = 65536, 24 at U = 32768) so that chunking is exercised
CASES = [(8, 5), (256, 9), (4096, 4), (16384, 3), (32768, 26), (65536, 13)]


@pytest.mark.gpu
@pytest.mark.parametrize("U,count", CASES)
def test_noalloc_matches_fi_tau_on_two_calls_in_a_row(U, count):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1000 + U)
    for call in range(2):
        blocks_h = rng.standard_normal((count, U)).astype(np.float32)
        taps_h = rng.standard_normal((count, 2 * U + 2)).astype(np.float32)
        blocks = torch.from_numpy(blocks_h).cuda()
        taps = torch.from_numpy(taps_h).cuda()
        start = torch.from_numpy(rng.standard_normal((count, U)).astype(np.float32)).cuda()
        accumulate = call == 1
        ref = start.clone()
        fi.tau(fi.FI_TAU_FFT, U, blocks, taps, ref, accumulate=accumulate)
        got = start.clone()
        fi.tau_fft_noalloc(U, blocks, taps, got, accumulate=accumulate)
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        base = start.cpu().numpy() if accumulate else 0.0
        assert np.isfinite(g).all()
        assert rel(g - base, r - base) < TOL, (U, count, call)
        rows, want = oracle_tau(blocks_h, taps_h, rng)
        assert rel((g - base)[:, rows], want) < TOL, (U, count, call, "oracle")

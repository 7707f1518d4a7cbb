"""How far fp32 rounding alone carries a closed loop away from the fp64 definition.

The closed-loop criterion (GPU within 1e-3 of the RMS over the first 4096 steps) is
only meaningful if rounding by itself does not drive the trajectory away: the tanh
feedback could in principle amplify the difference between two exact evaluations in
different precisions.  The oracle runs the same stack (section "LCSM-Inferenz-
Algorithmus (Algorithmus 2)" of the Flash Inference paper summary, tanh block and
sampler) in fp32 and in fp64 on sampled chains of the measured shapes, and the two
must stay well inside the criterion.  Chains never interact, so the sampled
channels' chains are computed alone, with the filters the full draw gives them.

Measured once over 16384 steps (recorded with the design notes): the running maximum
of |fp32 - fp64| / RMS passes 1e-5 at step 26 (headline) and 65 (Hyena shape) and
stays below 1e-4 throughout; it never reaches 1e-3.
"""
import numpy as np
import pytest

import oracle
from long_convolution_sequence_b200 import synth


def test_filter_rows_equal_the_full_draw():
    for decay in (True, False):
        full = synth.filters(3, 130, 512, seed=2, decay=decay)
        rows = synth.filter_rows(3, 130, 512, [0, 5, 64, 129], 100, seed=2, decay=decay)
        np.testing.assert_array_equal(rows, full[:, [0, 5, 64, 129], :100])


@pytest.mark.parametrize("shape", [(18, 1, 864, 1 << 17), (18, 4, 768, 1 << 15)],
                         ids=["headline", "hyena_shape"])
def test_fp32_oracle_tracks_fp64_over_the_criterion_window(shape):
    M, B, D, L = shape
    T = 4096
    chans = [0, 1, D // 2, D - 1]
    h = synth.filter_rows(M, D, L, chans, T, seed=0)
    x0 = np.ascontiguousarray(synth.start_token(B, D, seed=0)[:, chans])
    r64 = oracle.stack(h, x0, T=T, closed_loop=True)["y_last"]
    r32 = oracle.stack(h, x0, T=T, closed_loop=True, fp32=True)["y_last"]
    assert np.isfinite(r64).all() and np.isfinite(r32).all()
    err = np.abs(r32 - r64).reshape(T, -1).max(axis=1)
    rms = np.sqrt(np.cumsum((r64.reshape(T, -1) ** 2).mean(axis=1)) / np.arange(1, T + 1))
    running = np.maximum.accumulate(err) / rms
    assert running[-1] < 1e-4, running[-1]
    # and rounding is visible at all (the fp32 run is not secretly the fp64 one)
    assert running[-1] > 1e-8

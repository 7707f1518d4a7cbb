"""The Lazy and Eager baselines (FI_PATH_LAZY / FI_PATH_EAGER, and their non-parallel
forms FI_PATH_LAZY_NP / FI_PATH_EAGER_NP) against the oracle.

Both evaluate the same stack as the relaxed tiling by the two plain strategies of the
Flash Inference summary's section "Kern-Algorithmus: Relaxierte
Polynominterpolation" (part 1): Lazy sums each position's history when it is needed,
Eager pushes each activation onto every later position as soon as it is known.  They
must give the oracle's result to the same tolerances as the tiled paths, continue
across calls, and refuse a switch of path in the middle of a generation."""
import math

import numpy as np
import pytest

import long_convolution_sequence_b200 as fi
import oracle
from long_convolution_sequence_b200 import synth

TOL_TF = 1e-4   # teacher-forced: max |err| / RMS(y)
TOL_CL = 1e-3   # closed loop

PATHS = {"lazy": fi.FI_PATH_LAZY, "eager": fi.FI_PATH_EAGER,
         "lazy_np": fi.FI_PATH_LAZY_NP, "eager_np": fi.FI_PATH_EAGER_NP}


def rel(got, ref):
    return float(np.abs(got - ref).max() / math.sqrt(float(np.mean(ref.astype(np.float64) ** 2))))


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(PATHS))
def test_closed_loop_matches_oracle(name):
    M, B, D, L = 3, 2, 6, 512
    h = synth.filters(M, D, L, seed=3)
    x0 = synth.start_token(B, D, seed=3)
    ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_path(PATHS[name])
        out = np.empty((L, B, D), np.float32)
        ctx.generate(x0, L, out)
    assert rel(out, ref) < TOL_CL


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(PATHS))
def test_teacher_forced_every_layer(name):
    M, B, D, L = 4, 1, 5, 256
    h = synth.filters(M, D, L, seed=5)
    x = synth.inputs(L, B, D, seed=5)
    ref = oracle.stack(h, x, want=("y_all",))["y_all"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_path(PATHS[name])
        y = np.empty((L, B, D), np.float32)
        ctx.forward(x, L, y)
        a = np.empty((L, B, D), np.float32)
        for l in range(1, M + 1):
            ctx.read_layer(l, 0, L, a)
            rms = math.sqrt(float(np.mean(ref[l - 1] ** 2)))
            assert np.abs(a - np.tanh(ref[l - 1])).max() < TOL_TF * rms, l
    assert rel(y, ref[-1]) < TOL_TF


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(PATHS))
def test_call_split_and_agreement_with_the_tiled_path(name):
    M, B, D, L = 18, 1, 8, 1024
    h = synth.filters(M, D, L, seed=6)
    x0 = synth.start_token(B, D, seed=6)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        whole = np.empty((L, B, D), np.float32)
        ctx.generate(x0, L, whole)          # the tiled (window) path
        ctx.reset()
        ctx.set_path(PATHS[name])
        part = np.empty((L, B, D), np.float32)
        ctx.generate(x0, 300, part[:300])   # split at a position inside a window
        ctx.generate(None, L - 300, part[300:])
    # two exact evaluations of the same closed loop, in different summation orders
    n = 256
    assert rel(part[:n], whole[:n]) < TOL_CL


@pytest.mark.gpu
def test_path_switch_only_at_the_start():
    M, B, D, L = 2, 1, 3, 64
    h = synth.filters(M, D, L, seed=7)
    x0 = synth.start_token(B, D, seed=7)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        out = np.empty((8, B, D), np.float32)
        ctx.generate(x0, 8, out)
        with pytest.raises(fi.FiError):
            ctx.set_path(fi.FI_PATH_LAZY)
        ctx.reset()
        ctx.set_path(fi.FI_PATH_LAZY)
        ctx.generate(x0, 8, out)
        with pytest.raises(fi.FiError):
            ctx.set_path(fi.FI_PATH_EAGER)
        ctx.reset()
        ctx.set_path(fi.FI_PATH_EAGER)

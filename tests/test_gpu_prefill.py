"""fi_prefill: a prompt folded in with one FFT convolution per layer.

The prefill must leave exactly the tiled paths' state at t = p, so the strongest check
is to continue the sequence: prefill p tokens, run the rest teacher-forced with
fi_forward, and compare every output with the oracle's teacher-forced run over the
whole sequence (section "LCSM-Inferenz-Algorithmus (Algorithmus 2)" with tanh).  Wrong
running sums at the positions after the prompt would show at once after it."""
import math

import numpy as np
import pytest

import long_convolution_sequence_b200 as fi
import oracle
from long_convolution_sequence_b200 import synth

TOL_TF = 1e-4   # teacher-forced: max |err| / RMS(y)
TOL_CL = 1e-3   # closed loop


def rel(got, ref):
    return float(np.abs(got - ref).max() / math.sqrt(float(np.mean(ref.astype(np.float64) ** 2))))


@pytest.fixture(scope="module")
def stack():
    M, B, D, L = 3, 2, 5, 1024
    h = synth.filters(M, D, L, seed=11)
    x = synth.inputs(L, B, D, seed=11)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    return M, B, D, L, h, x, ref


@pytest.mark.gpu
@pytest.mark.parametrize("path", ["window", "token"])
@pytest.mark.parametrize("p", [8, 13, 64, 100, 128, 300, 512, 1000, 1024])
def test_prefill_then_forward_matches_the_oracle(stack, p, path):
    M, B, D, L, h, x, ref = stack
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_path(fi.FI_PATH_WINDOW if path == "window" else fi.FI_PATH_TOKEN)
        y = np.empty((L, B, D), np.float32)
        ctx.prefill(np.ascontiguousarray(x[:p]), p, y[:p])
        assert ctx.info().t == p
        if p < L:
            ctx.forward(np.ascontiguousarray(x[p:]), L - p, y[p:])
    assert rel(y[:p], ref[:p]) < TOL_TF
    assert rel(y, ref) < TOL_TF


@pytest.mark.gpu
def test_prefill_of_the_18_layer_stack_with_a_batch():
    M, B, D, L, p = 18, 2, 5, 2048, 777
    h = synth.filters(M, D, L, seed=14)
    x = synth.inputs(L, B, D, seed=14)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        ctx.prefill(np.ascontiguousarray(x[:p]), p, y[:p])
        ctx.forward(np.ascontiguousarray(x[p:]), L - p, y[p:])
    assert rel(y, ref) < TOL_TF


@pytest.mark.gpu
def test_short_prompt_takes_the_online_path(stack):
    M, B, D, L, h, x, ref = stack
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        ctx.prefill(np.ascontiguousarray(x[:5]), 5, y[:5])
        ctx.forward(np.ascontiguousarray(x[5:]), L - 5, y[5:])
    assert rel(y, ref) < TOL_TF


@pytest.mark.gpu
def test_prefill_then_generate_agrees_with_forward_then_generate():
    M, B, D, L, p = 18, 1, 8, 2048, 700
    h = synth.filters(M, D, L, seed=12)
    x = synth.inputs(p, B, D, seed=12)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ya = np.empty((p, B, D), np.float32)
        ctx.forward(x, p, ya)
        ga = np.empty((L - p, B, D), np.float32)
        ctx.generate(np.tanh(ya[-1]).astype(np.float32), L - p, ga)
        ctx.reset()
        yb = np.empty((p, B, D), np.float32)
        ctx.prefill(x, p, yb)
        gb = np.empty((L - p, B, D), np.float32)
        ctx.generate(np.tanh(yb[-1]).astype(np.float32), L - p, gb)
    assert rel(yb, ya) < TOL_TF
    assert rel(gb[:256], ga[:256]) < TOL_CL


@pytest.mark.gpu
def test_prefill_of_a_cluster_sized_prompt():
    # p = 20000 -> U = 32768: the prefill's convolutions run on the cluster FFT
    M, B, D, L, p = 2, 1, 3, 32768, 20000
    h = synth.filters(M, D, L, seed=13)
    x = synth.inputs(L, B, D, seed=13)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        ctx.prefill(np.ascontiguousarray(x[:p]), p, y[:p])
        ctx.forward(np.ascontiguousarray(x[p:]), L - p, y[p:])
    assert rel(y, ref) < TOL_TF


@pytest.mark.gpu
def test_prefill_argument_errors(stack):
    M, B, D, L, h, x, ref = stack
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        with pytest.raises(fi.FiError):
            ctx.prefill(np.ascontiguousarray(x[:1]), L + 1, y)
        ctx.forward(np.ascontiguousarray(x[:4]), 4, y[:4])
        with pytest.raises(fi.FiError):  # not at t = 0
            ctx.prefill(np.ascontiguousarray(x[:64]), 64, y[:64])
        ctx.reset()
        ctx.set_path(fi.FI_PATH_LAZY)
        with pytest.raises(fi.FiError):  # the baselines have no prefill
            ctx.prefill(np.ascontiguousarray(x[:64]), 64, y[:64])


@pytest.mark.gpu
def test_prefill_beyond_the_largest_fft_is_rejected_before_any_work():
    # L = 2^18 is a valid capacity, but one FFT convolution serves prompts of at most
    # 2^17 tokens: a longer prompt must fail with FI_EINVAL and leave the context at t = 0
    M, B, D, L = 1, 1, 2, 1 << 18
    h = synth.filters(M, D, L, seed=9)
    p = (1 << 17) + 1
    x = synth.inputs(p, B, D, seed=9)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((p, B, D), np.float32)
        with pytest.raises(fi.FiError) as e:
            ctx.prefill(x, p, y)
        assert e.value.code == fi.FI_EINVAL and "131072" in str(e.value)
        assert ctx.info().t == 0
        ctx.prefill(np.ascontiguousarray(x[: 1 << 17]), 1 << 17, y[: 1 << 17])  # the largest one works
        assert ctx.info().t == 1 << 17

"""The Hyena-like language model (fi_lm_*) against its oracle (oracle/hyena.py).

Tolerance.  Both sides round every GEMM operand to bf16; they differ by fp32
accumulation on the GPU (relative ~2^-24 sqrt(K)) and, where the GPU's fp32 value of
an activation and the oracle's fp64 value fall on two sides of a bf16 rounding
boundary, by one bf16 step (2^-8 relative) of that operand.  One such step moves a
GEMV output by about 2^-8 / sqrt(K) of its scale; a token passes 3 GEMVs per layer and
the LM head, so even one step in every GEMV at its largest input stays below
(3 M + 1) 2^-8 of the RMS.  The check: max |logits - oracle| <= (3 M + 1) 2^-8 RMS.
Integer decisions: a greedy choice must equal the oracle's wherever the oracle's two
best logits are further apart than 4x the largest logit error measured.
"""
import math

import numpy as np
import pytest

import long_convolution_sequence_b200 as fi
from long_convolution_sequence_b200 import synth
from oracle import hyena

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def model(p, M, B, D, L, V):
    return fi.LanguageModel(M, B, D, L, V, p["E"], p["W_lm"], np.ascontiguousarray(np.stack(p["W_in"])),
                            np.ascontiguousarray(np.stack(p["c"])), np.ascontiguousarray(np.stack(p["W1"])),
                            np.ascontiguousarray(np.stack(p["W2"])), np.ascontiguousarray(np.stack(p["h"])))


def margins(logits):
    s = np.sort(logits, axis=-1)
    return s[..., -1] - s[..., -2]


@pytest.mark.parametrize("M,B,D,L,V,T", [(2, 2, 64, 256, 1000, 256), (3, 4, 32, 512, 300, 200),
                                          (2, 6, 40, 128, 700, 128)])
def test_teacher_forced_logits_and_choices_match_oracle(M, B, D, L, V, T):
    p = synth.hyena_params(M, D, L, V, seed=1)
    tok = synth.token_ids(T, B, V, seed=2)
    ref = hyena.run(p, tokens=tok)
    with model(p, M, B, D, L, V) as lm:
        logits = np.empty((T, B, V), np.float32)
        nxt = np.empty((T, B), np.int32)
        lm.forward(tok, T, logits, nxt)
    rms = math.sqrt(float(np.mean(ref["logits"] ** 2)))
    err = np.abs(logits - ref["logits"])
    assert err.max() <= (3 * M + 1) * 2.0 ** -8 * rms, err.max() / rms
    clear = margins(ref["logits"]) > 4 * err.max()
    assert clear.mean() > 0.5
    np.testing.assert_array_equal(nxt[clear], ref["next"][clear])


def test_greedy_generation_matches_oracle_until_a_near_tie():
    M, B, D, L, V, T = 2, 2, 64, 256, 1000, 128
    p = synth.hyena_params(M, D, L, V, seed=3)
    tok0 = synth.token_ids(1, B, V, seed=4)[0]
    ref = hyena.run(p, tok0=tok0, T=T)
    with model(p, M, B, D, L, V) as lm:
        nxt = np.empty((T, B), np.int32)
        lm.generate(tok0, T, nxt)
        # teacher-forced replay of the oracle's own inputs gives the logit error scale
        lm.reset()
        logits = np.empty((T, B, V), np.float32)
        tf = np.empty((T, B), np.int32)
        lm.forward(np.ascontiguousarray(ref["tokens"].astype(np.int32)), T, logits, tf)
    thr = 4 * float(np.abs(logits - ref["logits"]).max())
    m = margins(ref["logits"])
    first_tie = next((k for k in range(T) if (m[k] <= thr).any()), T)
    assert first_tie >= 1
    np.testing.assert_array_equal(nxt[:first_tie], ref["next"][:first_tie])


def test_calls_split_and_reset_repeat():
    M, B, D, L, V = 2, 2, 32, 128, 200
    p = synth.hyena_params(M, D, L, V, seed=5)
    tok = synth.token_ids(L, B, V, seed=6)
    with model(p, M, B, D, L, V) as lm:
        whole = np.empty((L, B), np.int32)
        lm.forward(tok, L, None, whole)
        lm.reset()
        part = np.empty((L, B), np.int32)
        td = torch.from_numpy(tok).cuda()
        pd = torch.empty((L, B), dtype=torch.int32, device="cuda")
        lm.forward(td[:37], 37, None, pd[:37])           # device arrays, a split inside a block
        lm.forward(tok[37:], L - 37, None, part[37:])    # host arrays
        torch.cuda.synchronize()
        part[:37] = pd[:37].cpu().numpy()
        np.testing.assert_array_equal(part, whole)
        with pytest.raises(fi.FiError) as e:
            lm.forward(tok[:1], 1, None, part[:1])
        assert e.value.code == fi.FI_ECAPACITY


def test_trace_reports_a_mixer_share():
    M, B, D, L, V = 2, 2, 32, 256, 200
    p = synth.hyena_params(M, D, L, V, seed=7)
    with model(p, M, B, D, L, V) as lm:
        lm.set_trace(True)
        nxt = np.empty((L, B), np.int32)
        lm.generate(np.array([1, 2], np.int32), L, nxt)
        mix, tot = lm.split()
        assert 0 < mix < tot


def test_generation_from_graphs_equals_host_launches():
    # the replayed per-token graphs run the same kernels on the same data: identical choices
    M, B, D, L, V = 2, 3, 32, 256, 300
    p = synth.hyena_params(M, D, L, V, seed=11)
    tok0 = np.array([5, 17, 200], np.int32)
    outs = []
    with model(p, M, B, D, L, V) as lm:
        for graphs in (True, False, True):
            lm.reset()
            lm.set_graphs(graphs)
            nxt = np.empty((L, B), np.int32)
            lm.generate(tok0, 100, nxt[:100])      # two calls: the record is set again
            lm.generate(None, L - 100, nxt[100:])
            outs.append(nxt)
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_traced_run_with_its_own_mixer_kernel_equals_the_fused_run():
    # a traced run launches the mixer step as its own kernel after a plain in-projection;
    # otherwise it is fused into the in-projection's epilogue: the same fp32 operations,
    # so the same choices and logits, bit for bit
    M, B, D, L, V = 2, 4, 64, 256, 500
    p = synth.hyena_params(M, D, L, V, seed=13)
    tok = synth.token_ids(L, B, V, seed=14)
    outs = []
    with model(p, M, B, D, L, V) as lm:
        for trace in (False, True):
            lm.reset()
            lm.set_trace(trace)
            logits = np.empty((64, B, V), np.float32)
            nxt = np.empty((64, B), np.int32)
            lm.forward(tok[:64], 64, logits, nxt)
            outs.append((logits, nxt))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])

"""Pins of the Hyena-like model's oracle (oracle/hyena.py), on the CPU.

Each piece is checked against something other than itself: torch's bfloat16
conversion, layer_norm and gelu (library routines the oracle does not call), closed
forms of the short convolution, the C oracle's causal convolution (pinned on its own
in test_oracle_pins.py) for the long convolution inside the model, and a reduction of
the whole model to the embedding and the LM head when every layer is the identity.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import hyena
from long_convolution_sequence_b200 import synth


def test_bf16_round_matches_torch_including_ties():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000) * 10 ** rng.uniform(-6, 6, 10000),
                        [0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40]]).astype(np.float32)
    # exact ties: the low 16 bits are 0x8000 (even and odd upper halves)
    ties = (rng.integers(0x3F000000, 0x41000000, 2000, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(hyena.bf16_round(x), ref)


def test_layer_norm_and_gelu_match_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 96)) * 3 + 1.5
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (96,), eps=hyena.LN_EPS).numpy()
    np.testing.assert_allclose(hyena.layer_norm(x), ref, rtol=1e-12, atol=1e-12)
    g = np.linspace(-8, 8, 1001)
    np.testing.assert_allclose(hyena.gelu(g), torch.nn.functional.gelu(torch.from_numpy(g)).numpy(),
                               rtol=1e-12, atol=1e-14)


def test_short_conv_closed_forms():
    rng = np.random.default_rng(2)
    z = [rng.standard_normal((2, 6)) for _ in range(3)]
    one, zero = np.ones(6), np.zeros(6)
    np.testing.assert_array_equal(hyena.short_conv(z, np.stack([one, zero, zero])), z[0])
    np.testing.assert_array_equal(hyena.short_conv(z, np.stack([zero, one, zero])), z[1])
    np.testing.assert_array_equal(hyena.short_conv(z, np.stack([zero, zero, one])), z[2])


def small_model(M=2, D=8, L=64, V=50, seed=3):
    return synth.hyena_params(M, D, L, V, seed=seed)


def test_the_long_convolution_inside_the_model_is_the_causal_convolution():
    M, D, L, V, B = 2, 8, 64, 50, 3
    p = small_model(M, D, L, V)
    tok = synth.token_ids(L, B, V, seed=4)
    out = hyena.run(p, tokens=tok, want=("tokens",))
    # the C oracle's fp64 causal convolution of the mixer inputs the model recorded
    for l in range(M):
        for b in range(B):
            for c in (0, D - 1):
                ref = oracle.causal_conv(p["h"][l][c].astype(np.float64), out["x"][l][:, b, c])
                np.testing.assert_allclose(out["y"][l][:, b, c], ref, rtol=1e-12, atol=1e-12)


def test_identity_layers_reduce_to_embedding_and_lm_head():
    # h = 0 removes the mixer's output and W2 = 0 the MLP's: every layer is the
    # identity, so the logits are W_lm bf16(LN(E[tok])) and the greedy loop iterates
    # tok -> argmax of that, computed here with torch
    M, D, L, V, B = 2, 16, 32, 40, 2
    p = small_model(M, D, L, V, seed=5)
    p["h"] = [np.zeros_like(h) for h in p["h"]]
    p["W2"] = [np.zeros_like(w) for w in p["W2"]]
    E = torch.from_numpy(p["E"]).double()
    W = torch.from_numpy(p["W_lm"]).double()

    def logits_of(tok):
        a = torch.nn.functional.layer_norm(E[torch.as_tensor(tok)], (D,), eps=hyena.LN_EPS)
        a = a.float().to(torch.bfloat16).double()
        return (a @ W.T).numpy()

    tok = synth.token_ids(L, B, V, seed=6)
    tf = hyena.run(p, tokens=tok)
    for t in (0, 7, L - 1):
        np.testing.assert_allclose(tf["logits"][t], logits_of(tok[t]), rtol=1e-12, atol=1e-12)
    cl = hyena.run(p, tok0=tok[0], T=12)
    cur = tok[0]
    for t in range(12):
        assert (cl["tokens"][t] == cur).all()
        cur = np.argmax(logits_of(cur), axis=-1)
        assert (cl["next"][t] == cur).all()


def test_teacher_forced_and_closed_loop_agree_on_the_closed_loops_tokens():
    # feeding the greedy tokens back as teacher tokens reproduces the closed loop
    M, D, L, V, B = 2, 8, 48, 30, 2
    p = small_model(M, D, L, V, seed=7)
    cl = hyena.run(p, tok0=np.array([3, 11]), T=L)
    tf = hyena.run(p, tokens=cl["tokens"])
    np.testing.assert_array_equal(tf["next"], cl["next"])
    np.testing.assert_allclose(tf["logits"], cl["logits"], rtol=0, atol=0)


def test_one_layer_with_a_delta_filter_against_torch():
    # h = delta_0 and short-conv taps (1, 0, 0): y_t = x_t = k_t v_t, so one layer is
    # u + q k v followed by the MLP residual, per token, with no history
    M, D, L, V, B = 1, 16, 8, 30, 2
    p = small_model(M, D, L, V, seed=8)
    p["h"] = [np.zeros_like(h) for h in p["h"]]
    p["h"][0][:, 0] = 1.0
    p["c"][0] = np.stack([np.ones(3 * D), np.zeros(3 * D), np.zeros(3 * D)]).astype(np.float32)
    tok = synth.token_ids(L, B, V, seed=9)
    out = hyena.run(p, tokens=tok)
    T = torch
    bf = lambda a: a.float().to(T.bfloat16).double()
    ln = lambda a: T.nn.functional.layer_norm(a, (a.shape[-1],), eps=hyena.LN_EPS)
    E, Win, W1, W2, Wlm = (T.from_numpy(np.asarray(w)).double() for w in
                           (p["E"], p["W_in"][0], p["W1"][0], p["W2"][0], p["W_lm"]))
    for t in range(L):
        u = E[T.as_tensor(tok[t])]
        z = bf(ln(u)) @ Win.T
        q, k, v = z[:, :D], z[:, D:2 * D], z[:, 2 * D:]
        r = u + q * (k * v)
        u2 = r + bf(T.nn.functional.gelu(bf(ln(r)) @ W1.T)) @ W2.T
        np.testing.assert_allclose(out["u"][t], u2.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out["logits"][t], (bf(ln(u2)) @ Wlm.T).numpy(), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- the pins can fail
# Each plausible mistake is planted in a copy of oracle/hyena.py's source (loaded as a
# module of its own; the oracle itself is untouched) and must break at least one pin.
HYENA_MUTANTS = {
    "gemv_operand_not_rounded": ("    return bf16_round(a) @ np.asarray(W, dtype=np.float64).T",
                                 "    return np.asarray(a, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T"),
    "short_conv_wrong_tap": ("c[1] * z_hist[1] + c[2] * z_hist[2]", "c[1] * z_hist[2] + c[2] * z_hist[1]"),
    "layer_norm_without_eps": ("    return (x - mu) / np.sqrt(var + LN_EPS)", "    return (x - mu) / np.sqrt(var)"),
    "gelu_tanh_form": ("    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))",
                       "    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))"),
    "gate_uses_q": ("            x_hist[l, t] = k * v", "            x_hist[l, t] = q * v"),
    "residual_dropped": ("            u = r + m", "            u = m"),
    "mixer_lag_off_by_one": ("            lag = h[l][:, t::-1][:, : t + 1]",
                             "            lag = np.concatenate([h[l][:, t + 1:t + 2], h[l][:, t::-1]], axis=1)[:, : t + 1]"),
    "output_gate_dropped": ("            r = u + q * y", "            r = u + y"),
}


def _planted(name):
    import types
    from pathlib import Path
    src = Path(hyena.__file__).read_text()
    old, new = HYENA_MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("hyena_mutant_" + name)
    exec(compile(src.replace(old, new), "hyena_mutant_" + name, "exec"), mod.__dict__)
    return mod


def _pins_pass(mod):
    """True if every pin above holds with `mod` standing in for oracle.hyena."""
    global hyena
    real = hyena
    hyena = mod
    try:
        test_bf16_round_matches_torch_including_ties()
        test_layer_norm_and_gelu_match_torch()
        test_short_conv_closed_forms()
        test_the_long_convolution_inside_the_model_is_the_causal_convolution()
        test_identity_layers_reduce_to_embedding_and_lm_head()
        test_teacher_forced_and_closed_loop_agree_on_the_closed_loops_tokens()
        test_one_layer_with_a_delta_filter_against_torch()
        return True
    except AssertionError:
        return False
    finally:
        hyena = real


def test_the_unmodified_oracle_passes_the_pins():
    assert _pins_pass(hyena)


@pytest.mark.parametrize("name", sorted(HYENA_MUTANTS))
def test_every_planted_mistake_fails_a_pin(name):
    assert not _pins_pass(_planted(name)), name

"""Plain fp64 CPU oracle of the Hyena-like language model built around the mixer.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it; the CUDA
path never imports it and it imports nothing of the CUDA path.

What it computes.  The Flash Inference summary describes an LCSM layer as a mixer
(the long convolution, section "LCSM-spezifische Definition") followed by a block
that may hold "MLP, Schicht-Normalisierung, etc." (section "Modellarchitektur"), and
its experiments run a real Hyena model with random weights (section "Experimentelle
Einrichtung").  The pages give no more detail; the model taken here (the plainest
reading of the measured configuration: in-projection to 3D, short depthwise
convolution of 3 taps, gated long convolution, MLP 4D with GELU, bf16 GEMMs, fp32
mixer, vocabulary 50257, greedy decoding) is, per token t and batch row b:

    u      = E[tok_t]                                       embedding row
    for each layer l:
      z_t  = W_in^l  bf16(LN(u))                            3D values: (q, k, v)
      zc_t = c0 z_t + c1 z_{t-1} + c2 z_{t-2}               short causal conv, per channel
      x_t  = kc_t * vc_t                                    gate into the mixer
      y_t  = sum_{s<=t} h^l[t-s] x_s                        the long convolution (mixer)
      r    = u + qc_t * y_t                                 gated output, residual
      u    = r + W2^l bf16(GELU(W1^l bf16(LN(r))))          MLP 4D, residual
    logits = W_lm bf16(LN(u));  tok_{t+1} = argmax logits   greedy (ties: lowest id)

LN is a layer normalisation without affine parameters (eps 1e-5); GELU is the exact
erf form; bf16(.) rounds to the nearest bfloat16 (ties to even), the operand rounding
of a bf16 GEMM whose products are summed in higher precision.  Everything else is
exact here (fp64); the GEMM weights are bf16 values.  The mixer is evaluated by its
lazy definition: at token t the sum over the whole history of x.
"""
from __future__ import annotations

import math

import numpy as np

LN_EPS = 1e-5


def bf16_round(x):
    """Round to the nearest bfloat16 (ties to even), returned as float64.  Values
    are first rounded to float32 the way the GPU holds them, then the low 16 bits of
    the float32 pattern are rounded off."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def layer_norm(x):
    """(x - mean) / sqrt(var + eps) over the last axis (population variance)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + LN_EPS)


def gelu(x):
    """x * Phi(x) with the normal distribution function Phi(x) = (1 + erf(x / sqrt 2)) / 2."""
    x = np.asarray(x, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def short_conv(z_hist, c):
    """zc_t = c0 z_t + c1 z_{t-1} + c2 z_{t-2}; z_hist = [z_t, z_{t-1}, z_{t-2}] (zeros
    before position 0); c [3][C]."""
    return c[0] * z_hist[0] + c[1] * z_hist[1] + c[2] * z_hist[2]


def gemv_bf16(W, a):
    """W [N][K] (bf16 values) times bf16(a) [B][K] -> [B][N], products summed exactly."""
    return bf16_round(a) @ np.asarray(W, dtype=np.float64).T


def run(params, tokens=None, tok0=None, T=None, want=("logits", "tokens")):
    """The model over T positions.

    params: dict with E [V][D], and per layer lists W_in [3D][D], c [3][3D], h [D][>=T],
    W1 [4D][D], W2 [D][4D]; W_lm [V][D] (all float32 arrays; the GEMM weights hold
    bf16 values).  Teacher-forced: tokens int [T][B] (token t is the input at t).
    Closed loop (greedy): tok0 int [B] and T; the input at t+1 is argmax of the logits
    at t.  Returns a dict: "logits" [T][B][V], "tokens" [T][B] (the inputs used),
    "next" [T][B] (greedy choices), "x" and "y" [M][T][B][D] (mixer input and output
    per layer), "u" [T][B][D] (last hidden state before the final LN).
    """
    E = np.asarray(params["E"], np.float64)
    V, D = E.shape
    M = len(params["W_in"])
    if tokens is not None:
        tokens = np.asarray(tokens, np.int64)
        T, B = tokens.shape
    else:
        B = len(tok0)
    x_hist = np.zeros((M, T, B, D))
    y_all = np.zeros((M, T, B, D))
    z_prev = np.zeros((M, 2, B, 3 * D))  # z_{t-1}, z_{t-2} per layer
    logits_all = np.zeros((T, B, V)) if "logits" in want else None
    used = np.zeros((T, B), np.int64)
    nxt = np.zeros((T, B), np.int64)
    u_last = np.zeros((T, B, D))
    h = [np.asarray(hl, np.float64) for hl in params["h"]]
    cur = np.asarray(tok0, np.int64) if tokens is None else tokens[0]
    for t in range(T):
        if tokens is not None:
            cur = tokens[t]
        used[t] = cur
        u = E[cur].copy()  # [B][D]
        for l in range(M):
            z = gemv_bf16(params["W_in"][l], layer_norm(u))  # [B][3D]
            c = np.asarray(params["c"][l], np.float64)
            zc = short_conv([z, z_prev[l, 0], z_prev[l, 1]], c)
            z_prev[l, 1] = z_prev[l, 0]
            z_prev[l, 0] = z
            q, k, v = zc[:, :D], zc[:, D:2 * D], zc[:, 2 * D:]
            x_hist[l, t] = k * v
            # the long convolution by its definition: y_t = sum_{s<=t} h[t-s] x_s
            lag = h[l][:, t::-1][:, : t + 1]  # [D][t+1]: h[t-s] for s = 0..t
            y = np.einsum("tbd,dt->bd", x_hist[l, : t + 1], lag)
            y_all[l, t] = y
            r = u + q * y
            m = gemv_bf16(params["W2"][l], gelu(gemv_bf16(params["W1"][l], layer_norm(r))))
            u = r + m
        u_last[t] = u
        logits = gemv_bf16(params["W_lm"], layer_norm(u))
        if logits_all is not None:
            logits_all[t] = logits
        nxt[t] = np.argmax(logits, axis=-1)
        if tokens is None:
            cur = nxt[t]
    return {"logits": logits_all, "tokens": used, "next": nxt, "x": x_hist, "y": y_all, "u": u_last}

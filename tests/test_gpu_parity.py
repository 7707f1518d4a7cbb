"""Parity of the CUDA path (called through the C-ABI) with the CPU oracle.

Pass criteria: teacher-forced outputs within max-abs error 1e-4 * RMS(y) of the
oracle, per layer; closed-loop generation within 1e-3 relative over the first 4096
steps; schedules bit-exact.  Inputs come from the seeded generator module shared by
both sides; expected values come only from the oracle or from closed forms.
"""
import math
import os

import numpy as np
import pytest

import oracle
from long_convolution_sequence_b200 import synth

torch = pytest.importorskip("torch")
import long_convolution_sequence_b200 as fi  # noqa: E402

pytestmark = pytest.mark.gpu

TOL_TF = 1e-4   # teacher-forced: max |err| / RMS(y)
TOL_CL = 1e-3   # closed loop, first 4096 steps


def rel(got, ref):
    return float(np.abs(got - ref).max() / math.sqrt(float(np.mean(ref.astype(np.float64) ** 2))))


@pytest.fixture
def window(monkeypatch):
    def set_w(W):
        if W is None:
            monkeypatch.delenv("FI_WINDOW", raising=False)
        else:
            monkeypatch.setenv("FI_WINDOW", str(W))
    return set_w


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def read_layers(ctx, M, T, B, D):
    out = np.empty((M + 1, T, B, D), np.float32)
    for l in range(M + 1):
        ctx.read_layer(l, 0, T, out[l])
    return out


# ------------------------------------------------------------------ tau kernels
@pytest.mark.parametrize("U", [1 << q for q in range(0, 13)])
def test_tau_direct_matches_oracle(U):
    rng = np.random.default_rng(U)
    cnt = 5
    blocks = rng.standard_normal((cnt, U)).astype(np.float32)
    taps = rng.standard_normal((cnt, 2 * U + 3)).astype(np.float32)
    ref = oracle.tau(blocks, taps)
    out = torch.empty(cnt, U, device="cuda")
    fi.tau(fi.FI_TAU_DIRECT, U, dev(blocks), dev(taps), out)
    assert rel(out.cpu().numpy(), ref) < TOL_TF
    base = torch.ones(cnt, U, device="cuda")
    fi.tau(fi.FI_TAU_DIRECT, U, dev(blocks), dev(taps), base, accumulate=True)
    assert rel(base.cpu().numpy() - 1.0, ref) < TOL_TF


@pytest.mark.parametrize("U", [1 << q for q in range(3, 18)])
def test_tau_fft_matches_oracle(U):
    rng = np.random.default_rng(U + 1)
    cnt = 3
    blocks = rng.standard_normal((cnt, U)).astype(np.float32)
    taps = rng.standard_normal((cnt, 2 * U)).astype(np.float32)
    ref = oracle.tau(blocks, taps)
    out = torch.empty(cnt, U, device="cuda")
    fi.tau(fi.FI_TAU_FFT, U, dev(blocks), dev(taps), out)
    assert rel(out.cpu().numpy(), ref) < TOL_TF


# ------------------------------------------------------------------ block function
def test_tanh_of_the_red_cell_is_accurate():
    # one layer, h = delta_0: a^1_0 = tanh(x_0) for a sweep of x_0 values, on both the
    # per-token and the window path; absolute and relative accuracy
    grid = np.linspace(-12, 12, 4096)
    tiny = np.logspace(-30, 0, 2048)
    x = np.concatenate([grid, tiny, -tiny]).astype(np.float32)
    D = x.size
    for L in (2, 64):
        h = np.zeros((1, D, L), np.float32)
        h[0, :, 0] = 1.0
        with fi.FlashInference(1, 1, D, L, h) as ctx:
            xs = np.zeros((L, 1, D), np.float32)
            xs[0, 0] = x
            y = np.empty((L, 1, D), np.float32)
            ctx.forward(xs, L, y)
            a = np.empty((1, 1, D), np.float32)
            ctx.read_layer(1, 0, 1, a)
        # h_0 = 1 and nothing before token 0: the red cell is fma(1, x, 0) = x exactly, on
        # the per-token path (L = 2) and on the window path (L = 64, no residual at t = 0)
        np.testing.assert_array_equal(y[0, 0], x)
        ref = np.tanh(x.astype(np.float64))
        got = a[0, 0].astype(np.float64)
        assert np.abs(got - ref).max() < 5e-7
        nz = np.abs(ref) > 1e-30
        assert (np.abs(got - ref)[nz] / np.abs(ref[nz])).max() < 3e-6
        assert got[np.argmin(x)] == -1.0 and got[np.argmax(x)] == 1.0


# ------------------------------------------------------------------ schedule
def test_schedule_bit_exact_with_oracle():
    L = 1 << 12
    h = synth.filters(2, 3, L)
    with fi.FlashInference(2, 1, 3, L, h) as ctx:
        ref = oracle.schedule(L)
        for n, U, slo, shi, dlo, dhi in ref:
            s = ctx.schedule(int(n))
            assert (s["U"], s["src_lo"], s["dst_lo"], s["dst_hi"]) == (U, slo, dlo, dhi)
            assert s["impl"] in (fi.FI_TAU_DIRECT, fi.FI_TAU_FFT)


# ------------------------------------------------------------------ the stack
CASES_TF = [
    # M, B, D, L, W (None: library's choice)
    (3, 2, 5, 256, None),
    (2, 1, 3, 2048, 32),
    (4, 3, 7, 1024, 32),
    (1, 1, 16, 1024, 64),
    (2, 2, 33, 4096, 128),
    (2, 1, 5, 4096, 256),
    (18, 2, 3, 1024, 64),
    (36, 1, 2, 512, 64),
    (20, 1, 3, 512, 128),
]


@pytest.mark.parametrize("M,B,D,L,W", CASES_TF)
def test_teacher_forced_all_layers(M, B, D, L, W, window):
    window(W)
    h = synth.filters(M, D, L, seed=1)
    x = synth.inputs(L, B, D, seed=1)
    ref = oracle.stack(h, x, want=("y_all", "a_all"))
    with fi.FlashInference(M, B, D, L, h) as ctx:
        if W:
            assert ctx.info().window == W
        y = np.empty((L, B, D), np.float32)
        ctx.forward(x, L, y)
        assert rel(y, ref["y_all"][-1]) < TOL_TF
        a = read_layers(ctx, M, L, B, D)
    np.testing.assert_array_equal(a[0], x)
    for l in range(1, M + 1):
        # |tanh(u) - tanh(v)| <= |u - v|: the activation error is bounded by the y error
        rms = math.sqrt(float(np.mean(ref["y_all"][l - 1] ** 2)))
        assert np.abs(a[l] - np.tanh(ref["y_all"][l - 1])).max() < TOL_TF * rms, l


def test_window_launch_of_several_waves(window):
    # 18 layers, B = 4, D = 512 at W = 64: the rows of 4 channels per CTA do not fit in
    # shared memory, so the window launch holds 3 channels per CTA: 171 CTAs, more than
    # the SMs, in two waves
    M, B, D, L = 18, 4, 512, 512
    window(64)
    h = synth.filters(M, D, L, seed=4)
    x = synth.inputs(L, B, D, seed=4)
    ref = oracle.stack(h, x, want=("y_last",))
    with fi.FlashInference(M, B, D, L, h) as ctx:
        info = ctx.info()
        assert info.window == 64
        kch = info.chains_per_cta // B
        assert -(-D // kch) > info.sm_count
        y = np.empty((L, B, D), np.float32)
        ctx.forward(x, L, y)
    assert rel(y, ref["y_last"]) < TOL_TF


def test_closed_loop_on_a_window_launch_of_several_waves(window):
    # as above, two waves of 3-channel CTAs, now in the closed loop
    M, B, D, L = 18, 4, 512, 512
    window(64)
    h = synth.filters(M, D, L, seed=5)
    x0 = synth.start_token(B, D, seed=5)
    ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        assert ctx.info().window == 64
        out = np.empty((L, B, D), np.float32)
        ctx.generate(x0, L, out)
    assert rel(out, ref) < TOL_CL


@pytest.mark.parametrize("M,B,D,L,W", [(1, 1, 16, 1024, None), (3, 2, 6, 4096, 64), (18, 1, 8, 4096, None)])
def test_closed_loop_matches_oracle(M, B, D, L, W, window):
    window(W)
    h = synth.filters(M, D, L, seed=0)
    x0 = synth.start_token(B, D, seed=0)
    ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        out = np.empty((L, B, D), np.float32)
        ctx.generate(x0, L, out)
    n = min(L, 4096)
    assert rel(out[:n], ref[:n]) < TOL_CL


@pytest.mark.parametrize("graphs", [True, False])
def test_paths_and_call_splits_agree(graphs, window):
    window(32)
    M, B, D, L = 3, 2, 5, 1024
    h = synth.filters(M, D, L, seed=2)
    x = synth.inputs(L, B, D, seed=2)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_graphs(graphs)
        y = np.empty((L, B, D), np.float32)
        t = 0
        # windowed calls that start and stop inside windows, per-token steps, token path
        for kind, n in [("fwd", 5), ("step", 3), ("fwd", 40), ("tok", 17), ("fwd", 64), ("step", 1),
                        ("fwd", 300), ("tok", 90), ("fwd", L - 520)]:
            if kind == "step":
                for k in range(n):
                    ctx.step(x[t + k], y[t + k])
            else:
                ctx.set_path(fi.FI_PATH_TOKEN if kind == "tok" else fi.FI_PATH_WINDOW)
                ctx.forward(x[t:t + n], n, y[t:t + n])
            t += n
        assert t == L and ctx.info().t == L
    assert rel(y, ref) < TOL_TF


def test_generate_continues_across_calls_and_reset_repeats(window):
    window(64)
    M, B, D, L = 2, 1, 8, 2048
    h = synth.filters(M, D, L, seed=3)
    x0 = synth.start_token(B, D, seed=3)
    ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        out = np.empty((L, B, D), np.float32)
        ctx.generate(x0, 100, out[:100])
        ctx.set_path(fi.FI_PATH_TOKEN)
        ctx.generate(None, 29, out[100:129])
        ctx.set_path(fi.FI_PATH_WINDOW)
        ctx.generate(None, L - 129, out[129:])
        assert rel(out, ref) < TOL_CL
        runs = []
        for _ in range(2):  # a rewound context repeats itself bit for bit
            ctx.reset()
            again = np.empty_like(out)
            ctx.generate(x0, L, again)
            runs.append(again)
    np.testing.assert_array_equal(runs[0], runs[1])
    assert rel(runs[0], ref) < TOL_CL


@pytest.mark.parametrize("closed", [True, False])
def test_token_path_graphs_replay_the_eager_launches(closed):
    # the per-token path from one captured graph per block size must compute exactly
    # what the same launches issued from the host compute, and match the oracle
    M, B, D, L = 3, 2, 5, 2048
    h = synth.filters(M, D, L, seed=8)
    x0 = synth.start_token(B, D, seed=8)
    x = synth.inputs(L, B, D, seed=8)
    if closed:
        ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    else:
        ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    outs = []
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_path(fi.FI_PATH_TOKEN)
        for graphs in (True, False, True):
            ctx.reset()
            ctx.set_graphs(graphs)
            n0 = ctx.info().launches
            y = np.empty((L, B, D), np.float32)
            if closed:
                ctx.generate(x0, 700, y[:700])           # two calls: the step record is
                ctx.generate(None, L - 700, y[700:])      # set again by the second
            else:
                ctx.forward(x[:700], 700, y[:700])
                ctx.forward(x[700:], L - 700, y[700:])
            if graphs:
                # per token: the step kernel and the block launch unless the block is fused
                # into the step kernel (or the last token, which releases none); per call
                # one record write
                assert L + 2 <= ctx.info().launches - n0 <= L * 2 + 2
            outs.append(y)
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])
    assert rel(outs[0], ref) < (TOL_CL if closed else TOL_TF)


def test_step_calls_with_changing_pointers_replay_graphs():
    # fi_step: every call names new input and output buffers (device and host); the
    # replayed graphs read them from the step record
    M, B, D, L = 2, 1, 6, 512
    h = synth.filters(M, D, L, seed=9)
    x = synth.inputs(L, B, D, seed=9)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        xd = dev(x)
        yd = torch.empty((L, B, D), device="cuda")
        yh = np.empty((L, B, D), np.float32)
        for t in range(L):
            if t % 3 == 0:
                ctx.step(np.ascontiguousarray(x[t]), yh[t])
            else:
                ctx.step(xd[t], yd[t])
        torch.cuda.synchronize()
        got = yd.cpu().numpy()
        for t in range(0, L, 3):
            got[t] = yh[t]
        assert ctx.info().t == L
    assert rel(got, ref) < TOL_TF


@pytest.mark.parametrize("path", ["window", "token"])
def test_traced_runs_report_every_launch(path):
    # tracing brackets every launch with events, on the captured window path and on the
    # host-issued per-token path; the per-launch list covers the whole run, in order
    M, B, D, L = 3, 1, 8, 1024
    h = synth.filters(M, D, L, seed=10)
    x0 = synth.start_token(B, D, seed=10)
    ref = oracle.stack(h, x0, T=L, closed_loop=True, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        ctx.set_path(fi.FI_PATH_WINDOW if path == "window" else fi.FI_PATH_TOKEN)
        ctx.set_trace(True)
        out = np.empty((L, B, D), np.float32)
        n0 = ctx.info().launches
        ctx.generate(x0, L, out)
        n = ctx.info().launches - n0
        cls, q, us = ctx.trace_launches()
        assert len(cls) == n and (us > 0).all()
        if path == "token":
            assert (cls == fi.FI_K_TOKEN_STEP).sum() == L
        else:
            W = ctx.info().window
            assert (cls == fi.FI_K_WINDOW).sum() == L // W
            assert sorted(q[cls != fi.FI_K_WINDOW].tolist()) == sorted((k & -k).bit_length() - 1
                                                                    for k in range(W, L, W))
        per_class = ctx.trace()
        assert sum(v[0] for v in per_class.values()) == n
    assert rel(out, ref) < TOL_CL


@pytest.mark.parametrize("force", ["direct", "fft"])
def test_forced_tau_everywhere(force, window):
    window(32)
    M, B, D, L = 2, 1, 4, 1 << 13
    h = synth.filters(M, D, L, seed=4, decay=False)
    x = synth.inputs(L, B, D, seed=4)
    ref = oracle.stack(h, x, want=("y_last",))["y_last"]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        P = L.bit_length() - 1
        for q in range(P):
            if force == "direct" and q <= 12:
                ctx.set_tau(q, fi.FI_TAU_DIRECT)
            if force == "fft" and q >= 3:
                ctx.set_tau(q, fi.FI_TAU_FFT)
        for path in (fi.FI_PATH_WINDOW, fi.FI_PATH_TOKEN):
            ctx.reset()
            ctx.set_path(path)
            y = np.empty((L, B, D), np.float32)
            ctx.forward(x, L, y)
            assert rel(y, ref) < TOL_TF, path


def test_nondecaying_filters_exercise_every_block_size():
    # filters without decay make the largest blocks (FFT, split FFT at U = 2^15, 2^16)
    # contribute at full weight; one layer, two channels, the full 2^17 positions
    M, B, D, L = 1, 1, 2, 1 << 17
    h = synth.filters(M, D, L, seed=5, decay=False)
    x = synth.inputs(L, B, D, seed=5)
    ref = oracle.causal_conv_batch(h[0], np.ascontiguousarray(x[:, 0, :].T))  # [D][L]
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        ctx.forward(x, L, y)
    assert rel(y[:, 0, :].T, ref) < TOL_TF


def test_geometric_filter_closed_form_full_length():
    # h_k = g r^k  =>  y_t = r y_{t-1} + g x_t; long memory (r = 1 - 2^-12)
    M, B, D, L = 1, 1, 4, 1 << 17
    r = 1.0 - 2.0 ** -12
    g = np.array([0.5, -1.0, 0.25, 2.0])
    k = np.arange(L)
    h = (g[:, None] * r ** k[None, :]).astype(np.float32)[None]
    x = synth.inputs(L, B, D, seed=6)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        y = np.empty((L, B, D), np.float32)
        ctx.forward(x, L, y)
    state = np.zeros(D)
    ref = np.empty((L, D))
    xd = x[:, 0, :].astype(np.float64)
    for t in range(L):
        state = r * state + g * xd[t]
        ref[t] = state
    # float32 taps deviate from g r^k by <= 2^-24 |h_k|; bound their effect too
    bound = 2.0 ** -24 * np.abs(h[0].astype(np.float64)).sum(axis=1) * np.abs(xd).max()
    err = np.abs(y[:, 0, :] - ref)
    rms = np.sqrt(np.mean(ref ** 2))
    assert (err.max(axis=0) < TOL_TF * rms + bound).all()


# ------------------------------------------------------------------ errors
def test_capacity_and_argument_errors():
    M, B, D, L = 1, 1, 4, 16
    h = synth.filters(M, D, L)
    with fi.FlashInference(M, B, D, L, h) as ctx:
        out = np.empty((L + 1, B, D), np.float32)
        with pytest.raises(fi.FiError) as e:
            ctx.generate(None, 4, out)  # no start token at t = 0
        assert e.value.code == fi.FI_EINVAL
        with pytest.raises(fi.FiError) as e:
            ctx.generate(np.zeros((B, D), np.float32), L + 1, out)
        assert e.value.code == fi.FI_ECAPACITY
        ctx.generate(np.zeros((B, D), np.float32), L, out[:L])
        with pytest.raises(fi.FiError) as e:
            ctx.step(np.zeros((B, D), np.float32), out[0])
        assert e.value.code == fi.FI_ECAPACITY
        with pytest.raises(fi.FiError):
            ctx.read_layer(0, 0, L + 1, out)
        handle = ctx._h
    assert fi.get_lib().fi_reset(handle) == fi.FI_ESTATE  # destroyed


def test_injected_allocation_failure_leaves_no_context(monkeypatch):
    monkeypatch.setenv("FI_FAULT", "alloc")
    h = synth.filters(1, 4, 64)
    with pytest.raises(fi.FiError) as e:
        fi.FlashInference(1, 1, 4, 64, h)
    assert "injected" in str(e.value)
    monkeypatch.delenv("FI_FAULT")
    with fi.FlashInference(1, 1, 4, 64, h) as ctx:
        assert ctx.info().t == 0


def test_injected_capture_failure_reports_error(monkeypatch):
    h = synth.filters(1, 4, 256)
    with fi.FlashInference(1, 1, 4, 256, h) as ctx:
        monkeypatch.setenv("FI_FAULT", "capture")
        out = np.empty((256, 1, 4), np.float32)
        with pytest.raises(fi.FiError) as e:
            ctx.generate(np.ones((1, 4), np.float32), 256, out)
        assert e.value.code == fi.FI_ECUDA
        monkeypatch.delenv("FI_FAULT")
        ctx.generate(np.ones((1, 4), np.float32), 256, out)  # the context stays usable

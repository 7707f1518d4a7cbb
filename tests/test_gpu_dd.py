"""The long convolution with a data-dependent filter (fi_dd_*) against the oracle.

The oracle is the causal convolution by its definition (oracle.causal_conv_batch,
fp64 sums of the float32 inputs), which the online evaluation of the tiling
(oracle/dd.py) equals (tests/test_dd_schedule.py).  Tolerance as for the fixed
filter's teacher-forced parity: max |err| / RMS(y) < 1e-4 (fp32 products, FFT
rounding).  Both sequences arrive online; the closed-loop test derives x_{t+1} and
rho_{t+1} from y_t on the host, so nothing of either sequence exists before its step.
"""
import math

import numpy as np
import pytest

import long_convolution_sequence_b200 as fi
from long_convolution_sequence_b200 import synth
import oracle

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TOL = 1e-4


def rel(got, ref):
    return float(np.abs(got - ref).max() / math.sqrt(float(np.mean(ref.astype(np.float64) ** 2))))


def ref_of(x, rho):
    """y [T][G] = causal convolution of every channel's x with its rho (fp64)."""
    return oracle.causal_conv_batch(np.ascontiguousarray(rho.T), np.ascontiguousarray(x.T)).T


@pytest.mark.parametrize("G,L,tau", [(37, 1024, "default"), (5, 512, "direct"), (6, 2048, "fft"),
                                     (1, 2, "default"), (300, 4096, "default")])
def test_online_convolution_matches_oracle(G, L, tau):
    x, rho = synth.dd_inputs(L, G, seed=G + L)
    with fi.DataDependentConvolution(G, L) as dd:
        P = L.bit_length() - 1
        for q in range(P):
            if tau == "direct" and q <= 12:
                dd.set_tau(q, fi.FI_TAU_DIRECT)
            if tau == "fft" and q >= 3:
                dd.set_tau(q, fi.FI_TAU_FFT)
        y = np.empty((L, G), np.float32)
        dd.forward(x, rho, L, y)
    assert rel(y, ref_of(x, rho)) < TOL


def test_calls_split_anywhere_and_device_arrays():
    G, L = 19, 1024
    x, rho = synth.dd_inputs(L, G, seed=3)
    ref = ref_of(x, rho)
    with fi.DataDependentConvolution(G, L) as dd:
        y = np.empty((L, G), np.float32)
        cuts = [0, 1, 2, 3, 7, 64, 65, 300, 512, 1023, L]
        for a, b in zip(cuts[:-1], cuts[1:]):
            if a % 2:
                xd, rd = torch.from_numpy(x[a:b]).cuda(), torch.from_numpy(rho[a:b]).cuda()
                yd = torch.empty((b - a, G), device="cuda")
                dd.forward(xd, rd, b - a, yd)
                y[a:b] = yd.cpu().numpy()
            else:
                dd.forward(np.ascontiguousarray(x[a:b]), np.ascontiguousarray(rho[a:b]), b - a, y[a:b])
        assert rel(y, ref) < TOL
        with pytest.raises(fi.FiError) as e:
            dd.forward(x[:1], rho[:1], 1, y[:1])
        assert e.value.code == fi.FI_ECAPACITY
        with pytest.raises(fi.FiError) as e:
            dd.set_tau(5, fi.FI_TAU_DIRECT)
        assert e.value.code == fi.FI_ESTATE
        # a second sequence after reset
        dd.reset()
        x2, rho2 = synth.dd_inputs(L, G, seed=4)
        y2 = np.empty((L, G), np.float32)
        dd.forward(x2, rho2, L, y2)
        assert rel(y2, ref_of(x2, rho2)) < TOL


def test_roles_of_input_and_filter_are_symmetric_on_the_gpu():
    G, L = 8, 256
    x, rho = synth.dd_inputs(L, G, seed=9)
    ys = []
    for a, b in ((x, rho), (rho, x)):
        with fi.DataDependentConvolution(G, L) as dd:
            y = np.empty((L, G), np.float32)
            dd.forward(a, b, L, y)
            ys.append(y)
    assert rel(ys[0], ys[1]) < TOL


def test_closed_loop_both_sequences_made_from_the_outputs():
    # x_{t+1} = tanh(y_t + s_t), rho_{t+1} = 0.05 sin(3 y_t) exp(-t / 64): each step's
    # inputs exist only once the previous output is known (s_t: a fixed drive)
    G, L, T = 4, 256, 256
    drive = synth.dd_inputs(T, G, seed=11)[0]
    x0, r0 = np.ones(G, np.float32), np.full(G, 0.5, np.float32)

    def step_inputs(t, y_prev):
        if t == 0:
            return x0, r0
        xt = np.tanh(y_prev + drive[t]).astype(np.float32)
        rt = (0.05 * np.sin(3.0 * y_prev) * math.exp(-t / 64.0)).astype(np.float32)
        return xt, rt

    with fi.DataDependentConvolution(G, L) as dd:
        xs, rs, ys = [], [], []
        y_prev = None
        for t in range(T):
            xt, rt = step_inputs(t, y_prev)
            y = np.empty((1, G), np.float32)
            dd.forward(xt[None].copy(), rt[None].copy(), 1, y)
            xs.append(xt)
            rs.append(rt)
            ys.append(y[0])
            y_prev = y[0]
    x, rho, y = np.stack(xs), np.stack(rs), np.stack(ys)
    # the GPU's own realised inputs: its outputs are the causal convolution of them
    assert rel(y, ref_of(x, rho)) < TOL
    # and the fp64 closed loop of the same recurrence stays close over these steps
    xo, ro, yo = [], [], []
    y_prev = None
    for t in range(T):
        xt, rt = step_inputs(t, y_prev)
        xo.append(xt.astype(np.float64))
        ro.append(rt.astype(np.float64))
        X, R = np.stack(xo), np.stack(ro)
        yt = np.einsum("ig,ig->g", R[::-1], X)
        yo.append(yt)
        y_prev = yt.astype(np.float32)
    assert rel(y, np.stack(yo)) < 1e-3


def test_full_size_sampled_channels():
    # the bench's workload (18 x 864 channels, L = 2^17, inputs drawn on the device):
    # every output of 4 sampled channels over the first 8192 steps against the oracle
    G, L, T = 18 * 864, 1 << 17, 8192
    x, rho = synth.device_dd_inputs(L, G, seed=0)
    chans = [0, 1, 5000, G - 1]
    with fi.DataDependentConvolution(G, L) as dd:
        y = torch.empty((T, G), device="cuda")
        dd.forward(x[:T], rho[:T], T, y)
        torch.cuda.synchronize()
        got = y[:, chans].cpu().numpy()
    xs = x[:T, chans].cpu().numpy()
    rs = rho[:T, chans].cpu().numpy()
    assert rel(got, ref_of(xs, rs)) < TOL

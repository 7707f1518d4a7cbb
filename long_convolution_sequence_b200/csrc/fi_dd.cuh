// fi_dd.cuh -- device code of the long convolution with a data-dependent filter
// (sm_100a): one step's red cells with its blocks of U <= 8 (k_dd_step), and a whole
// aligned window of given steps with every block below the window's size folded in
// (k_dd_window).  The larger blocks are the tile kernels of fi_kernels.cuh (direct or
// FFT tau) with one layer of G channels: Algorithm 1's block with the input sequence's
// buffer as `act`, the other sequence's buffer as the taps `h`, and the running sums
// as `act_out`.
//
// The Flash Inference summary (section "Technische Innovationen", item 4,
// "Datenabhaengige Filter-Erweiterung") and the rebuttal's answer on data-dependent
// filters state that such a filter takes a different tiling with two FFT
// convolutions of the same size per step; the reading built here is documented in
// fi.h (fi_dd_create).
#pragma once

namespace fi {

// Step t for every channel g: x_t and rho_t join the buffers (x, rho [G][L]), and
// y_t = (running sum at t) + rho_0 x_t + rho_t x_0  (t > 0),  rho_0 x_0  (t = 0).
// The running sum holds every product rho_i x_j with i, j >= 1 and i + j = t, added by
// the blocks released after tokens 1 .. t.  With U > 0 the same thread then adds the
// blocks of size U released after token n = t + 1 (U = lowbit(n) <= 8, the direct
// tau): x[n - U, n) against rho[0, 2U) and, unless n is a power of two, rho[n - U, n)
// against x[0, 2U), onto the running sums [n, n + U) of its channel.  Its reads are
// its own channel's values, written by earlier steps or just now by this thread; at a
// power of two rho[U, 2U) is still zero, as the tiling needs.
template <int U>
__global__ void k_dd_step(float* __restrict__ xb, float* __restrict__ rb, float* __restrict__ acc,
                          const float* __restrict__ x_t, const float* __restrict__ rho_t, float* __restrict__ y_t,
                          long long t, int G, long long L) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= G) return;
    const long long row = (long long)g * L;
    const long long n = t + 1;
    // every load first, in one round trip: this step's values, the prefixes' first
    // values, the running sum at t and, with a block, its inputs, taps and outputs
    // (the value at position t is this step's own, taken from registers)
    const float xv = x_t[g], rv = rho_t[g];
    const float x0 = t == 0 ? xv : xb[row], r0 = t == 0 ? rv : rb[row];
    const float run = t == 0 ? 0.f : acc[row + t];
    constexpr int UU = U > 0 ? U : 1;
    float xi[UU], ri[UU], xp[2 * UU], rp[2 * UU], ao[UU];
    if (U > 0) {
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const long long pos = n - U + j;  // <= t
            xi[j] = pos == t ? xv : xb[row + pos];
            ri[j] = pos == t ? rv : rb[row + pos];
        }
#pragma unroll
        for (int k = 1; k < 2 * U; ++k) {
            // positions above t are still zero (the power-of-two case reads them)
            xp[k] = k == t ? xv : xb[row + k];
            rp[k] = k == t ? rv : rb[row + k];
        }
#pragma unroll
        for (int r = 0; r < U; ++r) ao[r] = acc[row + n + r];
    }
    y_t[g] = t == 0 ? rv * xv : fmaf(r0, xv, fmaf(rv, x0, run));
    xb[row + t] = xv;
    rb[row + t] = rv;
    if (U > 0) {
        const bool both = (n & (n - 1)) != 0;
#pragma unroll
        for (int r = 0; r < U; ++r) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < U; ++j) {
                s = fmaf(xi[j], rp[U + r - j], s);
                if (both) s = fmaf(ri[j], xp[U + r - j], s);
            }
            acc[row + n + r] = ao[r] + s;
        }
    }
}

// A whole aligned window [kW, kW + W) of steps at once, kW >= W, when its inputs are
// all given.  The blocks of size U < W released inside the window read and write only
// the window (Algorithm 1's window property), and together they add, for every pair of
// window positions j < t, x_j rho_{t-j} + rho_j x_{t-j}: the window's values against
// the prefixes' first W values (lags t - j < W <= kW, so the lag indices are prefix
// indices and never window ones).  With the running sums staged (the blocks released at
// or before kW), every output of the window is then
//   y_t = acc[t] + rho_0 x_t + rho_t x_0 + sum_{j=kW}^{t-1} (x_j rho_{t-j} + rho_j x_{t-j}),
// independent of the window's other outputs: no step has to wait for another.  The
// in-window blocks are not added to the running sums (they would only feed positions
// of this window, all final here).  One CTA: 32 channels x W steps; inputs x_in, rho_in
// and outputs y_out are [W][G] rows of the caller's arrays; x and rho also go to their
// [G][L] buffers for the blocks of U >= W.  Shared memory rows are padded to W + 1
// floats, so that the 32 channels of a warp (one step) read 32 different banks.
constexpr int kDdWinCh = 32;
constexpr int kDdWin = 128;
template <int W>
constexpr size_t dd_window_smem() { return sizeof(float) * 4 * kDdWinCh * (W + 1); }

template <int W>
__global__ void __launch_bounds__(256) k_dd_window(float* __restrict__ xb, float* __restrict__ rb,
                                                   const float* __restrict__ acc, const float* __restrict__ x_in,
                                                   const float* __restrict__ rho_in, float* __restrict__ y_out,
                                                   long long kW, int G, long long L) {
    constexpr int NT = 256, P = W + 1, C = kDdWinCh;
    extern __shared__ float dd_sm[];  // [4][C][W + 1]
    float(*sx)[P] = reinterpret_cast<float(*)[P]>(dd_sm);
    float(*sr)[P] = reinterpret_cast<float(*)[P]>(dd_sm + C * P);
    float(*px)[P] = reinterpret_cast<float(*)[P]>(dd_sm + 2 * C * P);
    float(*pr)[P] = reinterpret_cast<float(*)[P]>(dd_sm + 3 * C * P);
    const int g0 = blockIdx.x * C;
    const int nc = min(C, G - g0);
    const int tid = threadIdx.x;
    // the window's inputs, [W][G] rows: 32 channels of one step per warp (128 bytes)
    for (int e = tid; e < W * C; e += NT) {
        const int s = e / C, c = e - s * C;
        float xv = 0.f, rv = 0.f;
        if (c < nc) {
            xv = x_in[(long long)s * G + g0 + c];
            rv = rho_in[(long long)s * G + g0 + c];
        }
        sx[c][s] = xv;
        sr[c][s] = rv;
    }
    // the prefixes' first W values of every channel (positions 0 .. W-1 < kW)
    for (int e = tid; e < W * C; e += NT) {
        const int c = e / W, k = e - c * W;
        float xv = 0.f, rv = 0.f;
        if (c < nc) {
            xv = xb[(long long)(g0 + c) * L + k];
            rv = rb[(long long)(g0 + c) * L + k];
        }
        px[c][k] = xv;
        pr[c][k] = rv;
    }
    __syncthreads();
    // the window's values into the [G][L] buffers (row segments of W floats)
    for (int e = tid; e < W * C; e += NT) {
        const int c = e / W, k = e - c * W;
        if (c < nc) {
            xb[(long long)(g0 + c) * L + kW + k] = sx[c][k];
            rb[(long long)(g0 + c) * L + kW + k] = sr[c][k];
        }
    }
    // outputs: thread (c, jb) takes two blocks of 8 consecutive steps of channel c, jb and
    // 15 - jb (their triangles together as long as any other pair).  Per chunk of 8 lags
    // it holds the 15 window values of each sequence those lags reach and the 8 prefix
    // values: 46 shared-memory reads per 128 multiply-adds.  A lag past the row (only
    // beyond every step of the block, where the window value is taken as zero) is
    // clamped to the row's last entry.
    constexpr int QB = 8, NB = W / QB;
    static_assert(NT / C * 2 == NB, "two blocks of 8 steps per thread cover the window");
    const int c = tid % C, jb = tid / C;
    if (c < nc) {
        const long long row = (long long)(g0 + c) * L;
        const float x0 = px[c][0], r0 = pr[c][0];
        for (int half = 0; half < 2; ++half) {
            const int s0 = (half == 0 ? jb : NB - 1 - jb) * QB;
            float accq[QB];
#pragma unroll
            for (int q = 0; q < QB; ++q) accq[q] = 0.f;
            for (int l0 = 1; l0 <= s0 + QB - 1; l0 += 8) {
                float xv[QB + 7], rv[QB + 7], pl[8], xl[8];
#pragma unroll
                for (int m = 0; m < QB + 7; ++m) {
                    const int pos = s0 - l0 - 7 + m;  // window position s0 + q - (l0 + d), m = q - d + 7
                    xv[m] = pos >= 0 ? sx[c][pos] : 0.f;
                    rv[m] = pos >= 0 ? sr[c][pos] : 0.f;
                }
#pragma unroll
                for (int d = 0; d < 8; ++d) {
                    const int lg = min(l0 + d, W - 1);
                    pl[d] = pr[c][lg];
                    xl[d] = px[c][lg];
                }
#pragma unroll
                for (int d = 0; d < 8; ++d)
#pragma unroll
                    for (int q = 0; q < QB; ++q)
                        accq[q] = fmaf(xv[q - d + 7], pl[d], fmaf(rv[q - d + 7], xl[d], accq[q]));
            }
#pragma unroll
            for (int q = 0; q < QB; ++q) {
                const int s = s0 + q;
                const float v = fmaf(r0, sx[c][s], fmaf(sr[c][s], x0, acc[row + kW + s] + accq[q]));
                y_out[(long long)s * G + g0 + c] = v;
            }
        }
    }
}

}  // namespace fi

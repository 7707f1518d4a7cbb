// fi_dd.cuh -- device code of the long convolution with a data-dependent filter
// (sm_100a): the red cells of one step.  The blocks are the tile kernels of
// fi_kernels.cuh (direct or FFT tau) with one layer of G channels: Algorithm 1's block
// with the input sequence's buffer as `act`, the other sequence's buffer as the taps
// `h`, and the running sums as `act_out`.
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

}  // namespace fi

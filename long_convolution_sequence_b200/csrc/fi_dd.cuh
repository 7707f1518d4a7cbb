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
// the blocks released after tokens 1 .. t.
__global__ void k_dd_red(float* __restrict__ xb, float* __restrict__ rb, const float* __restrict__ acc,
                         const float* __restrict__ x_t, const float* __restrict__ rho_t, float* __restrict__ y_t,
                         long long t, int G, long long L) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= G) return;
    const long long row = (long long)g * L;
    const float xv = x_t[g], rv = rho_t[g];
    float y;
    if (t == 0) {
        y = rv * xv;
    } else {
        const float x0 = xb[row], r0 = rb[row], run = acc[row + t];
        y = fmaf(r0, xv, fmaf(rv, x0, run));
    }
    xb[row + t] = xv;
    rb[row + t] = rv;
    y_t[g] = y;
}

}  // namespace fi

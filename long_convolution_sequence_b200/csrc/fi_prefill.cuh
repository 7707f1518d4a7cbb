// fi_prefill.cuh -- element-wise kernels of the prompt prefill (fi_prefill): a prompt
// of p tokens is folded in layer by layer with one FFT convolution each instead of p
// online steps.  Layer l's pre-activations on the prompt are the causal convolution
//   y^l_t = sum_{j<=t} h^l[t-j] a^{l-1}_j,   t < p,
// which is the block tau of Lemma 1 ("Beitrags-Aggregations-Definition") with U >= p,
// the prompt as the block (zero past p) and the taps shifted by U: taps[m] = 0 for
// m < U and h^l[m - U] for m >= U, so that taps[U + t - j] = h^l[t - j] for j <= t and
// 0 for j > t.  All kernels are grid-stride loops over plain index ranges.
#pragma once

namespace fi {

// act[0][g][t] = x[t * G + g], t < p (the teacher-forced prompt)
__global__ void k_prefill_input(const float* __restrict__ x, long long G, long long L, int p, float* act) {
    const long long n = (long long)p * G;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const long long g = e % G, t = e / G;
        act[g * L + t] = x[e];
    }
}

// blocks[g][t] = act[layer][g][t] for t < p, 0 for p <= t < U
__global__ void k_prefill_gather(const float* __restrict__ act, int layer, long long G, long long L, int p, int U,
                                 float* blocks) {
    const long long n = G * U;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const long long g = e / U, t = e - g * U;
        blocks[e] = t < p ? act[((long long)layer * G + g) * L + t] : 0.f;
    }
}

// taps[g][m] = 0 for m < U, h[layer - 1][g % D][m - U] for U <= m < 2U
__global__ void k_prefill_taps(const float* __restrict__ h, int layer, int D, long long G, long long L, int U,
                               float* taps) {
    const long long n = G * 2 * U;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const long long g = e / (2 * U), m = e - g * 2 * U;
        taps[e] = m < U ? 0.f : h[((long long)(layer - 1) * D + g % D) * L + (m - U)];
    }
}

// act[layer][g][t] = tanh(out[g][t]) for t < p; y[t * G + g] = out[g][t] when y is given
__global__ void k_prefill_scatter(const float* __restrict__ out, int layer, long long G, long long L, int p, int U,
                                  float* act, float* y) {
    const long long n = (long long)p * G;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const long long g = e % G, t = e / G;
        const float v = out[g * U + t];
        act[((long long)layer * G + g) * L + t] = act_tanh(v);
        if (y) y[e] = v;
    }
}

// copy positions [t0, t1) of every row of layers 1..M between act and buf
// ([M][G][t1 - t0]); to_buf selects the direction
__global__ void k_prefill_rows(float* act, float* buf, int M, long long G, long long L, int t0, int t1, int to_buf) {
    const long long w = t1 - t0, n = (long long)M * G * w;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const long long r = e / w, t = t0 + (e - r * w);
        float* a = act + (G + r) * L + t;  // row r of layers 1..M starts after layer 0's G rows
        if (to_buf) buf[e] = *a;
        else *a = buf[e];
    }
}

}  // namespace fi

// fi_fft.cuh -- register-resident FFT convolution of gray blocks (sm_100a).
//
// One gray block ("tile") of edge U for one (layer, chain): outputs [n, n+U) gain
// tau(inputs [n-U, n)) = the samples [U, 2U) of the 2U-point circular convolution of
// [block, 0^U] with filter taps [0, 2U)  (section "Zirkulaere Faltungs-Trick" of the
// Flash Inference paper summary; tau is Lemma 1 of section
// "Beitrags-Aggregations-Definition").
//
// The 2U real samples are packed as N = U complex points z[m] = x[2m] + i x[2m+1]
// (z[m] = 0 for m >= N/2).  One tile runs:
//   forward  Z = DFT_N(z)                      Stockham passes, radix 16 (+ one radix R0)
//   multiply Q[k] from Z[k], Z[N-k] and the     the real 2N-point spectrum of the block,
//            precomputed filter spectrum H      times H, re-packed for a complex inverse
//   inverse  F = DFT_N(Q),  y[2m] = Re F[m],    only m >= N/2 is computed in the last pass
//            y[2m+1] = -Im F[m]                 and added straight onto the outputs
// Each thread owns E = 16 * B16 points; a pass reads its radix-16 butterflies from
// shared memory, applies twiddles, runs the 16-point DFT in registers and writes the
// results back.  The last forward pass and the first inverse pass use the same
// butterflies, so the thread keeps them in registers across the spectral multiply;
// only the partner values Z[N-k] come from shared memory.
//
// Spectral multiply.  With a = Z[k], b = Z[N-k], w = e^{-i pi k/N} = (c, -s), the real
// spectrum of the block is X[k] = ((a + conj b) - i w (a - conj b)) / 2 and the
// re-packed product for the inverse, conjugated, is linear in conj(a) and b:
//   Q[k] = conj(a) (|1-iw|^2 conj H[k] + |1+iw|^2 H[N-k]) / 4
//        + b ((1-iw) conj(1+iw) conj H[k] + (1+iw) conj(1-iw) H[N-k]) / 4,
// and |1-iw|^2 = 2 - 2s, |1+iw|^2 = 2 + 2s, (1-iw) conj(1+iw) = -2ic, so
//   Q[k] = conj(a) (S + s D) + b (i c D),  S = H'[N-k] + conj H'[k], D = H'[N-k] - conj H'[k]
// with H' = H / (2N): the stored spectrum carries the 1/2 and the 1/N of the
// inverse, so no other scaling appears in the kernel.
#pragma once
#include <cuda_runtime.h>

namespace fi {
namespace fft {

constexpr float kC16 = 0.92387953251128674f;  // cos(pi/8)
constexpr float kS16 = 0.38268343236508978f;  // sin(pi/8)
constexpr float kH2 = 0.70710678118654752f;   // sqrt(1/2)

// e^{-2 pi i m / 32}, m = 0..15
__device__ __forceinline__ float2 w32(int m) {
    switch (m) {
        case 0: return make_float2(1.f, 0.f);
        case 1: return make_float2(0.98078528040323043f, -0.19509032201612825f);
        case 2: return make_float2(kC16, -kS16);
        case 3: return make_float2(0.83146961230254524f, -0.55557023301960218f);
        case 4: return make_float2(kH2, -kH2);
        case 5: return make_float2(0.55557023301960218f, -0.83146961230254524f);
        case 6: return make_float2(kS16, -kC16);
        case 7: return make_float2(0.19509032201612825f, -0.98078528040323043f);
        case 8: return make_float2(0.f, -1.f);
        case 9: return make_float2(-0.19509032201612825f, -0.98078528040323043f);
        case 10: return make_float2(-kS16, -kC16);
        case 11: return make_float2(-0.55557023301960218f, -0.83146961230254524f);
        case 12: return make_float2(-kH2, -kH2);
        case 13: return make_float2(-0.83146961230254524f, -0.55557023301960218f);
        case 14: return make_float2(-kC16, -kS16);
        default: return make_float2(-0.98078528040323043f, -0.19509032201612825f);
    }
}

__device__ __forceinline__ float2 cm(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 ca(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 cs(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 mul_mi(float2 a) { return make_float2(a.y, -a.x); }  // a * (-i)
__device__ __forceinline__ float2 mul_pi(float2 a) { return make_float2(-a.y, a.x); }  // a * (+i)
// a * e^{-i pi/4} = a (1 - i) / sqrt 2,  a * e^{-3 i pi/4} = a (-1 - i) / sqrt 2
__device__ __forceinline__ float2 mul_w8_1(float2 a) { return make_float2(kH2 * (a.x + a.y), kH2 * (a.y - a.x)); }
__device__ __forceinline__ float2 mul_w8_3(float2 a) { return make_float2(kH2 * (a.y - a.x), -kH2 * (a.x + a.y)); }

// forward 4-point DFT in place, natural order
__device__ __forceinline__ void dft4(float2& a0, float2& a1, float2& a2, float2& a3) {
    const float2 s02 = ca(a0, a2), d02 = cs(a0, a2), s13 = ca(a1, a3), d13 = mul_mi(cs(a1, a3));
    a0 = ca(s02, s13);
    a2 = cs(s02, s13);
    a1 = ca(d02, d13);
    a3 = cs(d02, d13);
}

// Forward R-point DFT of v[0..R-1]: X[m] = sum_r v[r] e^{-2 pi i r m / R}.  The
// result X[m] is left in v[omap<R>(m)].
//  R = 16 = 4 x 4: r = 4 r1 + r0, m = m0 + 4 m1; 4-point DFTs over r1, twiddles
//          W16^{r0 m0}, 4-point DFTs over r0; X[m0 + 4 m1] lands in v[4 m0 + m1].
//  R = 8 = 4 x 2:  r = 2 r1 + r0, m = m0 + 4 m1; X[m0 + 4 m1] lands in v[2 m0 + m1].
template <int R>
__device__ __forceinline__ constexpr int omap(int m) {
    return R == 16 ? 4 * (m & 3) + (m >> 2) : (R == 8 ? 2 * (m & 3) + (m >> 2) : m);
}

template <int R>
__device__ __forceinline__ void dft(float2* v) {
    if constexpr (R == 1) {
    } else if constexpr (R == 2) {
        const float2 a = v[0], b = v[1];
        v[0] = ca(a, b);
        v[1] = cs(a, b);
    } else if constexpr (R == 4) {
        dft4(v[0], v[1], v[2], v[3]);
    } else if constexpr (R == 8) {
        dft4(v[0], v[2], v[4], v[6]);
        dft4(v[1], v[3], v[5], v[7]);
        v[3] = mul_w8_1(v[3]);
        v[5] = mul_mi(v[5]);
        v[7] = mul_w8_3(v[7]);
#pragma unroll
        for (int m0 = 0; m0 < 4; ++m0) {
            const float2 a = v[2 * m0], b = v[2 * m0 + 1];
            v[2 * m0] = ca(a, b);
            v[2 * m0 + 1] = cs(a, b);
        }
    } else {
        static_assert(R == 16, "radix");
#pragma unroll
        for (int r0 = 0; r0 < 4; ++r0) dft4(v[r0], v[r0 + 4], v[r0 + 8], v[r0 + 12]);
        // twiddles W16^{r0 m0} on v[r0 + 4 m0]
        v[5] = cm(v[5], make_float2(kC16, -kS16));    // W^1
        v[9] = mul_w8_1(v[9]);                         // W^2
        v[13] = cm(v[13], make_float2(kS16, -kC16));  // W^3
        v[6] = mul_w8_1(v[6]);                         // W^2
        v[10] = mul_mi(v[10]);                         // W^4
        v[14] = mul_w8_3(v[14]);                       // W^6
        v[7] = cm(v[7], make_float2(kS16, -kC16));    // W^3
        v[11] = mul_w8_3(v[11]);                       // W^6
        v[15] = cm(v[15], make_float2(-kC16, kS16));  // W^9
#pragma unroll
        for (int m0 = 0; m0 < 4; ++m0) dft4(v[4 * m0], v[4 * m0 + 1], v[4 * m0 + 2], v[4 * m0 + 3]);
    }
}

// Shared-memory position of complex element i: one pad entry after every 16, which
// makes the stride-R stores of the first passes bank-conflict free.
__device__ __forceinline__ int pad(int i) { return i + (i >> 4); }

// Twiddle table e^{-2 pi i j / 2^TWLOG}.
template <int TWLOG>
__device__ __forceinline__ float2 tw_at(const float2* __restrict__ tw, int j) {
    return __ldg(&tw[j & ((1 << TWLOG) - 1)]);
}

// v[r] *= W^{r k}, r = 1..R-1, with W = e^{-2 pi i / 2^logRNs}: two table entries
// (W^k, W^{4k}) and products of depth <= 3, applied as they are formed so that
// only a few twiddles are live at a time.
template <int R, int TWLOG>
__device__ __forceinline__ void apply_twiddles(float2* v, const float2* __restrict__ tw, int logRNs, int k) {
    const int sh = TWLOG - logRNs;
    const float2 w1 = tw_at<TWLOG>(tw, k << sh);
    v[1] = cm(v[1], w1);
    if constexpr (R >= 4) {
        const float2 w2 = cm(w1, w1);
        const float2 w3 = cm(w2, w1);
        v[2] = cm(v[2], w2);
        v[3] = cm(v[3], w3);
        if constexpr (R >= 8) {
            const float2 w4 = tw_at<TWLOG>(tw, (4 * k) << sh);
            v[4] = cm(v[4], w4);
            v[5] = cm(v[5], cm(w4, w1));
            v[6] = cm(v[6], cm(w4, w2));
            v[7] = cm(v[7], cm(w4, w3));
            if constexpr (R == 16) {
                const float2 w8 = cm(w4, w4);
                v[8] = cm(v[8], w8);
                v[9] = cm(v[9], cm(w8, w1));
                v[10] = cm(v[10], cm(w8, w2));
                v[11] = cm(v[11], cm(w8, w3));
                const float2 w12 = cm(w8, w4);
                v[12] = cm(v[12], w12);
                v[13] = cm(v[13], cm(w12, w1));
                v[14] = cm(v[14], cm(w12, w2));
                v[15] = cm(v[15], cm(w12, w3));
            }
        }
    }
}

// Stockham pass of radix R at sub-transform size Ns = 2^logNs over N = 2^LOGN points:
// butterfly b reads X[b + r N/R], twiddles by W_{R Ns}^{r (b mod Ns)}, runs the R-point
// DFT and writes output m to X[(b - b mod Ns) R + b mod Ns + m Ns].  This thread does
// butterflies b = t + u T, u < BPT.  v receives the outputs (element m of butterfly u
// in v[u][omap<R>(m)]).  Reads, barrier, writes, barrier.
template <int LOGN, int R, int BPT, int TWLOG>
__device__ __forceinline__ void pass(float2* X, float2 (*v)[R], int t, int T, int logNs,
                                     const float2* __restrict__ tw) {
    constexpr int N = 1 << LOGN, NB = N / R;
    constexpr int LOGR = R == 16 ? 4 : (R == 8 ? 3 : (R == 4 ? 2 : (R == 2 ? 1 : 0)));
    const int Ns = 1 << logNs;
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
        const int b = t + u * T;
#pragma unroll
        for (int r = 0; r < R; ++r) v[u][r] = X[pad(b + r * NB)];
    }
    if (Ns > 1) {
#pragma unroll
        for (int u = 0; u < BPT; ++u) apply_twiddles<R, TWLOG>(v[u], tw, logNs + LOGR, (t + u * T) & (Ns - 1));
    }
#pragma unroll
    for (int u = 0; u < BPT; ++u) dft<R>(v[u]);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
        const int b = t + u * T;
        const int k = b & (Ns - 1);
        const int base = (b - k) * R + k;
#pragma unroll
        for (int m = 0; m < R; ++m) X[pad(base + m * Ns)] = v[u][omap<R>(m)];
    }
    __syncthreads();
}

}  // namespace fft
}  // namespace fi

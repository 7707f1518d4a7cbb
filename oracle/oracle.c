/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the Flash Inference mixer stack.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may include, link, load or call this file.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * Source of every definition below: the web summary of arXiv 2410.12982,
 * "Flash Inference: Near Linear Time Inference for Long Convolution Sequence
 * Models and Beyond" (Oncescu, Purandare, Idreos, Kakade), cited by section
 * heading of that page:
 *   [Aufgabendefinition]            z_t = sum_{i<=t} y_i * rho_{t-i}, per channel
 *   [LCSM-spezifische Definition]   mixer^l(y)_t = sum_{i<=t} y_i (.) rho^l_{t-i}
 *   [Modellarchitektur]             a^l_i = block^l(mixer^l(a^{l-1})_i)
 *   [Drei Berechnungsstrategien]    the Lazy strategy: z_t computed when needed
 *   [Beitrags-Aggregations-Definition] tau(y,[l,r],rho,[l',r'])_t = sum_{i=l}^{r} y_i rho_{t-i}
 *   [Kachelung-Strategie (Algorithmus 1)] U = largest power of two dividing i,
 *                                   red cell, then gray block onto [i+1, i+U]
 *   [LCSM-Inferenz-Algorithmus (Algorithmus 2)] the same over M layers, with
 *                                   a^l_i = block^l(b^l_i) and a^0_{i+1} = sampler(a^M_i)
 *
 * Readings (the pages leave these open):
 *   - Positions are stored 0-based: token t = 0..T-1.  The pages' 1-based loop
 *     counter i is the count n = t + 1 of tokens already finalised; the gray block
 *     released after token t reads inputs [n-U, n-1] and writes outputs [n, n+U-1]
 *     with U = lowbit(n).
 *   - block^l = tanh and sampler = tanh (the synthetic mixer stack being measured);
 *     "y" returned to callers is the pre-tanh mixer output of a layer.
 *   - Filters have length >= T; filter l, channel c is h[(l*D + c)*ldh + k].
 *   - Closed loop: a^0_{t+1} = a^M_t = tanh(y^M_t).
 *
 * Pins (checked by the CPU tests, never by this file): numpy.convolve and
 * numpy.fft on small inputs, closed forms (delta, shifted delta, geometric and
 * constant filters), the lowbit schedule counts of Proposition 1, brute-force
 * pair coverage, the circular-window identity.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL -1
#define ORC_ENOMEM -3

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* [Aufgabendefinition] / [Drei Berechnungsstrategien]: the lazy causal
 * convolution of one sequence, z_t = sum_{s=0}^{t} h[t-s] * y[s], in fp64.    */
void orc_causal_conv(int64_t T, const double *h, const double *y, double *z) {
    for (int64_t t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int64_t s = 0; s <= t; ++s) acc += h[t - s] * y[s];
        z[t] = acc;
    }
}

/* Batched version over independent channels (OpenMP), float inputs:
 * z[c][t] = sum_{s<=t} h[c][t-s] * y[c][s]; h has leading dimension ldh.        */
void orc_causal_conv_batch(int64_t C, int64_t T, int64_t ldh, const float *h,
                           const float *y, double *z) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < C; ++c) {
        const float *hc = h + c * ldh;
        const float *yc = y + c * T;
        double *zc = z + c * T;
        for (int64_t t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int64_t s = 0; s <= t; ++s) acc += (double)hc[t - s] * (double)yc[s];
            zc[t] = acc;
        }
    }
}

/* Single sampled output: z_t for one sequence (used for spot checks at full size). */
double orc_conv_at(int64_t t, const float *h, const float *y, int64_t ystride) {
    double acc = 0.0;
    for (int64_t s = 0; s <= t; ++s) acc += (double)h[t - s] * (double)y[s * ystride];
    return acc;
}

/* ------------------------------------------------------------------------- */
/* [LCSM-Inferenz-Algorithmus (Algorithmus 2)] evaluated lazily: the plain
 * definition of the whole stack, position by position, layer by layer.
 *
 *   for t in 0..T-1:
 *     a^0_t = x_t (teacher-forced) | x0 if t == 0 else a^M_{t-1} (closed loop)
 *     for l in 1..M:  y^l_t = sum_{s<=t} h^l[t-s] a^{l-1}_s ;  a^l_t = tanh(y^l_t)
 *
 * h: [M][D][ldh] float.  x: teacher [T][B][D], closed loop [B][D].
 * y_all: [M][T][B][D] or NULL.  y_last: [T][B][D] or NULL (layer M only).
 * a_all: [M+1][T][B][D] or NULL (layer 0 = the realised input sequence).
 * fp32 != 0 runs the same definition with float accumulation and tanhf (used only
 * to measure how fast a float evaluation drifts away from the fp64 one).          */
int orc_stack(int M, int B, int D, int64_t T, int64_t ldh, const float *h,
              int closed_loop, const float *x, double *y_all, double *y_last,
              double *a_all, int fp32) {
    if (M < 1 || B < 1 || D < 1 || T < 1 || ldh < T || !h || !x) return ORC_EINVAL;
    const int64_t BD = (int64_t)B * D;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t g = 0; g < BD; ++g) {
        const int c = (int)(g % D);
        double *a = NULL;
        float *af = NULL;
        if (fp32) af = (float *)malloc(sizeof(float) * (size_t)(M + 1) * (size_t)T);
        else a = (double *)malloc(sizeof(double) * (size_t)(M + 1) * (size_t)T);
        if (!a && !af) {
#pragma omp atomic write
            err = ORC_ENOMEM;
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            double in;
            if (!closed_loop) in = x[t * BD + g];
            else if (t == 0) in = x[g];
            else in = fp32 ? (double)af[(int64_t)M * T + t - 1] : a[(int64_t)M * T + t - 1];
            if (fp32) af[t] = (float)in; else a[t] = in;
            if (a_all) a_all[t * BD + g] = fp32 ? (double)(float)in : in;
            for (int l = 1; l <= M; ++l) {
                const float *hl = h + ((int64_t)(l - 1) * D + c) * ldh;
                double y;
                if (fp32) {
                    const float *prev = af + (int64_t)(l - 1) * T;
                    float acc = 0.0f;
                    for (int64_t s = 0; s <= t; ++s) acc += hl[t - s] * prev[s];
                    af[(int64_t)l * T + t] = tanhf(acc);
                    y = acc;
                } else {
                    const double *prev = a + (int64_t)(l - 1) * T;
                    double acc = 0.0;
                    for (int64_t s = 0; s <= t; ++s) acc += (double)hl[t - s] * prev[s];
                    a[(int64_t)l * T + t] = tanh(acc);
                    y = acc;
                }
                if (y_all) y_all[((int64_t)(l - 1) * T + t) * BD + g] = y;
                if (l == M && y_last) y_last[t * BD + g] = y;
                if (a_all)
                    a_all[((int64_t)l * T + t) * BD + g] =
                        fp32 ? (double)af[(int64_t)l * T + t] : a[(int64_t)l * T + t];
            }
        }
        free(a);
        free(af);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* [Kachelung-Strategie (Algorithmus 1)] schedule.  For n = 1..L-1 (the pages'
 * loop counter i): U = largest power of two dividing n; the gray block reads
 * inputs [n-U, n-1] and writes outputs [n, n+U-1], clipped to L-1.  Returns the
 * number of entries (L-1).  Arrays may be NULL.                                  */
int64_t orc_schedule(int64_t L, int64_t *n_out, int64_t *U_out, int64_t *src_lo,
                     int64_t *src_hi, int64_t *dst_lo, int64_t *dst_hi) {
    int64_t k = 0;
    for (int64_t n = 1; n <= L - 1; ++n, ++k) {
        /* largest power of two dividing n, found by repeated halving */
        int64_t U = 1;
        while ((n % (2 * U)) == 0) U *= 2;
        int64_t hi = n + U - 1;
        if (hi > L - 1) hi = L - 1;
        if (n_out) n_out[k] = n;
        if (U_out) U_out[k] = U;
        if (src_lo) src_lo[k] = n - U;
        if (src_hi) src_hi[k] = n - 1;
        if (dst_lo) dst_lo[k] = n;
        if (dst_hi) dst_hi[k] = hi;
    }
    return k;
}

/* ------------------------------------------------------------------------- */
/* [Beitrags-Aggregations-Definition]: tau for one gray block of edge U, written
 * out directly.  With the block b_j = y_{n-U+j} (j < U) and output row r (r < U)
 * standing for position n+r, tau_r = sum_j b_j * rho_{(n+r)-(n-U+j)}
 *                                  = sum_j b_j * rho_{U+r-j}.
 * blocks: [count][U] float, taps: [count][ldt] float (rho_0 .. rho_{2U-1} at least),
 * out: [count][U] double.                                                          */
void orc_tau(int64_t U, int64_t count, const float *blocks, int64_t ldt,
             const float *taps, double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const float *b = blocks + i * U;
        const float *rho = taps + i * ldt;
        for (int64_t r = 0; r < U; ++r) {
            double acc = 0.0;
            for (int64_t j = 0; j < U; ++j) acc += (double)b[j] * (double)rho[U + r - j];
            out[i * U + r] = acc;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* [LCSM-Inferenz-Algorithmus (Algorithmus 2)] simulated on the CPU exactly as
 * the pages order it, with tau evaluated directly (fp64): per token, red cells in
 * layer order, then every layer's gray block.  One buffer per layer: the slot of
 * position s first accumulates b^l_s and is then overwritten by a^l_s
 * ([Speicheroptimierung], activation reuse).  Same argument conventions as
 * orc_stack; the capacity of the buffers is T (blocks are clipped to T-1).        */
int orc_relaxed_stack(int M, int B, int D, int64_t T, int64_t ldh, const float *h,
                      int closed_loop, const float *x, double *y_all) {
    if (M < 1 || B < 1 || D < 1 || T < 1 || ldh < T || !h || !x) return ORC_EINVAL;
    const int64_t BD = (int64_t)B * D;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t g = 0; g < BD; ++g) {
        const int c = (int)(g % D);
        double *buf = (double *)calloc((size_t)(M + 1) * (size_t)T, sizeof(double));
        if (!buf) {
#pragma omp atomic write
            err = ORC_ENOMEM;
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            /* token t enters layer 0 */
            if (!closed_loop) buf[t] = x[t * BD + g];
            else if (t == 0) buf[0] = x[g];
            else buf[t] = buf[(int64_t)M * T + t - 1];
            /* red cells, sequential in l */
            for (int l = 1; l <= M; ++l) {
                const float *hl = h + ((int64_t)(l - 1) * D + c) * ldh;
                double y = buf[(int64_t)l * T + t] + (double)hl[0] * buf[(int64_t)(l - 1) * T + t];
                buf[(int64_t)l * T + t] = tanh(y);
                if (y_all) y_all[((int64_t)(l - 1) * T + t) * BD + g] = y;
            }
            /* gray blocks released after token t: n = t + 1 */
            int64_t n = t + 1;
            if (n >= T) continue;
            int64_t U = 1;
            while ((n % (2 * U)) == 0) U *= 2;
            for (int l = 1; l <= M; ++l) {
                const float *hl = h + ((int64_t)(l - 1) * D + c) * ldh;
                const double *in = buf + (int64_t)(l - 1) * T;
                double *out = buf + (int64_t)l * T;
                for (int64_t r = 0; r < U && n + r < T; ++r) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < U; ++j) acc += in[n - U + j] * (double)hl[U + r - j];
                    out[n + r] += acc;
                }
            }
        }
        free(buf);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Own fp64 FFT (iterative radix-2, decimation in time, bit-reversed input order).
 * Used for the whole-sequence zero-padded FFT convolution pin and for reference
 * filter spectra.  sign = -1: forward, e^{-2 pi i k m / N}; sign = +1: inverse
 * without the 1/N factor.  N must be a power of two.                                */
int orc_fft(int64_t N, double *re, double *im, int sign) {
    if (N < 1 || (N & (N - 1))) return ORC_EINVAL;
    /* bit-reversal permutation */
    for (int64_t i = 1, j = 0; i < N; ++i) {
        int64_t bit = N >> 1;
        for (; j & bit; bit >>= 1) j ^= bit;
        j ^= bit;
        if (i < j) {
            double tr = re[i]; re[i] = re[j]; re[j] = tr;
            double ti = im[i]; im[i] = im[j]; im[j] = ti;
        }
    }
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t len = 2; len <= N; len <<= 1) {
        int64_t half = len >> 1;
        for (int64_t k = 0; k < half; ++k) {
            double ang = sign * two_pi * (double)k / (double)len;
            double wr = cos(ang), wi = sin(ang);
            for (int64_t s = 0; s < N; s += len) {
                int64_t p = s + k, q = s + k + half;
                double xr = re[q] * wr - im[q] * wi;
                double xi = re[q] * wi + im[q] * wr;
                re[q] = re[p] - xr; im[q] = im[p] - xi;
                re[p] += xr; im[p] += xi;
            }
        }
    }
    return ORC_OK;
}

/* Lemma 1 route for a whole sequence: causal convolution of y (length T) with
 * h (length >= T) through a zero-padded FFT of size N >= 2T; z has length T.      */
int orc_fft_conv(int64_t T, const double *h, const double *y, double *z) {
    int64_t N = 1;
    while (N < 2 * T) N <<= 1;
    double *ar = calloc((size_t)N, sizeof(double)), *ai = calloc((size_t)N, sizeof(double));
    double *br = calloc((size_t)N, sizeof(double)), *bi = calloc((size_t)N, sizeof(double));
    if (!ar || !ai || !br || !bi) { free(ar); free(ai); free(br); free(bi); return ORC_ENOMEM; }
    for (int64_t i = 0; i < T; ++i) { ar[i] = y[i]; br[i] = h[i]; }
    orc_fft(N, ar, ai, -1);
    orc_fft(N, br, bi, -1);
    for (int64_t k = 0; k < N; ++k) {
        double r = ar[k] * br[k] - ai[k] * bi[k];
        double i = ar[k] * bi[k] + ai[k] * br[k];
        ar[k] = r; ai[k] = i;
    }
    orc_fft(N, ar, ai, +1);
    for (int64_t t = 0; t < T; ++t) z[t] = ar[t] / (double)N;
    free(ar); free(ai); free(br); free(bi);
    return ORC_OK;
}

/* [Speicheroptimierung] FFT precompute: the DFT of the first 2U filter taps,
 * H_U[k] = sum_{m<2U} rho_m e^{-2 pi i k m / 2U} for k = 0..U (the non-redundant
 * half of a real signal's spectrum).  taps: [count][ldt] float starting at the
 * desired first tap; out_re/out_im: [count][U+1].                                  */
int orc_filter_spectrum(int64_t U, int64_t count, const float *taps, int64_t ldt,
                        double *out_re, double *out_im) {
    const int64_t N = 2 * U;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < count; ++i) {
        double *re = malloc(sizeof(double) * (size_t)N), *im = calloc((size_t)N, sizeof(double));
        if (!re || !im) {
            free(re); free(im);
#pragma omp atomic write
            err = ORC_ENOMEM;
            continue;
        }
        for (int64_t m = 0; m < N; ++m) re[m] = (double)taps[i * ldt + m];
        orc_fft(N, re, im, -1);
        for (int64_t k = 0; k <= U; ++k) {
            out_re[i * (U + 1) + k] = re[k];
            out_im[i * (U + 1) + k] = im[k];
        }
        free(re); free(im);
    }
    return err;
}

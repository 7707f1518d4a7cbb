// fi_kernels.cuh -- device code of the B200 Flash Inference mixer (sm_100a).
//
// Notation (web summary of arXiv 2410.12982, "Flash Inference: Near Linear Time
// Inference for Long Convolution Sequence Models and Beyond"):
//   * section "LCSM-spezifische Definition": y^l_t = sum_{s<=t} h^l[c][t-s] a^{l-1}_s
//   * section "Kachelung-Strategie (Algorithmus 1)": after the n-th token (n = t+1)
//     the gray block of edge U = lowbit(n) adds tau of inputs [n-U, n-1] onto
//     outputs [n, n+U-1]; the red cell adds h_0 a_t onto y_t.
//   * section "LCSM-Inferenz-Algorithmus (Algorithmus 2)": layers in order,
//     block = tanh, sampler = tanh.
//   * section "Speicheroptimierung": one buffer per layer; position s holds the
//     running sum b^l_s until token s is processed, then a^l_s.
//   * section "Zirkulaere Faltungs-Trick": a block is a 2U-point circular
//     convolution whose outputs [U, 2U-1] are free of wrap-around.
//
// Storage ("act"): [(M+1)][G][L] fp32, G = B*D chains (g = b*D + c), layer 0 holds
// the input sequence.  Filters ("h"): [M][D][L] fp32.  Spectra: per block size,
// [M][D][nspec][N+1] complex64.
//
// First-writer rule: the block released after token n = 2^p is the first one to
// touch positions [2^p, 2^(p+1)-1]; it stores with "=" and every later block
// accumulates.  Position 0 is never written by a block; its running sum is 0.
// Hence no buffer ever needs clearing, and rewinding a context is O(1).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "fi_fft.cuh"

namespace fi {

// ----------------------------------------------------------------- utilities
__host__ __device__ __forceinline__ long long lowbit(long long n) { return n & (-n); }
__host__ __device__ __forceinline__ bool is_pow2(long long n) { return n > 0 && (n & (n - 1)) == 0; }

// tanh on the SFU, accurate in relative terms:
//  * |y| >= 1/8: tanh(y) = 1 - 2 / (1 + 2^(K y)) with K = 2 / ln 2 (the definition of
//    tanh through the exponential), evaluated with the SFU's base-2 exponential and
//    reciprocal; absolute error ~2e-7, so relative error < 2e-6; saturates exactly
//    to +-1 for large |y|;
//  * |y| < 1/8: the odd Taylor series tanh(y) = y (1 - y^2/3 + 2 y^4/15 - 17 y^6/315),
//    whose first omitted term (62/2835 y^9) is below 2e-9 relative there.
// Both are computed and one is selected, so the latency is the exponential path's.
constexpr float kTanhK = 2.8853900817779268f;      // 2 / ln 2
constexpr float kTanhSmallZ = 0.36067376022224085f;  // K / 8: |y| < 1/8  <=>  |K y| < K / 8
__device__ __forceinline__ float sfu_ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float sfu_rcp(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
// the SFU's own tanh: one instruction, relative error up to about 2^-11
__device__ __forceinline__ float sfu_tanh(float x) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
// odd series part for small arguments: y * (1 + x (-1/3 + x (2/15 - 17/315 x))), x = y^2
__device__ __forceinline__ float tanh_series(float y) {
    const float x = y * y;
    float q = fmaf(x, -0.053968253968253971f, 0.13333333333333333f);
    q = fmaf(x, q, -0.33333333333333331f);
    q = fmaf(x, q, 1.0f);
    return y * q;
}
__device__ __forceinline__ float act_tanh(float y) {
#ifdef FI_TANH_LIBM
    return tanhf(y);
#else
    const float z = kTanhK * y;
    const float r = sfu_rcp(1.0f + sfu_ex2(z));
    const float big = fmaf(-2.0f, r, 1.0f);
    return fabsf(z) < kTanhSmallZ ? tanh_series(y) : big;
#endif
}

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 conjf2(float2 a) { return make_float2(a.x, -a.y); }

// ----------------------------------------------------------------- per-token step state
// The per-token path replays one captured CUDA graph per block size (section
// "Implementierungsdetails": the launches of one token step are recorded once and
// replayed), so the token a replay works on cannot be a kernel argument: it lives in
// this device-side record, written by k_set_step at the start of a call and advanced
// by the last CTA to finish the token's last launch (tok_advance_if_last).
struct TokIO {
    const float* x;  // teacher: tokens [.][G] from token tx on; closed loop: [G] token tx, or null
    float* y;        // y^M [.][G] from token tx on
    long long tx;    // token of x[0] / y[0]
    long long t;     // token being processed
    int closed;
    unsigned done;   // CTAs of the current launch that have finished (advancing launch only)
    int* itok;       // language model: greedy choices [.][B] from token tx on
};

__global__ void k_set_step(TokIO* io, TokIO v) { *io = v; }

// Called by every thread of every CTA at the very end of the launch that closes a
// token: each CTA has read io->t at its start; the last CTA to get here (every other
// one has counted itself, so every read is done) moves the record to the next token.
__device__ __forceinline__ void tok_advance_if_last(TokIO* io) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y * gridDim.z;
        if (atomicAdd(&io->done, 1u) == total - 1) {
            io->done = 0;
            io->t += 1;
            __threadfence();
        }
    }
}

// ----------------------------------------------------------------- tile addressing
// A "tile" is one gray block for one (layer, chain), or one stand-alone tau item.
struct TileArgs {
    // stack addressing: layer l1's block reads act[l1][g] and adds onto act_out[l1][g]
    // (for the tanh stack act_out = act + G L: layer l's output buffer is layer l+1's input)
    float* act;
    float* act_out;
    const float* h;
    long long L;
    long long G;
    int D;
    long long n;  // block released after the n-th token
    // flat addressing (stand-alone tau): in + i*U, out + i*U, taps + i*ldt
    const float* fin;
    float* fout;
    const float* ftaps;
    long long ldt;
    int flat;
    // common
    int U;
    int count;       // number of tiles
    int overwrite;   // 1: store, 0: accumulate
    const float2* spec;  // spectra of this block size (FFT)
    long long spec_stride;  // complex entries per item
    long long spec_mod;     // flat addressing: item i reads spectrum row i % spec_mod (0: row i)
    const float2* tw;    // e^{-2 pi i k / 2^twlog}, k < 2^twlog
    int twlog;
    TokIO* io;           // non-null: n = io->t + 1 (replayed per-token graph), overwrite = n a power of 2
    int advance;         // with io: this launch closes the token and advances the record
};

// The block position of a launch: from the arguments, or from the step record.
__device__ __forceinline__ TileArgs with_step(TileArgs a) {
    if (a.io) {
        a.n = a.io->t + 1;
        a.overwrite = (a.n & (a.n - 1)) == 0;
    }
    return a;
}

struct TilePtrs {
    const float* in;
    float* out;
    const float* taps;
    const float2* spec;
};

__device__ __forceinline__ TilePtrs tile_ptrs(const TileArgs& a, long long item) {
    TilePtrs p;
    if (a.flat) {
        p.in = a.fin + item * a.U;
        p.out = a.fout + item * a.U;
        p.taps = a.ftaps + item * a.ldt;
        p.spec = a.spec ? a.spec + (a.spec_mod ? item % a.spec_mod : item) * a.spec_stride : nullptr;
    } else {
        long long l1 = item / a.G;  // layer - 1
        long long g = item - l1 * a.G;
        long long c = g % a.D;
        p.in = a.act + (l1 * a.G + g) * a.L + (a.n - a.U);
        p.out = a.act_out + (l1 * a.G + g) * a.L + a.n;
        p.taps = a.h + (l1 * a.D + c) * a.L;
        p.spec = a.spec ? a.spec + (l1 * a.D + c) * a.spec_stride : nullptr;
    }
    return p;
}

// ----------------------------------------------------------------- direct tau
// out[r] (+)= sum_{j<U} in[j] * taps[U + r - j], one tile per CTA, operands staged
// in shared memory (block U floats, taps 2U floats).
template <int NT, int RG>
__global__ void __launch_bounds__(NT) k_tile_direct(TileArgs a0) {
    const TileArgs a = with_step(a0);
    extern __shared__ float sm[];
    const int U = a.U;
    float* sin = sm;
    float* stap = sm + U;
    TilePtrs p = tile_ptrs(a, blockIdx.x);
    for (int j = threadIdx.x; j < U; j += NT) sin[j] = p.in[j];
    for (int k = threadIdx.x; k < 2 * U; k += NT) stap[k] = p.taps[k];
    __syncthreads();
    // each thread owns RG consecutive rows of a strided group
    const int ngrp = (U + RG - 1) / RG;
    for (int grp = threadIdx.x; grp < ngrp; grp += NT) {
        const int r0 = grp * RG;
        float acc[RG];
#pragma unroll
        for (int q = 0; q < RG; ++q) acc[q] = 0.f;
        for (int j = 0; j < U; ++j) {
            const float x = sin[j];
#pragma unroll
            for (int q = 0; q < RG; ++q) {
                int lag = U + r0 + q - j;
                if (r0 + q < U) acc[q] = fmaf(x, stap[lag], acc[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < RG; ++q) {
            int r = r0 + q;
            if (r < U) p.out[r] = a.overwrite ? acc[q] : p.out[r] + acc[q];
        }
    }
    if (a.io && a.advance) tok_advance_if_last(a.io);
}

// The same sum for a small block (U <= 8): one thread per tile, operands in registers.
// A tile then costs a few 32-byte sectors (U inputs, 2U taps, U outputs each within one
// aligned run), where one CTA per tile would be almost all launch and barrier.
template <int U>
__global__ void __launch_bounds__(128) k_tile_direct_small(TileArgs a0) {
    const TileArgs a = with_step(a0);
    const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (item < a.count) {
        const TilePtrs p = tile_ptrs(a, item);
        float x[U], h[2 * U];
#pragma unroll
        for (int j = 0; j < U; ++j) x[j] = p.in[j];
#pragma unroll
        for (int k = 1; k < 2 * U; ++k) h[k] = __ldg(p.taps + k);
#pragma unroll
        for (int r = 0; r < U; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < U; ++j) acc = fmaf(x[j], h[U + r - j], acc);
            p.out[r] = a.overwrite ? acc : p.out[r] + acc;
        }
    }
    if (a.io && a.advance) tok_advance_if_last(a.io);
}

// ----------------------------------------------------------------- shared-memory FFT
// In-place Stockham autosort FFT (forward, e^{-2 pi i k m / N}) of N = 2^LOGN
// complex values in shared memory, radix-4 passes plus one radix-2 pass when LOGN
// is odd.  Pass with sub-transform size Ns: butterfly j reads X[j + r N/R], applies
// twiddle W_{Ns R}^{r (j mod Ns)}, does an R-point DFT and writes output m to
// X[(j - j mod Ns) R + j mod Ns + m Ns].  All reads of a pass complete before any
// write (barrier), so one buffer suffices.
template <int R>
__device__ __forceinline__ void dft_small(float2* v) {
    if (R == 2) {
        float2 a = v[0], b = v[1];
        v[0] = cadd(a, b);
        v[1] = csub(a, b);
    } else {  // R == 4, W_4 = -i
        float2 s02 = cadd(v[0], v[2]), d02 = csub(v[0], v[2]);
        float2 s13 = cadd(v[1], v[3]), d13 = csub(v[1], v[3]);
        v[0] = cadd(s02, s13);
        v[2] = csub(s02, s13);
        // -i * d13 = (d13.y, -d13.x)
        v[1] = make_float2(d02.x + d13.y, d02.y - d13.x);
        v[3] = make_float2(d02.x - d13.y, d02.y + d13.x);
    }
}

template <int LOGN, int NT, int R, int LOGR>
__device__ __forceinline__ void stockham_pass(float2* X, int logNs, const float2* __restrict__ tw,
                                              int twlog) {
    constexpr int N = 1 << LOGN;
    constexpr int NB = N / R;
    constexpr int J = (NB + NT - 1) / NT;
    const int Ns = 1 << logNs;
    float2 v[J][R];
#pragma unroll
    for (int jj = 0; jj < J; ++jj) {
        const int j = threadIdx.x + jj * NT;
        if (j < NB) {
            const int k = j & (Ns - 1);
#pragma unroll
            for (int r = 0; r < R; ++r) v[jj][r] = X[j + r * NB];
            if (Ns > 1) {
                const int sh = twlog - logNs - LOGR;
#pragma unroll
                for (int r = 1; r < R; ++r) v[jj][r] = cmul(v[jj][r], __ldg(&tw[(r * k) << sh]));
            }
            dft_small<R>(v[jj]);
        }
    }
    __syncthreads();
#pragma unroll
    for (int jj = 0; jj < J; ++jj) {
        const int j = threadIdx.x + jj * NT;
        if (j < NB) {
            const int k = j & (Ns - 1);
            const int base = (j - k) * R + k;
#pragma unroll
            for (int m = 0; m < R; ++m) X[base + m * Ns] = v[jj][m];
        }
    }
    __syncthreads();
}

template <int LOGN, int NT>
__device__ __forceinline__ void fft_smem(float2* X, const float2* __restrict__ tw, int twlog) {
    int logNs = 0;
#pragma unroll
    for (int p = 0; p < LOGN / 2; ++p) {
        stockham_pass<LOGN, NT, 4, 2>(X, logNs, tw, twlog);
        logNs += 2;
    }
    if (LOGN & 1) stockham_pass<LOGN, NT, 2, 1>(X, logNs, tw, twlog);
}

// Real-signal helpers.  A real sequence x of length 2N is packed as z[m] = x[2m] +
// i x[2m+1] (m < N).  With Z = DFT_N(z), E[k] = (Z[k] + conj Z[N-k]) / 2 and
// O[k] = (Z[k] - conj Z[N-k]) / (2i) are the DFTs of the even and odd samples, and
// X[k] = E[k] + W^k O[k], X[k+N] = E[k] - W^k O[k] with W = e^{-2 pi i / 2N}.
// unpack_pair returns X[k] and X[N-k] (X[N] when k = 0).
__device__ __forceinline__ void unpack_pair(float2 Zk, float2 Zn, float2 Wk, float2 Wnk, bool k0,
                                            float2& Xk, float2& Xn) {
    float2 E = make_float2(0.5f * (Zk.x + Zn.x), 0.5f * (Zk.y - Zn.y));
    float2 Dd = make_float2(Zk.x - Zn.x, Zk.y + Zn.y);  // Z[k] - conj Z[N-k]
    float2 O = make_float2(0.5f * Dd.y, -0.5f * Dd.x);   // D / (2i)
    Xk = cadd(E, cmul(Wk, O));
    if (k0) Xn = make_float2(E.x - O.x, E.y - O.y);      // X[N] = E[0] - O[0]
    else Xn = cadd(conjf2(E), cmul(Wnk, conjf2(O)));    // E[N-k] = conj E[k], same for O
}
// Twiddle e^{-2 pi i k / 2N} from the table e^{-2 pi i m / 2^twlog}.
template <int LOGN>
__device__ __forceinline__ float2 tw2n(const float2* __restrict__ tw, int twlog, int k) {
    return __ldg(&tw[k << (twlog - LOGN - 1)]);
}

// ----------------------------------------------------------------- fused FFT tau
// Blocks of one edge U = N for every layer and chain (or stand-alone tau items), one
// tile per group of T = N / E threads, register-resident radix-16 FFTs (fi_fft.cuh).
// Forward passes: one radix-R0 pass when log2 N is not a multiple of 4 (twiddle-free,
// first), then radix-16 passes.  Inverse passes: radix-16 first (the first one
// continues in registers from the forward's last), the radix-R0 pass last, so that
// the last pass of each direction is the one that touches global memory only for the
// half it needs (the zero half of the input is never read, the wrap-around half of
// the output is never formed).
template <int LOGN>
struct FftTile {
    static constexpr int N = 1 << LOGN;
    static constexpr int RB = N >= 16 ? 16 : N;           // main radix
    static constexpr int LOGRB = RB == 16 ? 4 : LOGN;
    static constexpr int NP = LOGN / LOGRB;                // main-radix passes per FFT
    static constexpr int LOGR0 = LOGN - NP * LOGRB;
    static constexpr int R0 = 1 << LOGR0;                  // extra radix (1: none)
    static constexpr int E = RB;                           // points per thread
    static constexpr int T = N / E;                        // threads per tile
    static constexpr int NT = T >= 256 ? T : 256;          // threads per CTA
    static constexpr int TPC = NT / T;                     // tiles per CTA
    static constexpr int SME = N + N / 16;                 // padded entries per tile
    static constexpr bool STAGE_H = N <= 8192;             // spectrum staged in shared memory
    static constexpr int HST = STAGE_H ? N + 2 : 0;        // staged spectrum entries per tile
    static constexpr int OST = N / 2;                      // staged old outputs (float2) per tile
    static constexpr size_t smem = (size_t)TPC * (SME + HST + OST) * sizeof(float2);
    static constexpr int MINB = NT <= 256 ? 2 : 1;         // CTAs per SM the registers allow
};

// Asynchronous 16-byte global -> shared copy (cp.async, L2 only), completed by
// cp_async_wait_all() of the same thread; a barrier then publishes it to the CTA.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while its predecessor in the stream is finishing; it
// reads nothing the predecessor writes before grid_dep_wait(), which returns once
// the predecessor has completed and its writes are visible (at once when launched
// normally).  grid_dep_launch() lets the successor start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Radix-R Stockham pass whose inputs come from shared memory and whose outputs
// m >= R/2 (the elements i = b + m N/R >= N/2, i.e. real samples [U, 2U)) are added
// onto the tile's outputs: y[2(i - N/2)] = Re F[i], y[2(i - N/2) + 1] = -Im F[i].
template <int LOGN, int R, int BPT, int TWLOG>
__device__ __forceinline__ void fft_last_pass_store(const float2* X, int t, int T, const float2* __restrict__ tw,
                                                    float* out, const float2* old_out, int overwrite, bool valid) {
    constexpr int N = 1 << LOGN, NB = N / R;
    float2* o2 = reinterpret_cast<float2*>(out);
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
        const int b = t + u * T;
        float2 v[R];
#pragma unroll
        for (int r = 0; r < R; ++r) v[r] = X[fft::pad(b + r * NB)];
        if (NB > 1) fft::apply_twiddles<R, TWLOG>(v, tw, LOGN, b);  // Ns = N/R > b: k = b
        fft::dft<R>(v);
        if (valid) {
#pragma unroll
            for (int m = R / 2; m < R; ++m) {
                const float2 F = v[fft::omap<R>(m)];
                const int q = b + m * NB - N / 2;
                const float2 y = make_float2(F.x, -F.y);
                if (overwrite) o2[q] = y;
                else {
                    const float2 old = old_out[q];
                    o2[q] = make_float2(old.x + y.x, old.y + y.y);
                }
            }
        }
    }
}

template <int LOGN, int TWLOG>
__global__ void __launch_bounds__(FftTile<LOGN>::NT, FftTile<LOGN>::MINB) k_block_fft(TileArgs a0) {
    const TileArgs a = with_step(a0);
    using G = FftTile<LOGN>;
    constexpr int N = G::N, RB = G::RB, R0 = G::R0, T = G::T, NP = G::NP, LOGRB = G::LOGRB;
    extern __shared__ __align__(16) float2 fft_sm[];
    const int grp = threadIdx.x / T, t = threadIdx.x - grp * T;
    float2* X = fft_sm + grp * G::SME;
    float2* Hs = fft_sm + G::TPC * G::SME + grp * G::HST;
    float2* Os = fft_sm + G::TPC * (G::SME + G::HST) + grp * G::OST;
    const long long item = (long long)blockIdx.x * G::TPC + grp;
    const bool valid = item < a.count;
    const TilePtrs p = tile_ptrs(a, valid ? item : 0);
    const float2* __restrict__ in2 = reinterpret_cast<const float2*>(p.in);
    float2 v[1][RB];

    // ---- the spectrum and (when accumulating) the old outputs stream into shared
    // memory while the forward transform runs
    if constexpr (G::STAGE_H) {
        if (valid)
            for (int c = t; c < (N + 2) / 2; c += T) cp_async16(Hs + 2 * c, p.spec + 2 * c);
    }
    grid_dep_wait();  // the block's inputs and old outputs come from the previous launches
    if (valid && !a.overwrite) {
        for (int c = t; c < N / 4; c += T) cp_async16(Os + 2 * c, p.out + 4 * c);
    }
    cp_async_commit();

    // ---- forward: first pass from global memory (packed block, zero upper half), Ns = 1
    if constexpr (R0 > 1) {
        constexpr int BPT = RB / R0, NB = N / R0;
        float2 w[BPT][R0];
#pragma unroll
        for (int u = 0; u < BPT; ++u) {
            const int b = t + u * T;
#pragma unroll
            for (int r = 0; r < R0; ++r) w[u][r] = (r < R0 / 2) ? __ldg(in2 + b + r * NB) : make_float2(0.f, 0.f);
            fft::dft<R0>(w[u]);
#pragma unroll
            for (int m = 0; m < R0; ++m) X[fft::pad(b * R0 + m)] = w[u][fft::omap<R0>(m)];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < NP; ++j) fft::pass<LOGN, RB, 1, TWLOG>(X, v, t, T, G::LOGR0 + j * LOGRB, a.tw);
    } else {
        constexpr int NB = N / RB;
#pragma unroll
        for (int r = 0; r < RB; ++r) v[0][r] = (r < RB / 2) ? __ldg(in2 + t + r * NB) : make_float2(0.f, 0.f);
        fft::dft<RB>(v[0]);
#pragma unroll
        for (int m = 0; m < RB; ++m) X[fft::pad(t * RB + m)] = v[0][fft::omap<RB>(m)];
        __syncthreads();
#pragma unroll
        for (int j = 1; j < NP; ++j) fft::pass<LOGN, RB, 1, TWLOG>(X, v, t, T, j * LOGRB, a.tw);
    }

    cp_async_wait_all();
    __syncthreads();

    // ---- spectral multiply: this thread holds Z[k], k = t + m N/RB, in v[0][omap(m)];
    // the partners Z[N-k] are in shared memory (the last pass stored every Z[k]).
    float2 q[RB];
    {
        constexpr int NB = N / RB;
        const float2* H = G::STAGE_H ? Hs : p.spec;
        const float2 wb = fft::tw_at<TWLOG>(a.tw, t << (TWLOG - LOGN - 1));  // W_{2N}^t
#pragma unroll
        for (int m = 0; m < RB; ++m) {
            const int k = t + m * NB;
            const float2 Zk = v[0][fft::omap<RB>(m)];
            const float2 Zn = X[fft::pad((N - k) & (N - 1))];
            const float2 Hk = H[k], Hn = H[N - k];
            const float2 w = fft::cm(wb, fft::w32(m * (16 / RB)));  // W_{2N}^k = (cos, -sin) of pi k / N
            // Q[k] = conj(Z[k]) (S + sin D) + Z[N-k] (i cos D),  S, D = H[N-k] +- conj H[k]
            const float2 S = make_float2(Hn.x + Hk.x, Hn.y - Hk.y);
            const float2 D = make_float2(Hn.x - Hk.x, Hn.y + Hk.y);
            const float sn = -w.y, cs = w.x;
            const float2 G1 = make_float2(fmaf(sn, D.x, S.x), fmaf(sn, D.y, S.y));
            const float2 G2 = make_float2(-cs * D.y, cs * D.x);
            float2 r = make_float2(fmaf(Zk.x, G1.x, Zk.y * G1.y), fmaf(Zk.x, G1.y, -Zk.y * G1.x));
            r.x = fmaf(Zn.x, G2.x, fmaf(-Zn.y, G2.y, r.x));
            r.y = fmaf(Zn.x, G2.y, fmaf(Zn.y, G2.x, r.y));
            q[m] = r;
        }
    }
    __syncthreads();  // partner reads complete before the inverse overwrites X
    grid_dep_launch();

    // ---- inverse: first pass in registers (Ns = 1), then shared-memory passes
    fft::dft<RB>(q);
    if constexpr (NP == 1 && R0 == 1) {
        // a single pass: N = RB, the outputs are q[omap(m)] at i = m
        if (valid) {
            float2* o2 = reinterpret_cast<float2*>(p.out);
#pragma unroll
            for (int m = RB / 2; m < RB; ++m) {
                const float2 F = q[fft::omap<RB>(m)];
                const float2 y = make_float2(F.x, -F.y);
                if (a.overwrite) o2[m - RB / 2] = y;
                else {
                    const float2 old = Os[m - RB / 2];
                    o2[m - RB / 2] = make_float2(old.x + y.x, old.y + y.y);
                }
            }
        }
    } else {
#pragma unroll
        for (int m = 0; m < RB; ++m) X[fft::pad(t * RB + m)] = q[fft::omap<RB>(m)];
        __syncthreads();
        if constexpr (R0 > 1) {
#pragma unroll
            for (int j = 1; j < NP; ++j) fft::pass<LOGN, RB, 1, TWLOG>(X, v, t, T, j * LOGRB, a.tw);
            fft_last_pass_store<LOGN, R0, RB / R0, TWLOG>(X, t, T, a.tw, p.out, Os, a.overwrite, valid);
        } else {
#pragma unroll
            for (int j = 1; j + 1 < NP; ++j) fft::pass<LOGN, RB, 1, TWLOG>(X, v, t, T, j * LOGRB, a.tw);
            fft_last_pass_store<LOGN, RB, 1, TWLOG>(X, t, T, a.tw, p.out, Os, a.overwrite, valid);
        }
    }
    if (a.io && a.advance) tok_advance_if_last(a.io);
}

// ----------------------------------------------------------------- filter spectra
// H[k] = scale * sum_{m<2N} taps[off + m] e^{-2 pi i k m / 2N}, k = 0..N, for every
// (layer, channel) item and every offset e (off = e * offstep).  Run once when a
// context is created (section "Speicheroptimierung": DFT of the filters per block size).
template <int LOGN, int NT>
__global__ void __launch_bounds__(NT) k_spectra(const float* __restrict__ taps, long long ld,
                                                int nspec, long long offstep, float2* spec,
                                                const float2* __restrict__ tw, int twlog, float scale,
                                                long long hstride) {
    extern __shared__ float2 X[];
    constexpr int N = 1 << LOGN;
    const long long item = blockIdx.x / nspec;
    const int e = blockIdx.x % nspec;
    const float2* t2 = reinterpret_cast<const float2*>(taps + item * ld + e * offstep);
    for (int m = threadIdx.x; m < N; m += NT) X[m] = t2[m];
    __syncthreads();
    fft_smem<LOGN, NT>(X, tw, twlog);
    float2* H = spec + ((long long)blockIdx.x) * hstride;
    for (int k = threadIdx.x; k <= N / 2; k += NT) {
        const int kn = (N - k) & (N - 1);
        float2 Xk, Xn;
        unpack_pair(X[k], X[kn], tw2n<LOGN>(tw, twlog, k), tw2n<LOGN>(tw, twlog, N - k), k == 0,
                    Xk, Xn);
        H[k] = make_float2(Xk.x * scale, Xk.y * scale);
        H[N - k] = make_float2(Xn.x * scale, Xn.y * scale);
    }
}

// ----------------------------------------------------------------- per-token step
// The pages' per-token order (Algorithm 2 with Algorithm 3's layer parallelism):
// red cells of token t for every layer in order (block and sampler = tanh), then,
// when the released block is small, the gray block of every layer in the same
// launch.  One lane per chain; 32 chains per CTA.
struct StepArgs {
    float* act;
    const float* h;
    int M, D;
    long long L, G;
    long long t;
    const float* x;  // [G] token t, or null: take act[0][g][t]
    float* y;        // [G] y^M_t
    int closed;      // write a^M_t as token t+1
    int fuseU;       // edge of the block n = t+1 done here (0: none)
    TokIO* io;       // non-null: t, x and y come from the step record (replayed graph)
    int advance;     // with io: this launch closes the token and advances the record
};

template <int NT>
__global__ void __launch_bounds__(NT) k_token_step(StepArgs a) {
    const long long g0 = (long long)blockIdx.x * 32;
    const int lane = threadIdx.x;
    long long t = a.t;
    const float* xt = a.x;
    float* yt = a.y;
    if (a.io) {
        const TokIO io = *a.io;
        t = io.t;
        yt = io.y + (t - io.tx) * a.G;
        xt = io.closed ? (t == io.tx ? io.x : nullptr) : io.x + (t - io.tx) * a.G;
    }
    if (lane < 32) {
        const long long g = g0 + lane;
        if (g < a.G) {
            const long long c = g % a.D;
            float av = xt ? xt[g] : a.act[g * a.L + t];
            a.act[g * a.L + t] = av;
            float y = 0.f;
            // the running sums and taps h_0 of the layers do not depend on the chain:
            // eight layers' worth is loaded before their links run, so the chain waits for
            // global memory once per eight layers, not once per layer
            constexpr int KB = 8;
            for (int l0 = 1; l0 <= a.M; l0 += KB) {
                float pv[KB], hv[KB];
#pragma unroll
                for (int k = 0; k < KB; ++k) {
                    const int l = l0 + k;
                    const bool ok = l <= a.M;
                    pv[k] = (ok && t > 0) ? a.act[((long long)l * a.G + g) * a.L + t] : 0.f;
                    hv[k] = ok ? a.h[((long long)(l - 1) * a.D + c) * a.L] : 0.f;
                }
#pragma unroll
                for (int k = 0; k < KB; ++k) {
                    const int l = l0 + k;
                    if (l <= a.M) {
                        y = fmaf(hv[k], av, pv[k]);
                        av = act_tanh(y);
                        a.act[((long long)l * a.G + g) * a.L + t] = av;
                    }
                }
            }
            yt[g] = y;
            if (a.closed && t + 1 < a.L) a.act[g * a.L + t + 1] = av;
        }
    }
    const int U = a.fuseU;
    if (U != 0) {
        __syncthreads();
        const long long n = t + 1;
        const bool ow = is_pow2(n);
        const int nch = (int)min(32LL, a.G - g0);
        const int items = nch * a.M * U;
        for (int it = threadIdx.x; it < items; it += NT) {
            const int r = it % U;
            const int rest = it / U;
            const int i = rest % nch;
            const int l = rest / nch + 1;
            const long long g = g0 + i;
            const long long c = g % a.D;
            const float* in = a.act + ((long long)(l - 1) * a.G + g) * a.L + (n - U);
            const float* hp = a.h + ((long long)(l - 1) * a.D + c) * a.L + U + r;
            float acc = 0.f;
            for (int j = 0; j < U; ++j) acc = fmaf(in[j], hp[-j], acc);
            float* o = a.act + ((long long)l * a.G + g) * a.L + n + r;
            *o = ow ? acc : *o + acc;
        }
    }
    if (a.io && a.advance) tok_advance_if_last(a.io);
}

// ----------------------------------------------------------------- window kernel
// Persistent per-window kernel (the B200 form of the per-token CUDA graph): one
// CTA holds `kch` channels x B batch rows ("chains") and runs tokens [t0, t1) of one
// aligned window [kW, kW+W) entirely in shared memory.  Every block of edge U < W
// released inside the window reads and writes only positions of that window (n =
// kW + m with 0 < m < W, U = lowbit(m): [n-U, n+U-1] lies in the window), so the
// window is self-contained; blocks of edge >= W are released only at window ends
// and run as separate launches over all chains.
//
// Inside the window every block row is evaluated one token before it is needed:
//  * chain lanes (warp 0, one lane per chain) run the red cells of all layers in
//    order, plus the single term of row 0 of block n = t that needs a^{l-1}_{t-1};
//  * helper warps, concurrently, finish position T = t+1: they add the rows of the
//    blocks n in (t0, T] that cover T, except that newest term.  Walking n = T,
//    T - lowbit(T), ... (each step clears the lowest set bit) lists exactly those
//    blocks; their input ranges are adjacent, so the rows form one dot product over
//    inputs [lo, t-1] per (layer, chain).
// A block is therefore never computed as a burst on the chain's critical path, and
// each step costs one barrier.  Blocks released at or before t0 were completed by
// the previous launch (or by the large-block launch at a window start); a launch
// that stops inside the window completes the blocks it released before storing, so
// the buffers always hold the state the per-token path expects: every block
// n <= t applied.
struct WinArgs {
    float* act;
    const float* h;
    int M, B, D;
    long long L, G;
    long long t0, t1;   // tokens of this launch (one window)
    long long tx;       // token of x[0] / out[0]
    const float* x;     // teacher: [.][G] tokens; closed loop: [G] token t0 or null
    float* out;         // [.][G] y^M
    int closed;
    int kch;            // channels per CTA
};

// Warp 0: spec lanes; warp 1: exact lanes; warps 2..8: helper pairs.  (Warp w runs on
// scheduler w % 4: the spec warp shares its scheduler with helper warps 4 and 8, the
// exact warp with helper warp 5; layouts giving the spec or exact warp a scheduler of
// its own measured slower.)
constexpr int kWinThreads = 288;
constexpr int kWinExactWarp = 1;
constexpr int kWinPairs = 7 * 16;
__device__ __forceinline__ bool win_helper(int warp) { return warp >= 2; }
__device__ __forceinline__ int win_helper_index(int warp) { return warp - 2; }
// Every shared-memory row of the window kernel (positions, taps, shifted copies) is
// followed by kWinPad zero floats, and a zero row precedes the first: a row whose
// blocks start at window position 0 may then read up to 31 positions below 0 and
// get zeros, so its lag pairs need no per-term masking.  W + kWinPad = 4 mod 32
// keeps the helpers' 8-byte loads free of bank conflicts.
constexpr int kWinPad = 36;

// Lowest input of the blocks released at n in (s0, hi] that cover window position T
// (window-local), walking n = T, T - lowbit(T), ...; returns -1 if none.  *top gets
// the highest such input (the first covering block released at or before hi).
__device__ __forceinline__ int cover_range(int T, int s0, int hi, int* top) {
    int lo = -1, n = T;
    *top = -1;
    while (n > s0 && n > 0) {
        const int lon = n - (n & (-n));
        if (n <= hi) {
            if (*top < 0) *top = n - 1;
            lo = lon;
        }
        n = lon;
    }
    return lo;
}

// One lane of a helper pair: sum over j = lo + part + 2k (k < n2) of in[j] * tp[T - j],
// where n2 = ceil((hi - lo + 1) / 2) is the same for both lanes, so the two lanes run
// identical trip counts (no divergence).  Full batches of 16 terms per lane, which lie
// in range for both lanes, issue their 32 shared-memory loads (immediate offsets from
// two running pointers) before the multiply-adds; one predicated batch takes the
// remaining 1..16 terms, where a term past hi (the odd lane's last one when the length
// is odd) loads a valid element and is multiplied by 0.
__device__ __forceinline__ float dot_pair(const float* in, const float* tp, int T, int lo, int hi, int part) {
    const int n2 = (hi - lo + 2) >> 1;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    const float* pi = in + lo + part;
    const float* pt = tp + T - lo - part;
    int k = 0;
    for (; k + 16 < n2; k += 16) {
        float x[16], y[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            x[u] = pi[2 * u];
            y[u] = pt[-2 * u];
        }
#pragma unroll
        for (int u = 0; u < 16; u += 4) {
            a0 = fmaf(x[u], y[u], a0);
            a1 = fmaf(x[u + 1], y[u + 1], a1);
            a2 = fmaf(x[u + 2], y[u + 2], a2);
            a3 = fmaf(x[u + 3], y[u + 3], a3);
        }
        pi += 32;
        pt -= 32;
    }
    if (k < n2) {
        // terms k .. n2-1 (1..16 of them); the last is past hi for the odd lane of an
        // odd-length row
        const int rem = n2 - k;
        const int last_ok = (lo + part + 2 * (n2 - 1) <= hi) ? rem : rem - 1;
        float x[16], y[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const bool ok = u < last_ok;
            const int o = ok ? 2 * u : 0;
            x[u] = pi[o];
            y[u] = pt[-o];
            x[u] = ok ? x[u] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 16; u += 4) {
            a0 = fmaf(x[u], y[u], a0);
            a1 = fmaf(x[u + 1], y[u + 1], a1);
            a2 = fmaf(x[u + 2], y[u + 2], a2);
            a3 = fmaf(x[u + 3], y[u + 3], a3);
        }
    }
    return (a0 + a1) + (a2 + a3);
}

// Two fp32 multiply-adds in one packed instruction (sm_100): c + a * b per lane.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n.reg .b64 pa, pb, pc;\nmov.b64 pa, {%2, %3};\nmov.b64 pb, {%4, %5};\nmov.b64 pc, {%6, %7};\n"
        "fma.rn.f32x2 pc, pa, pb, pc;\nmov.b64 {%0, %1}, pc;\n}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

// The main-loop row of a helper lane's own item, two lags per load and per
// multiply-add: the lags 2..dmax of row T are taken in pairs (2 + 2k, 3 + 2k); lane
// `part` takes k = part + 2m, m < nm_me, with trx[m] = (tap[3 + 2k], tap[2 + 2k]) in
// registers.  The inputs of pair k, positions (T - 3 - 2k, T - 2 - 2k), are one
// aligned 8-byte load: from the input row when T is odd, else from its copy shifted
// by one position (pbl points at pair m = 0 of this lane; pair m sits at pbl - 4m).
// nm_both pairs are whole for both lanes; when dmax is even the last pair's upper
// lag is past dmax and `last_half` (set on the lane that owns it) drops it.
template <int NTR2, int N>
__device__ __forceinline__ float dot_lags2(const float* pbl, const float2 (&trx)[N], int nm_both, int nm_me,
                                           bool last_half) {
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int b = 0; b < NTR2; b += 8) {
        if (b >= nm_me) break;
        float2 x[8];
        if (b + 8 <= nm_both) {
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = *reinterpret_cast<const float2*>(pbl - 4 * (b + u));
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool ok = b + u < nm_me;
                const float2 v = *reinterpret_cast<const float2*>(pbl - (ok ? 4 * (b + u) : 0));
                x[u] = ok ? v : make_float2(0.f, 0.f);
                if (last_half && b + u == nm_me - 1) x[u].x = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
            a0 = ffma2(x[u], trx[b + u], a0);
            a1 = ffma2(x[u + 1], trx[b + u + 1], a1);
        }
    }
    return (a0.x + a0.y) + (a1.x + a1.y);
}

// dot_lags2 for a row whose inputs start at window position 0: every lane runs nblk
// whole blocks of 8 lag pairs; the pairs past the row's last lag (and the upper lag
// of a partial last pair) read the zero padding below position 0, or meet zero taps
// past the window, and add exact zeros.
template <int NTR2, int N>
__device__ __forceinline__ float dot_lags2_padded(const float* pbl, const float2 (&trx)[N], int nblk) {
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int b = 0; b < NTR2; b += 8) {
        if (b >= 8 * nblk) break;
        float2 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = *reinterpret_cast<const float2*>(pbl - 4 * (b + u));
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
            a0 = ffma2(x[u], trx[b + u], a0);
            a1 = ffma2(x[u + 1], trx[b + u + 1], a1);
        }
    }
    return (a0.x + a0.y) + (a1.x + a1.y);
}

// One helper pair's first (layer, chain) item: shared-memory offsets of its input
// row, tap row and output row (out < 0: none).  Shapes with more items than pairs
// hand the pair further items pair + k * kWinPairs, decoded on the fly.
struct PairItem {
    int in, tp, out;
};

struct ItemGeom {
    int nitems, ncb, nch, CPB, kch, P, tap0;
};

__device__ __forceinline__ PairItem decode_item(const ItemGeom& g, int it) {
    PairItem r;
    if (it < g.nitems) {
        const int l = it / g.ncb + 1, i = it - (l - 1) * g.ncb;
        r.in = ((l - 1) * g.CPB + i) * g.P;
        r.tp = g.tap0 + ((l - 1) * g.kch + (i % g.nch)) * g.P;
        r.out = (l * g.CPB + i) * g.P;
    } else {
        r.in = r.tp = 0;
        r.out = -1;
    }
    return r;
}

__device__ __forceinline__ void add_row(float* sm, const PairItem& it, int T, int lo, int hi, bool ow, int part) {
    const bool mine = it.out >= 0;
    float acc = mine ? dot_pair(sm + it.in, sm + it.tp, T, lo, hi, part) : 0.f;
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (part == 0 && mine) {
        float* o = sm + it.out + T;
        *o = ow ? acc : *o + acc;
    }
}

// Helper pairs add the rows over inputs [lo, hi] onto position T of every
// (layer, chain); overwrite when these rows include the position's first writer.
// All lanes of a (fully active) helper warp make the same shuffles: the extra-item
// loop runs to the warp's largest count and lanes past their own count add 0.
__device__ __noinline__ void helper_rows_more(float* sm, const ItemGeom& g, int pair, int T, int lo, int hi,
                                              bool ow, int part) {
    const int mine_n = pair < g.nitems ? (g.nitems - pair + kWinPairs - 1) / kWinPairs : 0;
    const int nwarp = (int)__reduce_max_sync(0xffffffffu, (unsigned)mine_n);
    for (int k = 1; k < nwarp; ++k) add_row(sm, decode_item(g, pair + k * kWinPairs), T, lo, hi, ow, part);
}

__device__ __forceinline__ void helper_rows(float* sm, const ItemGeom& g, const PairItem& first, bool more,
                                            int pair, int T, int lo, int hi, bool ow, int part) {
    add_row(sm, first, T, lo, hi, ow, part);
    if (more) helper_rows_more(sm, g, pair, T, lo, hi, ow, part);
}

// One register array serves two roles that never share a thread: the helper lanes keep
// their tap pairs in it, the chain lanes their per-layer values.  Index i is a
// compile-time constant wherever these are called (unrolled loops).
template <int N>
__device__ __forceinline__ float rget(const float2 (&r)[N], int i) { return (i & 1) ? r[i >> 1].y : r[i >> 1].x; }
template <int N>
__device__ __forceinline__ void rset(float2 (&r)[N], int i, float v) {
    if (i & 1) r[i >> 1].y = v;
    else r[i >> 1].x = v;
}

// CPBT != 0: the launch has B = 1 and kch = CPBT chains per CTA, known at compile
// time, so every shared-memory row the chain lanes touch sits at an immediate offset.
template <int W, int MAXM, bool EXACT, int CPBT>
__global__ void __launch_bounds__(kWinThreads, 1) k_window(WinArgs a) {
    extern __shared__ float4 sm4[];
    constexpr int NT = kWinThreads;
    // row pitch = 4 mod 32: the 8-byte loads of the 16 lanes of half a helper warp
    // (pair i, lane p at word P i - 2p + c) hit 16 distinct bank pairs; 16-byte rows
    constexpr int P = W + kWinPad;
    float* sm = reinterpret_cast<float*>(sm4) + P;  // after the leading zero row
    const int M = EXACT ? MAXM : a.M;
    const int B = CPBT ? 1 : a.B, D = a.D, kch = CPBT ? CPBT : a.kch;
    const long long L = a.L, G = a.G;
    const int c0 = blockIdx.x * kch;
    const int nch = min(kch, D - c0);
    const int ncb = nch * B;
    const int CPB = kch * B;
    const int tap0 = (M + 1) * CPB * P;
    const int dup0 = tap0 + M * kch * P;  // copies of the input rows (layers 0..M-1), shifted by one
    float* slot = sm;               // [(M+1) * CPB][P]
    float* tap = sm + tap0;         // [M * kch][P]
    float* dup = sm + dup0;         // [M * CPB][P], dup[x + 1] = activation at window position x
    const long long kW = (a.t0 / W) * (long long)W;  // windows never cross L (W divides L)
    const int s0 = (int)(a.t0 - kW), s1 = (int)(a.t1 - kW);
    const int tid = threadIdx.x;

    // ---- stage the window of every layer and taps 0..W-1: every 16-byte copy in
    // flight at once (cp.async; rows of W floats at pitch P, 16-byte aligned).
    // Thread -> (column quad, first row); rows advance by a fixed stride.  The taps
    // (fixed for the whole generation) go first; the positions, written by the
    // previous launches, after grid_dep_wait().
    {
        constexpr int PER4 = W / 4;
        constexpr int RSTR = NT / PER4;
        const int rows_slot = (M + 1) * ncb;
        const int c4 = tid % PER4;
        for (int r2 = tid / PER4; r2 < M * nch; r2 += RSTR) {
            const int l = r2 / nch, ci = r2 - l * nch;
            cp_async16(sm + tap0 + (l * kch + ci) * P + 4 * c4, a.h + ((long long)l * D + c0 + ci) * L + 4 * c4);
        }
        grid_dep_wait();
        for (int row = tid / PER4; row < rows_slot; row += RSTR) {
            const int l = row / ncb, i = row - l * ncb;
            const long long g = (long long)(i / nch) * D + c0 + (i % nch);
            cp_async16(sm + (l * CPB + i) * P + 4 * c4, a.act + ((long long)l * G + g) * L + kW + 4 * c4);
        }
        // the zero row before the first row and the padding after every row (16-byte
        // stores: rows start on 16-byte boundaries, W and kWinPad are multiples of 4)
        static_assert(W % 4 == 0 && kWinPad % 4 == 0, "16-byte padding stores");
        for (int e = tid; e < P; e += NT) sm[e - P] = 0.f;
        const int nrows = dup0 / P + M * CPB;
        for (int r = tid; r < nrows; r += NT) {
            float4* pr = reinterpret_cast<float4*>(sm + r * P + W);
#pragma unroll
            for (int k = 0; k < kWinPad / 4; ++k) pr[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        if (!a.closed) {
            const int steps = s1 - s0;
            for (int e = tid; e < steps * ncb; e += NT) {
                const int i = e % ncb;
                const int s = s0 + e / ncb;
                const long long g = (long long)(i / nch) * D + c0 + (i % nch);
                slot[i * P + s] = a.x[(kW + s - a.tx) * G + g];
            }
        } else if (a.x) {
            for (int i = tid; i < ncb; i += NT) {
                const long long g = (long long)(i / nch) * D + c0 + (i % nch);
                slot[i * P + s0] = a.x[g];
            }
        }
        __syncthreads();
        // shifted copies of the input rows (only positions already final are ever
        // read); entry 0 stands for position -1 and is zero.  Every row l * CPB + i of
        // layers 0..M-1 is copied, the unused ones (i >= ncb) too: thread -> column
        // x = tid % W, rows advance by NT / W
        {
            constexpr int RS = NT / W;
            const int x = tid & (W - 1);
            if (tid < RS * W)
                for (int r = tid / W; r < M * CPB; r += RS)
                    dup[r * P + x] = x == 0 ? 0.f : slot[r * P + x - 1];
        }
        __syncthreads();
    }

    // ---- per-launch setup.  Warp 0 runs the layer chain of each token speculatively
    // (spec lanes), warp 1 follows one token behind with the exact activations (exact
    // lanes), warps 2..8 are helper pairs.  Lane c < ncb of warps 0 and 1 owns chain c.
    const int warp = tid >> 5, lane = tid & 31;
    const bool chain = (warp == 0 || warp == kWinExactWarp) && lane < ncb;
    long long gch = 0;
    int cich = 0;
    float h0r[MAXM], h1r[MAXM];
    // Shared register array R: helper lanes hold their tap pairs in R[m]; chain lanes
    // use it as floats (rget / rset): h2 of layer l at [l - 1], the activations
    // a^0..a^{M-1} the spec chain used for the previous token at [MAXM + l - 1], and the
    // exact lanes' e_0..e_{M-1} of the previous token (exact - speculative) at
    // [2 MAXM + l - 1].
    constexpr int NTR2 = ((W - 2) / 4 + 7) / 8 * 8;
    constexpr int NR2 = NTR2 > (3 * MAXM + 1) / 2 ? NTR2 : (3 * MAXM + 1) / 2;
    float2 R[NR2];
#pragma unroll
    for (int m = 0; m < NR2; ++m) R[m] = make_float2(0.f, 0.f);
    float aMsp = 0.f;      // spec: its last layer's activation (the closed loop's next input)
    float eM = 0.f;        // exact: e_M of the previous token
    if (chain) {
        cich = lane % nch;
        gch = (long long)(lane / nch) * D + c0 + cich;
#pragma unroll
        for (int l = 1; l <= MAXM; ++l) {
            const int lc = l <= M ? l : M;
            const float* tl = tap + ((lc - 1) * kch + cich) * P;
            h0r[l - 1] = tl[0];
            h1r[l - 1] = tl[1];
            rset(R, l - 1, tl[2]);
        }
    }
    // speculative (pre-activation, activation) of every layer, by token parity:
    // xch[((s & 1) * M + l - 1) * CPB + lane] (dense over (layer, chain): the exact
    // warp's lanes walk it by q = (l - 1) * CPB + c without bank conflicts)
    float2* xch = reinterpret_cast<float2*>(dup + M * CPB * P);
    const bool helper = win_helper(warp);
    const int pair = win_helper_index(warp) * 16 + (lane >> 1), part = tid & 1;
    ItemGeom geom;
    geom.nitems = M * ncb;
    geom.ncb = ncb;
    geom.nch = nch;
    geom.CPB = CPB;
    geom.kch = kch;
    geom.P = P;
    geom.tap0 = tap0;
    const PairItem first = decode_item(geom, helper ? pair : geom.nitems);
    const bool more = geom.nitems > kWinPairs;  // uniform over the CTA
    // the helper lane's own item keeps its taps in registers, as lag pairs
    // k = part + 2m: R[m] = (tap[4 + 2k], tap[3 + 2k])
    if (helper) {
        const bool ok = first.out >= 0;
#pragma unroll
        for (int m = 0; m < NTR2; ++m) {
            const int d = 3 + 2 * (part + 2 * m);
            R[m] = make_float2((ok && d + 1 < W) ? sm[first.tp + d + 1] : 0.f, (ok && d < W) ? sm[first.tp + d] : 0.f);
        }
    }

    // ---- tokens.  Iteration s runs the speculative chain of token s (warp 0), the exact
    // activations of token s - 1 (warp 1) and the helper rows of position s + 1 over
    // inputs up to s - 2 (lags >= 3); iteration s1 only finishes token s1 - 1.
    //
    // Spec lanes: y_l = p_l + h2 a^{l-1}_{s-2} + h1 a^{l-1}_{s-1} + h0 a^{l-1}_s with the
    // running sum p_l (lags >= 3, from the helpers) and the exact a_{s-2} (written by the
    // exact lanes one iteration earlier); the two newest inputs are the chain's own
    // speculative activations, so the chain is one FMA and one SFU tanh per link:
    //   yh_l = p_l + h2 a^{l-1}_{s-2} + h1 ah^{l-1}_{s-1} + h0 ah^{l-1}_s,  ah^l_s = tanh_sfu(yh_l).
    // Exact lanes, one token later: with e^l = a^l - ah^l, the exact pre-activation is
    // y_l = yh_l + u, u = h0 e^{l-1}_s + h1 e^{l-1}_{s-1}; with t = tanh(yh_l) in the
    // exact form and q = 1 - t^2,
    //   e^l_s = (t - ah^l_s) + q u (1 - t u)   (Taylor, error ~u^3/3),
    // a^l_s = ah^l_s + e^l_s.  |e| stays near 2^-11, so the dropped term is below 1e-9:
    // a^l_s is the exact-form tanh of the exact y_l to rounding.  In the closed loop the
    // speculative input of layer 1 is the chain's own ah^M_{s-1}, with e^0_s = e^M_{s-1}.
    for (int s = s0; s <= s1; ++s) {
        const long long t = kW + s;
        if (warp == 0) {
            if (chain && s < s1) {
                const float* rowp = slot + lane * P + s;  // layer 0, position s
                const bool newest = s > s0;                       // lag 1 not applied yet
                const bool lag2 = (s & 1) ? s > s0 + 1 : s > s0;  // lag 2 not applied yet
                const bool zero = t == 0;                         // position 0 has no block
                float pp[MAXM];
#pragma unroll
                for (int l = 1; l <= MAXM; ++l) {
                    const int lc = l <= M ? l : M;
                    float v = zero ? 0.f : rowp[lc * CPB * P];
                    if (newest) v = fmaf(h1r[l - 1], rget(R, MAXM + l - 1), v);
                    if (lag2) v = fmaf(rget(R, l - 1), rowp[(lc - 1) * CPB * P - 2], v);
                    pp[l - 1] = v;
                }
                const float a0 = (a.closed && newest) ? aMsp : rowp[0];
                float2* xo = xch + (s & 1) * M * CPB + lane;
                float ah = a0;
#pragma unroll
                for (int l = 1; l <= MAXM; ++l) {
                    if (EXACT || l <= M) {
                        rset(R, MAXM + l - 1, ah);
                        const float yh = fmaf(h0r[l - 1], ah, pp[l - 1]);
                        ah = sfu_tanh(yh);
                        xo[(l - 1) * CPB] = make_float2(yh, ah);
                    }
                }
                aMsp = ah;
            }
        } else if (warp == kWinExactWarp) {
            if (s > s0) {
                const int tau = s - 1;
                float2* xb = xch + (tau & 1) * M * CPB;  // this token's (yh, ah), owned by warp 1 now
                const float yM = chain ? xb[(M - 1) * CPB + lane].x : 0.f;
                __syncwarp();
                // phase 1, every lane: the exact-form tanh t of the speculative pre-activations
                // of (layer l, chain c) = (q / CPB + 1, q % CPB), entry q = lane + 32 r,
                // written over yh
                const int nq = M * CPB;
                for (int q0 = 0; q0 < nq; q0 += 128) {
                    float yv[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int q = q0 + lane + 32 * r;
                        yv[r] = q < nq ? xb[q].x : 0.f;
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int q = q0 + lane + 32 * r;
                        if (q < nq) xb[q].x = act_tanh(yv[r]);
                    }
                }
                __syncwarp();
                // phase 2, lane c < ncb: the residual recurrence of chain c through the layers
                if (chain) {
                    const bool lag1 = tau > s0;  // the chain used its speculative a_{tau-1}
                    float e = (a.closed && lag1) ? eM : 0.f;
                    float* rowo = slot + lane * P + tau;
                    float* rowd = dup + lane * P + tau + 1;
                    float2 xv[MAXM];  // (t, ah) of every layer, loaded before the first store
#pragma unroll
                    for (int l = 1; l <= MAXM; ++l)
                        if (EXACT || l <= M) xv[l - 1] = xb[(l - 1) * CPB + lane];
                    float av = 0.f, u = 0.f;
#pragma unroll
                    for (int l = 1; l <= MAXM; ++l) {
                        if (EXACT || l <= M) {
                            // with u = h0 e + c1: q u = (q h0) e + q c1 and 1 - t u =
                            // (-t h0) e + (1 - t c1), so each link is two dependent FMAs
                            const float te = xv[l - 1].x, ah = xv[l - 1].y;
                            const float c1 = lag1 ? h1r[l - 1] * rget(R, 2 * MAXM + l - 1) : 0.f;
                            const float se = fmaf(-te, te, 1.f);
                            const float w = fmaf(se * h0r[l - 1], e, se * c1);
                            const float z = fmaf(-te * h0r[l - 1], e, fmaf(-te, c1, 1.f));
                            if (l == M) u = fmaf(h0r[l - 1], e, c1);
                            const float en = fmaf(w, z, te - ah);
                            rset(R, 2 * MAXM + l - 1, e);
                            e = en;
                            av = ah + en;
                            rowo[l * CPB * P] = av;
                            if (l < M) rowd[l * CPB * P] = av;
                        }
                    }
                    eM = e;
                    a.out[(kW + tau - a.tx) * G + gch] = yM + u;
                    if (a.closed) {
                        if (tau + 1 < W) {
                            slot[lane * P + tau + 1] = av;
                            dup[lane * P + tau + 2] = av;
                        } else if (kW + tau + 1 < L) {
                            a.act[gch * L + kW + tau + 1] = av;
                        }
                    }
                }
            }
        } else if (helper && s < s1) {
            const int T = s + 1;
            if (T < W) {
                int top;
                // a launch that starts the window holds every block covering T: lo = 0
                const int lo = s0 == 0 ? 0 : cover_range(T, s0, T, &top);
                // lags 3 .. T - lo of row T (lags 1 and 2 are the chain's), in K lag pairs
                // (3 + 2k, 4 + 2k); pair k = part + 2m belongs to this lane.  Pair k reads
                // positions (T - 4 - 2k, T - 3 - 2k), one aligned 8-byte load: from the
                // input row when T is even, else from its copy shifted by one position.
                const int dmax = T - lo;
                const int K = (dmax - 1) >> 1;
                const bool ow = kW == 0 && lo == 0;
                const float* pb = (T & 1) ? sm + dup0 + first.in + T - 3 : sm + first.in + T - 4;
                float acc = 0.f;
                if (first.out >= 0) {
                    if (lo == 0) {
                        // uniform over the CTA; reads reach down to position -31
                        acc = dot_lags2_padded<NTR2>(pb - 2 * part, R, (((K + 1) >> 1) + 7) >> 3);
                    } else {
                        const int nm_me = (K - part + 1) >> 1;
                        const int nm_both = ((dmax & 1) ? K - 1 : K) >> 1;  // pairs whole for both lanes
                        const bool last_half = (dmax & 1) && (((K - 1) & 1) == part);
                        acc = dot_lags2<NTR2>(pb - 2 * part, R, nm_both, nm_me, last_half);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (part == 0 && first.out >= 0) {
                    float* o = sm + first.out + T;
                    *o = ow ? acc : *o + acc;
                }
                if (more) helper_rows_more(sm, geom, pair, T, lo, s - 2, ow, part);
            }
        }
        __syncthreads();
    }

    // ---- a launch that stops inside the window completes the blocks it released:
    // position s1 still lacks its lag-1 and lag-2 terms (lag 2 only when its block was
    // released after s0), later positions the rows of blocks released in (s0, s1]
    if (s1 < W && s1 > s0) {
        if (warp == 0 && chain) {
            const bool lag2 = (s1 & 1) ? s1 > s0 + 1 : true;
            for (int l = 1; l <= M; ++l) {
                const float* tl = tap + ((l - 1) * kch + cich) * P;
                const float* in = slot + ((l - 1) * CPB + lane) * P;
                float* o = slot + (l * CPB + lane) * P + s1;
                float v = fmaf(tl[1], in[s1 - 1], *o);
                if (lag2) v = fmaf(tl[2], in[s1 - 2], v);
                *o = v;
            }
        }
        if (helper) {
            for (int T = s1 + 1; T < W; ++T) {
                int top;
                const int lo = cover_range(T, s0, s1, &top);
                if (lo >= 0) helper_rows(sm, geom, first, more, pair, T, lo, top, kW == 0 && lo == 0, part);
            }
        }
        __syncthreads();
    }

    grid_dep_launch();

    // ---- write the window back (16-byte stores from position s0 rounded down to 4);
    // thread -> (column group, first row), rows advance by a fixed stride
    {
        constexpr int PER = W / 4;
        const int c4lo = s0 >> 2;
        const int span = PER - c4lo;
        const int rows = (M + 1) * ncb;
        const int rstride = NT / span;  // span <= W/4 <= 64 < NT
        const int c4 = c4lo + tid % span;
        int row = tid / span;
        if (row < rstride) {
            int l = row / ncb, i = row - l * ncb;
            const int dl = rstride / ncb, di = rstride - dl * ncb;
            for (; row < rows; row += rstride) {
                const long long g = (long long)(i / nch) * D + c0 + (i % nch);
                const float* sp = slot + (l * CPB + i) * P + 4 * c4;
                *reinterpret_cast<float4*>(a.act + ((long long)l * G + g) * L + kW + 4 * c4) =
                    make_float4(sp[0], sp[1], sp[2], sp[3]);
                l += dl;
                i += di;
                if (i >= ncb) {
                    i -= ncb;
                    ++l;
                }
            }
        }
    }
}

// ----------------------------------------------------------------- read-out
// dst[(t - t0) * G + g] = act[layer][g][t] for t in [t0, t1)
__global__ void k_read_layer(const float* __restrict__ act, long long L, long long G, int layer,
                             long long t0, long long t1, float* dst) {
    const long long total = (t1 - t0) * G;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long g = e % G;
        const long long t = t0 + e / G;
        dst[e] = act[((long long)layer * G + g) * L + t];
    }
}

}  // namespace fi

// cluster FFT tau (blocks beyond one CTA's shared memory)
#include "fi_cluster.cuh"

// the Lazy and Eager baselines
#include "fi_baselines.cuh"

// the prompt prefill's element-wise kernels
#include "fi_prefill.cuh"

/*
 * fi.h -- C-ABI of the B200 Flash Inference mixer library (libfi.so).
 *
 * The library runs exact autoregressive inference of a stack of long causal
 * convolutions ("LCSM" mixers), one filter per layer and channel, with the
 * relaxed power-of-two tiling of the Flash Inference paper.  Citations below
 * name the web summary of arXiv 2410.12982, "Flash Inference: Near Linear Time
 * Inference for Long Convolution Sequence Models and Beyond", by section:
 *
 *   [Def]   section "LCSM-spezifische Definition":
 *           mixer^l(y)_t = sum_{i<=t} y_i (.) rho^l_{t-i}  (per channel, depthwise)
 *   [Alg1]  section "Kachelung-Strategie (Algorithmus 1)": after token i, with U the
 *           largest power of two dividing i, the red cell z_i += y_i rho_0 and the
 *           gray block z[i+1 .. i+U] += tau(y, [i-U+1, i], rho, [i+1, i+U])
 *   [Alg2]  section "LCSM-Inferenz-Algorithmus (Algorithmus 2)": the same over M
 *           layers, a^l_i = block^l(b^l_i), a^0_{i+1} = sampler(a^M_i)
 *   [Alg3]  section "Schicht-uebergreifende Parallelisierung (Algorithmus 3)": red
 *           cells in layer order, the gray blocks of all layers in parallel
 *   [Mem]   section "Speicheroptimierung": a^l_i reuses the storage of b^l_i; the
 *           DFT of the filters is precomputed per block size
 *   [Circ]  section "Zirkulaere Faltungs-Trick": a 2U circular convolution suffices
 *   [Impl]  section "Implementierungsdetails": CUDA graphs per token, FFT precompute,
 *           Hybrid choice of the tau implementation by block size
 *   [Base]  section "Kern-Algorithmus: Relaxierte Polynominterpolation", part 1 (the
 *           Lazy and Eager evaluations) and "Vergleichsmethoden" (their parallel
 *           versions as the baselines)
 *   [Pre]   the rebuttal's note on prefill (appendix A.3 as cited there): the prompt
 *           is taken eagerly before the autoregressive stage
 *   [Lem1]  section "Beitrags-Aggregations-Definition", Lemma 1:
 *           tau(y,[l,r],rho,[l',r'])_t = sum_{i=l}^{r} y_i rho_{t-i}
 *
 * Model computed (block^l = tanh, sampler = tanh):
 *   y^l_t = sum_{s<=t} h^l[c][t-s] * a^{l-1}_s[b][c],   a^l_t = tanh(y^l_t),
 *   a^0_t = x_t (teacher-forced) or a^0_{t+1} = a^M_t (closed loop).
 * Positions t are 0-based; the pages' loop counter i is n = t + 1.
 *
 * Conventions for every entry point:
 *   - Arrays are fp32, row-major.  A "chain" is one (b, c) pair, index g = b*D + c.
 *   - Per-token arrays are [B][D]; sequences are [steps][B][D] (time-major).
 *   - Pointers may be host or device memory unless stated otherwise; the library
 *     detects which (cudaPointerGetAttributes).  Calls with host destinations
 *     return after the data has arrived; calls with device destinations are
 *     asynchronous on the context's stream.
 *   - The library never takes ownership of, frees or retains caller memory.
 *   - Return values: FI_OK (0) or a negative FI_E* code; the message of the last
 *     failure on the calling thread is available from fi_last_error().
 *   - A context is not thread-safe; distinct contexts are independent.
 */
#ifndef FI_H_
#define FI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FI_OK 0
#define FI_EINVAL (-1)      /* bad argument: dims, L not a power of two, null pointer */
#define FI_ECAPACITY (-2)   /* the call would run past position L-1 */
#define FI_ENOMEM (-3)      /* device or host allocation failed */
#define FI_ECUDA (-4)       /* a CUDA call failed; message carries cudaGetErrorString */
#define FI_ESTATE (-5)      /* null or destroyed context */

/* tau implementations ([Impl] Hybrid) */
#define FI_TAU_AUTO 0       /* measured choice per block size (the Hybrid scheme) */
#define FI_TAU_DIRECT 1     /* direct convolution of the block, U^2 multiply-adds */
#define FI_TAU_FFT 2        /* FFT of the 2U circular convolution against a precomputed
                               filter spectrum ([Circ], [Mem]) */

/* execution paths of a generation */
#define FI_PATH_WINDOW 0    /* default: one persistent kernel per aligned window of W
                               tokens (red cells + all blocks smaller than W, in shared
                               memory), one launch per larger block */
#define FI_PATH_TOKEN 1     /* the pages' design ([Impl]): per token the step kernel (red
                               cells of every layer), the block it releases over every
                               layer, and an advance of the device-side step record; with
                               graphs on, those launches are one captured CUDA graph per
                               block size 2^q (one more for the last token), replayed per
                               token with the token index read from device memory */
#define FI_PATH_LAZY 2      /* baseline ([Base] "Lazy"): y^l_t summed over the whole history
                               when token t needs it, O(t) per token; one launch per token */
#define FI_PATH_EAGER 3     /* baseline ([Base] "Eager"): each activation pushed onto every
                               later position as soon as it is known, O(L-t) per token */
#define FI_PATH_LAZY_NP 4   /* baseline ([Base] "Lazy NP"): Lazy without cross-layer
                               parallelism, one launch per layer and token, in layer order */
#define FI_PATH_EAGER_NP 5  /* baseline ([Base] "Eager NP"): Eager without cross-layer
                               parallelism, one launch per layer and token, in layer order */

typedef struct fi_ctx fi_ctx;

typedef struct fi_info {
    int layers, B, D, L;        /* as created */
    int t;                      /* tokens processed so far (next position) */
    int window;                 /* W of the window path */
    int chains_per_cta;         /* chains held by one CTA of the window kernel */
    int path;                   /* FI_PATH_* in use */
    int graphs;                 /* 1 if launches are replayed from captured CUDA graphs */
    int tau[32];                /* FI_TAU_DIRECT / FI_TAU_FFT chosen for block size 2^q */
    float tau_us[32][2];        /* measured microseconds per launch [q][direct, fft]; 0 = not timed */
    size_t device_bytes;        /* device memory held by the context */
    int sm_count;               /* SMs of the device */
    long long launches;         /* kernels launched by this context's runs so far */
} fi_info;

/* kernel classes reported by fi_trace_read */
#define FI_K_WINDOW 0        /* window kernel: red cells + blocks smaller than W */
#define FI_K_TOKEN_STEP 1    /* per-token step kernel: red cells (+ small blocks) */
#define FI_K_BLOCK_DIRECT 2  /* one block size, every layer and chain, direct tau */
#define FI_K_BLOCK_FFT 3     /* one block size, every layer and chain, fused FFT tau */
#define FI_K_BLOCK_CLUSTER 4 /* blocks larger than one CTA's FFT: FFT tau on a cluster of CTAs */
#define FI_K_CLASSES 5

typedef struct fi_trace {
    int launches[FI_K_CLASSES];     /* launches of each class in the last run */
    double total_us[FI_K_CLASSES];  /* summed device time of those launches */
    double max_us[FI_K_CLASSES];    /* longest single launch */
    int block_launches[32];         /* block launches of edge 2^q */
    double block_us[32];            /* their summed device time */
} fi_trace;

/* Create a context for `layers` stacked mixers over B sequences of D channels,
 * capacity L positions.  filters: [layers][D][L] fp32 (host or device), filter of
 * layer l (0-based), channel c, lag k at filters[(l*D + c)*L + k] ([Def]).  The
 * filters are copied; the caller keeps ownership.  L must be a power of two >= 2.
 * Precomputes the filter spectra for every block size served by FFT ([Mem]) and
 * measures the tau choice per block size ([Impl] Hybrid).  Returns NULL on error
 * (see fi_last_error).  The context starts at t = 0. */
fi_ctx *fi_create(int layers, int B, int D, int L, const float *filters);

/* Release every resource of the context.  NULL is accepted. */
void fi_destroy(fi_ctx *ctx);

/* Teacher-forced single token ([Alg2] one loop iteration): x_t [B][D] is token t
 * (t = the context's counter); y_t [B][D] receives y^M_t, the last layer's mixer
 * output before tanh.  Afterwards every gray block released by this token has been
 * applied and t advances by one.  FI_ECAPACITY if t == L. */
int fi_step(fi_ctx *ctx, const float *x_t, float *y_t);

/* Closed-loop generation of `steps` tokens from the current position t
 * ([Alg2], sampler = tanh): x0 [B][D] is token t, or NULL to continue from the
 * token the previous closed-loop call produced (a^M_{t-1}).  out [steps][B][D]
 * receives y^M_t .. y^M_{t+steps-1}; token t+1 = tanh(y^M_t) stays on the device.
 * FI_ECAPACITY if t + steps > L.  steps == 0 is a no-op. */
int fi_generate(fi_ctx *ctx, const float *x0, int steps, float *out);

/* Teacher-forced run over `steps` tokens (the windowed form of fi_step):
 * x [steps][B][D] are tokens t .. t+steps-1, y [steps][B][D] receives y^M. */
int fi_forward(fi_ctx *ctx, const float *x, int steps, float *y);

/* Prompt prefill ([Pre]): the p-token prompt x [p][B][D] (teacher-forced tokens
 * 0..p-1) folded in layer by layer with one FFT convolution per layer (the block tau
 * of [Lem1] with U = the power of two >= p and the taps shifted by U, so that only
 * lags 0..t reach position t) instead of p online steps; y [p][B][D] receives y^M of
 * the prompt positions.  Afterwards t = p and the buffers hold exactly the tiled
 * paths' state (every block released up to p applied, activations final below p),
 * so fi_generate / fi_forward / fi_step continue the sequence.  Needs t = 0 (after
 * fi_create or fi_reset) and a tiled path (FI_PATH_WINDOW or FI_PATH_TOKEN), else
 * FI_EINVAL; 1 <= p <= L.  Prompts shorter than 8 tokens take the online path.
 * The context keeps 4 * B * D * (2U + M (p - n0)) bytes of device scratch (n0 the
 * largest power of two <= p) and the spectra of the shifted taps of the prompt's size,
 * 8 * M * D * (U + 2) bytes, made by the first prefill of that size and reused by later
 * ones (FI_ENOMEM if it cannot get them); both are freed with the context.  Asynchronous on the context's stream like fi_forward; with host buffers
 * it synchronises before returning. */
int fi_prefill(fi_ctx *ctx, const float *x, int p, float *y);

/* Rewind to t = 0 for a new sequence.  O(1): stale buffer contents are never read
 * (the first block written onto any position overwrites instead of accumulating). */
int fi_reset(fi_ctx *ctx);

/* Copy the realised activations a^layer_s for s in [t0, t1) into dst
 * [t1-t0][B][D]; layer 0 is the input sequence, layer l >= 1 is tanh(y^l).
 * Requires 0 <= t0 <= t1 <= t (only finalised positions can be read). */
int fi_read_layer(fi_ctx *ctx, int layer, int t0, int t1, float *dst);

/* Use `stream` (a cudaStream_t, NULL = legacy default stream) for all later work. */
int fi_set_stream(fi_ctx *ctx, void *stream);

/* Choose the execution path (FI_PATH_*).  The two tiled paths (WINDOW, TOKEN) share
   their buffer state and may be switched at any token; the baselines (LAZY, EAGER and
   their NP forms) keep their own state, so a change to or from them is accepted only
   at t = 0 (after fi_create or fi_reset), else FI_EINVAL.  LAZY and EAGER are the
   pages' parallel baselines: the part of token t that does not depend on its own layer
   chain runs for every layer at once; LAZY_NP and EAGER_NP do each layer's share as a
   launch of its own, layer after layer.  The baselines take no graphs and record no
   trace. */
int fi_set_path(fi_ctx *ctx, int path);

/* Enable (1) or disable (0) replay of captured CUDA graphs ([Impl]).  Window path:
 * the launch sequence of a whole call is captured once per call shape and replayed.
 * Per-token path (and fi_step): one graph per block size, captured on first use and
 * replayed per token.  With graphs off every launch is issued from the host.  Graphs
 * are re-captured after fi_set_tau or fi_set_trace; the per-token graphs carry no trace
 * events, so with tracing on the per-token path launches from the host. */
int fi_set_graphs(fi_ctx *ctx, int on);

/* Override the tau choice for block size 2^q (FI_TAU_AUTO restores the measured
 * choice).  FI_EINVAL if the implementation cannot serve that size in this
 * context (FFT needs the spectrum of that size). */
int fi_set_tau(fi_ctx *ctx, int q, int impl);

/* Bracket every kernel launch of later runs with CUDA events (on = 1), also inside
 * captured graphs; off by default.  Toggling re-captures graphs. */
int fi_set_trace(fi_ctx *ctx, int on);

/* Per kernel class: launches and device time of the most recent run (fi_step,
 * fi_generate or fi_forward call) made with tracing on.  Synchronises the stream. */
int fi_trace_read(fi_ctx *ctx, fi_trace *out);

/* The launches of the most recent traced run, in issue order: kernel class (FI_K_*),
 * block size exponent q (-1 for launches that are not block launches) and device time
 * in microseconds of launch i in cls[i], q[i], us[i] for i < max.  Returns the number of
 * launches the run made (which may exceed max), or a negative FI_E* code.  Synchronises
 * the stream. */
int fi_trace_launches(fi_ctx *ctx, int max, int *cls, int *q, float *us);

/* Fill *info with the context's shape, state and tau table. */
int fi_get_info(const fi_ctx *ctx, fi_info *info);

/* The gray block released after the n-th token ([Alg1], 1 <= n <= L-1): its edge
 * U = lowbit(n), input positions [src_lo, n-1], output positions [n, dst_hi]
 * (dst_hi clipped to L-1) and the tau implementation the context will use. */
int fi_debug_schedule(const fi_ctx *ctx, int n, int *U, int *impl, int *src_lo,
                      int *dst_lo, int *dst_hi);

/* Stand-alone tau ([Lem1]) over `count` independent blocks of edge U, all pointers
 * DEVICE memory:  out[i][r] (+)= sum_{j<U} blocks[i][j] * taps[i*ldt + U + r - j],
 * r < U (lags 1 .. 2U-1 of each filter row; ldt >= 2U).  accumulate = 0 overwrites.
 * impl: FI_TAU_DIRECT (U <= 4096) or FI_TAU_FFT (8 <= U <= 131072, ldt even; out
 * 16-byte aligned, blocks and taps 8-byte aligned).  Runs on the legacy default stream and
 * returns after completion.  Used to test each tau kernel in isolation. */
int fi_tau(int impl, int U, int count, const float *blocks, const float *taps, int ldt,
           float *out, int accumulate);

/* The FFT tau of fi_tau (impl = FI_TAU_FFT) for callers that must not allocate
 * device memory.  The paper has no counterpart: this entry point exists for
 * callers whose device memory is owned by someone else -- an application whose
 * pool allocator has reserved the GPU's memory up front (so cudaMalloc fails or
 * fragments that pool), or a loop that cannot afford the device-wide
 * synchronisation cudaMalloc and cudaFree may imply.
 * Arguments and result are those of fi_tau with impl = FI_TAU_FFT: count blocks of
 * edge U (8 <= U <= 65536, a power of two), taps rows of ldt >= 2U (even) floats,
 * out[i][r] (+)= tau; all pointers DEVICE memory, out 16-byte and blocks, taps
 * 8-byte aligned; the caller owns them.  Every temporary (twiddle table, filter
 * spectra) lives in one fixed 8 MiB array in device memory, part of the library image, which every
 * GPU that loads the library holds until the process exits; large counts are
 * processed in chunks that fit it.  The first call on a device sets that device up
 * (looks up the array's device address and writes the twiddle table with a
 * synchronous copy), so make it before any stream capture.  The set-up is tied to
 * the device's context: after a cudaDeviceReset (or any teardown of the context) the
 * library is loaded afresh with a new array, and the next call repeats the set-up.  Nothing in the array
 * needs to start at zero: each call writes every part it reads.  All calls share
 * the array, so calls that overlap on the GPU race (for example from two host
 * threads); calls are serialised on the legacy default stream and return after
 * completion.  FI_EINVAL for U beyond 65536 (or any fi_tau argument error). */
int fi_tau_fft_noalloc(int U, int count, const float *blocks, const float *taps, int ldt,
                       float *out, int accumulate);

/* ---------------------------------------------------------------- language model
 * A Hyena-like language model built around the mixer: the pages describe an LCSM layer
 * as the mixer followed by a block with "MLP, Schicht-Normalisierung, etc." (section
 * "Modellarchitektur") and measure a Hyena model with random weights end to end
 * (sections "Experimentelle Einrichtung", "Hauptergebnisse").  Per token t, batch row b
 * (u: residual stream of D values; LN: layer norm without affine parameters, eps 1e-5;
 * bf16(.): rounding to bfloat16, the operand of a bf16 GEMM with fp32 accumulation):
 *   u = E[tok_t];  for each layer l:
 *     z = W_in^l bf16(LN(u)) = (q, k, v);   zc_t = c0 z_t + c1 z_{t-1} + c2 z_{t-2}
 *     x_t = kc vc;   y_t = sum_{s<=t} h^l[t-s] x_s  (the mixer, fp32, relaxed tiling)
 *     u += qc y_t;   u += W2^l bf16(GELU(W1^l bf16(LN(u))))
 *   logits = W_lm bf16(LN(u));   greedy: tok_{t+1} = argmax (lowest id among equal maxima)
 * Weights arrive as fp32 arrays holding bf16 values (host or device), row-major:
 * E, W_lm [V][D]; W_in [layers][3D][D]; conv [layers][3][3D] (taps c0, c1, c2, fp32);
 * W1 [layers][4D][D]; W2 [layers][D][4D]; filters [layers][D][L] fp32.  They are copied.
 * 1 <= B <= 8, D a multiple of 8, L a power of two.  Token arrays are int32, host or
 * device.  Returns NULL on error (fi_last_error). */
typedef struct fi_lm fi_lm;
fi_lm *fi_lm_create(int layers, int B, int D, int L, int V, const float *E, const float *W_lm,
                    const float *W_in, const float *conv, const float *W1, const float *W2,
                    const float *filters);

/* Release the model.  NULL is accepted. */
void fi_lm_destroy(fi_lm *m);

/* Rewind to t = 0 (a new sequence; the short-convolution history restarts at zero). */
int fi_lm_reset(fi_lm *m);

/* Teacher-forced tokens t .. t+steps-1: tokens [steps][B] are the inputs; logits
 * [steps][B][V] receives the logits (NULL: not returned); next [steps][B] the greedy
 * choices.  FI_ECAPACITY past L. */
int fi_lm_forward(fi_lm *m, const int *tokens, int steps, float *logits, int *next);

/* Greedy generation of `steps` tokens: tok0 [B] is the input at the current position
 * (NULL: continue from the previous call's last choice; required at t = 0); next
 * [steps][B] receives each step's choice, which is the following step's input. */
int fi_lm_generate(fi_lm *m, const int *tok0, int steps, int *next);

/* Greedy generation replays one captured CUDA graph per block size ([Impl]: the
 * launches of one token recorded once; the token index read from device memory) when
 * on (the default); off, or with tracing on, every launch is issued from the host. */
int fi_lm_set_graphs(fi_lm *m, int on);

/* Tracing (off by default): later calls record events around every block launch of
 * the mixers and around the mixer steps of every 64th token. */
int fi_lm_set_trace(fi_lm *m, int on);

/* Of the most recent traced call: its device time (total_us) and the part spent in
 * the mixers (mixer_us: the block launches, plus the sampled mixer steps scaled to
 * every token).  Synchronises. */
int fi_lm_split(fi_lm *m, double *mixer_us, double *total_us);

/* ---------------------------------------------------------------- data-dependent filter
 * The long convolution with a filter that depends on the data (the Flash Inference
 * summary, section "Technische Innovationen" item 4, "Datenabhaengige
 * Filter-Erweiterung"; the rebuttal's answer on data-dependent filters: a different
 * tiling with two FFT convolutions of the same size per step, at twice the cost).  G
 * independent channels; at step t the input x_t and the filter value rho_t of every
 * channel arrive together, and
 *     y_t = sum_{i + j = t} rho_i x_j
 * is returned before step t + 1 (the definition is the causal convolution; only what
 * is known when differs from a fixed filter).  Tiling (the appendix that holds the
 * pages' algorithm is not on the pages; this is the reading the library follows):
 * red cells rho_0 x_t + rho_t x_0 at step t; after the n-th token, U = lowbit(n),
 * Algorithm 1's block with x[n-U, n) as the input and rho[0, 2U) as the taps and,
 * unless n is a power of two, the same block with the roles swapped; at n = U the
 * x-block runs while rho[U, 2U) is still zero, which adds exactly the products of the
 * first U values of both sequences that are still due.  A block of size U takes the
 * direct tau or the FFT tau against the spectra of the prefixes x[0, 2U), rho[0, 2U),
 * made once at step 2U (when they are final; first used at step 3U).
 * Layout: x, rho and the running sums are [G][L] float32 on the device. */
typedef struct fi_dd fi_dd;

/* G >= 1 channels; L a power of two, 2 <= L <= 2^17.  Device memory: 3 G L floats (x,
 * rho, running sums) plus about 1.5 G L complex values of spectra (both prefixes for
 * every block size up to L/4, and the power-of-two block's up to L/2).  Returns NULL
 * on error (fi_last_error). */
fi_dd *fi_dd_create(int G, int L);

/* Release the context.  NULL is accepted. */
void fi_dd_destroy(fi_dd *d);

/* Back to step 0 (clears the buffers). */
int fi_dd_reset(fi_dd *d);

/* Steps t .. t+steps-1: x and rho [steps][G] float32 (host or device) are the inputs of
 * those steps; y [steps][G] (host or device, not overlapping x or rho) receives the
 * outputs.  Each aligned window of 128 steps at or after step 128 that the call covers
 * whole is evaluated in one launch (its inputs are all given); other steps one at a
 * time.  FI_ECAPACITY past L; FI_EINVAL for a NULL array with steps > 0. */
int fi_dd_forward(fi_dd *d, const float *x, const float *rho, int steps, float *y);

/* The implementation of blocks of size 2^q: FI_TAU_DIRECT (q <= 12), FI_TAU_FFT
 * (q >= 3), or FI_TAU_AUTO for the default (direct up to U = 8, added by the step
 * kernel itself; FFT above).  Only before step 1 (FI_ESTATE after): the FFT form needs
 * the prefix spectra made at step 2U. */
int fi_dd_set_tau(fi_dd *d, int q, int impl);

/* Message of the last failure on the calling thread ("" if none). */
const char *fi_last_error(void);

/* Library version string. */
const char *fi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FI_H_ */

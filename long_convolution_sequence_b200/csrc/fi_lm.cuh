// fi_lm.cuh -- device code of the Hyena-like language model around the mixer
// (sm_100a): the parts of a layer outside the long convolution, per token.
//
// The Flash Inference summary describes an LCSM layer as the mixer followed by a
// block with "MLP, Schicht-Normalisierung, etc." (section "Modellarchitektur") and
// measures a Hyena model with random weights end to end (sections "Experimentelle
// Einrichtung", "Hauptergebnisse").  The layer computed here, per token t and batch
// row b (u: the residual stream, D values):
//   z = W_in bf16(LN(u))                  3D values (q, k, v)         k_lm_gemv, LN
//   zc_t = c0 z_t + c1 z_{t-1} + c2 z_{t-2}, x_t = kc vc              k_lm_mixer
//   y_t  = running sum of the blocks + h_0 x_t   (the red cell)        k_lm_mixer
//   u   += qc y_t                                                      k_lm_mixer
//   u   += W2 bf16(GELU(W1 bf16(LN(u))))                               k_lm_gemv x2
// then logits = W_lm bf16(LN(u)) and the greedy next token (k_lm_argmax).  The gray
// blocks of the mixers (the long convolutions' history) are the block kernels of
// fi_kernels.cuh over the mixer inputs x of every layer, written onto the running
// sums y of the same layer.
//
// Every GEMM here has B (at most 8) rows: with bf16 weights it moves 2 bytes per
// weight for 2 B flops, far below what tensor cores are for, so these are weight-
// streaming matrix-vector kernels on the CUDA cores (16-byte weight loads, fp32
// accumulation; the activation rounded to bf16 as a bf16 GEMM's operand).
#pragma once
#include <cuda_bf16.h>

namespace fi {

constexpr int kLmMaxB = 8;        // batch rows per launch
constexpr int kLmThreads = 128;   // threads of the matrix-vector kernels (4 warps: small N still fills the SMs)
constexpr int kLmUnroll = 4;      // 16-byte weight loads a lane keeps in flight
constexpr float kLmLnEps = 1e-5f;

enum LmEpilogue { kLmStore = 0, kLmGelu = 1, kLmAdd = 2 };

// u[b][:] = E[tok[b]][:] (bf16 embedding rows to fp32)
//
// The kernels are written to run under programmatic dependent launch (they read
// nothing their predecessors write before griddepcontrol.wait, and the matrix-vector
// kernels prefetch their weight rows into L2 before it), but the host launches them
// without it: releasing each successor at once made the launches cascade and the
// waiting CTAs crowd the running kernel.  Reads of data another kernel writes go
// through L2 only (ld.global.cg), which stays correct however the launches overlap.
__global__ void k_lm_embed(const __nv_bfloat16* __restrict__ E, const int* __restrict__ tok, int B, int D,
                           float* __restrict__ u) {
    grid_dep_launch();
    grid_dep_wait();
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < B * D; e += gridDim.x * blockDim.x) {
        const int b = e / D, d = e - b * D;
        u[e] = __bfloat162float(E[(long long)__ldcg(tok + b) * D + d]);
    }
}

// y[b][n] (epilogue)= sum_k W[n][k] bf16(pre(x[b][k])), n < N, b < B; pre = layer norm
// over the row (ln = 1) or the identity.  Each warp takes rows n = warp + j * warps
// (grid-stride over the launch); the B input rows, normalised and rounded to bf16, sit in
// shared memory as fp32.  Epilogue: store, GELU then store, or add onto y (residual).
template <int EPI>
__global__ void __launch_bounds__(kLmThreads) k_lm_gemv(const __nv_bfloat16* __restrict__ W, int N, int K,
                                                        const float* __restrict__ x, int B, int ln,
                                                        float* __restrict__ y) {
    extern __shared__ float xs[];  // [B][K]
    __shared__ float stat[kLmMaxB][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kLmThreads / 32;
    grid_dep_launch();
    // this CTA's weight rows into L2 (128-byte lines), before waiting for the input
    {
        const int lines = K * 2 / 128;  // whole 128-byte lines of a row (a partial last one is left out)
        for (int n0 = blockIdx.x * nw; n0 < N; n0 += gridDim.x * nw) {
            const int rows = min(nw, N - n0);
            const char* base = reinterpret_cast<const char*>(W + (long long)n0 * K);
            for (int i = threadIdx.x; i < rows * lines; i += kLmThreads)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(base + (long long)i * 128));
        }
    }
    grid_dep_wait();
    for (int e = threadIdx.x; e < B * K; e += kLmThreads) xs[e] = __ldcg(x + e);
    __syncthreads();
    if (ln) {
        // mean and variance of row b by warp b (two passes over shared memory)
        for (int b = warp; b < B; b += nw) {
            float s = 0.f;
            for (int k = lane; k < K; k += 32) s += xs[b * K + k];
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const float mean = s / (float)K;
            float v = 0.f;
            for (int k = lane; k < K; k += 32) {
                const float d = xs[b * K + k] - mean;
                v = fmaf(d, d, v);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) {
                stat[b][0] = mean;
                stat[b][1] = 1.0f / sqrtf(v / (float)K + kLmLnEps);
            }
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < B * K; e += kLmThreads) {
        const int b = e / K;
        const float v = ln ? (xs[e] - stat[b][0]) * stat[b][1] : xs[e];
        xs[e] = __bfloat162float(__float2bfloat16_rn(v));
    }
    __syncthreads();
    // rows: 8 bf16 weights per 16-byte load, lanes stride over the row, kLmUnroll loads
    // in flight per lane before they are used
    const int K8 = K / 8;
    for (int n = blockIdx.x * nw + warp; n < N; n += gridDim.x * nw) {
        const uint4* wr = reinterpret_cast<const uint4*>(W + (long long)n * K);
        float acc[kLmMaxB];
#pragma unroll
        for (int b = 0; b < kLmMaxB; ++b) acc[b] = 0.f;
        for (int v0 = lane; v0 < K8; v0 += 32 * kLmUnroll) {
            uint4 pk[kLmUnroll];
#pragma unroll
            for (int u = 0; u < kLmUnroll; ++u) {
                const int v8 = v0 + 32 * u;
                pk[u] = v8 < K8 ? __ldg(wr + v8) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kLmUnroll; ++u) {
                const int v8 = v0 + 32 * u;
                if (v8 < K8) {
                    const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&pk[u]);
                    float w[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = __bfloat1622float2(w2[i]);
                        w[2 * i] = f.x;
                        w[2 * i + 1] = f.y;
                    }
#pragma unroll
                    for (int b = 0; b < kLmMaxB; ++b) {
                        if (b < B) {
                            const float4* xr = reinterpret_cast<const float4*>(xs + b * K + 8 * v8);
                            const float4 x0 = xr[0], x1 = xr[1];
                            float a = acc[b];
                            a = fmaf(w[0], x0.x, a);
                            a = fmaf(w[1], x0.y, a);
                            a = fmaf(w[2], x0.z, a);
                            a = fmaf(w[3], x0.w, a);
                            a = fmaf(w[4], x1.x, a);
                            a = fmaf(w[5], x1.y, a);
                            a = fmaf(w[6], x1.z, a);
                            a = fmaf(w[7], x1.w, a);
                            acc[b] = a;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kLmMaxB; ++b) {
            if (b < B) {
                float a = acc[b];
#pragma unroll
                for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                if (lane == 0) {
                    if (EPI == kLmGelu) a = 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
                    if (EPI == kLmAdd) y[(long long)b * N + n] = __ldcg(y + (long long)b * N + n) + a;
                    else y[(long long)b * N + n] = a;
                }
            }
        }
    }
}

// The mixer part of layer l at token t, one thread per (b, d): short convolution of the
// three in-projection streams (q, k, v) with the two previous tokens' values (ring
// zr[2][B][3D], shifted here), the gate x = kc vc stored as the mixer's input at t, the
// red cell y_t = (running sum at t) + h_0 x_t (the running sum is 0 at t = 0, where no
// block has written), y_t kept at t, and the gated residual u += qc y_t.
// With io (a replayed per-token graph) the token index comes from the step record.
__global__ void k_lm_mixer(const float* __restrict__ z, float* __restrict__ zr, const float* __restrict__ conv,
                           const float* __restrict__ h, long long L, int B, int D, long long t, float* X,
                           float* Y, float* u, const TokIO* io) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    grid_dep_launch();
    grid_dep_wait();
    if (io) t = io->t;
    if (e >= B * D) return;
    const int b = e / D, d = e - b * D;
    const int D3 = 3 * D;
    float zc[3];
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int j = s * D + d;
        const float z0 = __ldcg(z + b * D3 + j);
        float* r1 = zr + (long long)b * D3 + j;                 // z_{t-1}
        float* r2 = zr + (long long)B * D3 + (long long)b * D3 + j;  // z_{t-2}
        const float z1 = __ldcg(r1), z2 = __ldcg(r2);
        zc[s] = fmaf(conv[j], z0, fmaf(conv[D3 + j], z1, conv[2 * D3 + j] * z2));
        *r2 = z1;
        *r1 = z0;
    }
    const float x = zc[1] * zc[2];
    const long long g = (long long)b * D + d;
    X[g * L + t] = x;
    const float run = t == 0 ? 0.f : __ldcg(Y + g * L + t);
    const float yv = fmaf(h[(long long)d * L], x, run);
    Y[g * L + t] = yv;
    u[e] = fmaf(zc[0], yv, __ldcg(u + e));
}

// next[b] = argmax_v logits[b][v] (the lowest id among equal maxima), one CTA per row;
// also written to out[b] when given, and used as the next input token.  With io (a
// replayed per-token graph) out is the record's choice array at the record's token, and
// with advance this launch closes the token.
__global__ void k_lm_argmax(const float* __restrict__ logits, int V, int* next, int* out, TokIO* io, int advance) {
    __shared__ float bv[32];
    __shared__ int bi[32];
    const int b = blockIdx.x;
    grid_dep_launch();
    grid_dep_wait();
    const float* row = logits + (long long)b * V;
    float best = -INFINITY;
    int idx = 0x7fffffff;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
        const float x = __ldcg(row + v);
        if (x > best || (x == best && v < idx)) {
            best = x;
            idx = v;
        }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
        if (ob > best || (ob == best && oi < idx)) {
            best = ob;
            idx = oi;
        }
    }
    if (lane == 0) {
        bv[warp] = best;
        bi[warp] = idx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (bv[w] > best || (bv[w] == best && bi[w] < idx)) {
                best = bv[w];
                idx = bi[w];
            }
        next[b] = idx;
        if (io) out = io->itok + (io->t - io->tx) * gridDim.x;
        if (out) out[b] = idx;
    }
    if (io && advance) tok_advance_if_last(io);
}

// dst[i] = bf16(src[i]) (weights arrive as fp32 values)
__global__ void k_to_bf16(const float* __restrict__ src, long long n, __nv_bfloat16* dst) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

}  // namespace fi

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
// then logits = W_lm bf16(LN(u)) and the greedy next token (folded into the LM head's
// epilogue, read by k_lm_pick).  The gray
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
constexpr int kLmThreads = 256;   // threads of the matrix-vector kernels (8 warps; at most 2 CTAs an SM)
constexpr int kLmCtasPerSm = 2;   // matrix-vector grid: one wave, so the per-CTA set-up (inputs, statistics) is paid once an SM slot
constexpr int kLmUnroll = 3;      // 16-byte weight loads a lane keeps in flight per row (a 768-value slice: all of it)
constexpr float kLmLnEps = 1e-5f;

enum LmEpilogue { kLmStore = 0, kLmGelu = 1, kLmAdd = 2, kLmArgmax = 3, kLmMix = 4 };

// Greedy choice folded into the LM head: a logit and its id as one 64-bit key whose
// unsigned order is the order of (logit, -id), so the maximum key over a row is its
// largest logit with the lowest id among equal maxima.
__device__ __forceinline__ unsigned long long lm_key(float v, int id) {
    const unsigned u = __float_as_uint(v);
    const unsigned o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)o << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)id);
}
__device__ __forceinline__ int lm_key_id(unsigned long long k) { return (int)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull)); }

// u[b][:] = E[tok[b]][:] (bf16 embedding rows to fp32)
//
// The kernels run under programmatic dependent launch: they read nothing their
// predecessors write before griddepcontrol.wait (the matrix-vector kernels prefetch
// their weight rows into L2 and issue their first weight loads before it), and each
// releases its successor only once its own wait has returned, so at most one launch
// waits behind the running one (releasing successors at kernel start made the
// launches cascade).  Reads of data another kernel writes go through L2 only
// (ld.global.cg), which stays correct however the launches overlap.
__global__ void k_lm_embed(const __nv_bfloat16* __restrict__ E, const int* __restrict__ tok, int B, int D,
                           float* __restrict__ u, unsigned long long* amax) {
    grid_dep_wait();
    grid_dep_launch();
    if (blockIdx.x == 0 && threadIdx.x < B) amax[threadIdx.x] = 0ull;  // this token's greedy choice starts empty
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < B * D; e += gridDim.x * blockDim.x) {
        const int b = e / D, d = e - b * D;
        u[e] = __bfloat162float(E[(long long)__ldcg(tok + b) * D + d]);
    }
}

// The mixer part of layer l at token t for batch row b and channel d, given the
// in-projection's q, k, v values of the token: short convolution of the three streams
// with the two previous tokens' values (ring zr[2][B][3D], shifted here), the gate
// x = kc vc stored as the mixer's input at t, the red cell y_t = (running sum at t) +
// h_0 x_t (the running sum is 0 at t = 0, where no block has written), y_t kept at t,
// and the gated residual r = u + qc y_t.  Its loads (MixOps) do not depend on q, k, v
// and are issued first.
struct MixOps {
    float z1[3], z2[3], c0[3], c1[3], c2[3];
    float h0, u0, run;
};

__device__ __forceinline__ MixOps lm_mixer_load(int b, int d, const float* zr, const float* __restrict__ conv,
                                                const float* __restrict__ h, long long L, int B, int D, long long t,
                                                const float* Y, const float* u) {
    MixOps o;
    const int D3 = 3 * D;
    const float* r1 = zr + (long long)b * D3 + d;                      // z_{t-1}
    const float* r2 = zr + (long long)B * D3 + (long long)b * D3 + d;  // z_{t-2}
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int j = s * D + d;
        o.z1[s] = __ldcg(r1 + s * D);
        o.z2[s] = __ldcg(r2 + s * D);
        o.c0[s] = __ldg(conv + j);
        o.c1[s] = __ldg(conv + D3 + j);
        o.c2[s] = __ldg(conv + 2 * D3 + j);
    }
    o.h0 = __ldg(h + (long long)d * L);
    const long long g = (long long)b * D + d;
    o.u0 = __ldcg(u + g);
    o.run = t == 0 ? 0.f : __ldcg(Y + g * L + t);
    return o;
}

__device__ __forceinline__ void lm_mixer_finish(const MixOps& o, float zq, float zk, float zv, int b, int d,
                                                float* zr, long long L, int B, int D, long long t, float* X, float* Y,
                                                float* r) {
    const int D3 = 3 * D;
    const float z0[3] = {zq, zk, zv};
    float* r1 = zr + (long long)b * D3 + d;
    float* r2 = zr + (long long)B * D3 + (long long)b * D3 + d;
    float zc[3];
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        zc[s] = fmaf(o.c0[s], z0[s], fmaf(o.c1[s], o.z1[s], o.c2[s] * o.z2[s]));
        r2[s * D] = o.z1[s];
        r1[s * D] = z0[s];
    }
    const long long g = (long long)b * D + d;
    const float xv = zc[1] * zc[2];
    X[g * L + t] = xv;
    const float yv = fmaf(o.h0, xv, o.run);
    Y[g * L + t] = yv;
    r[g] = fmaf(zc[0], yv, o.u0);
}

// Epilogue operands of the matrix-vector kernel beyond y.
struct LmEpi {
    unsigned long long* amax;  // kLmArgmax: running greedy choice per batch row
    const float* res;          // kLmAdd: y = res + W x (res may be y)
    // kLmMix: the mixer step of the layer (as k_lm_mixer), u the kernel's input x
    float* zr;
    const float* conv;
    const float* h;
    long long L;
    long long t;
    float* X;
    float* Y;
    const TokIO* io;
    int D;
};

// y[b][n] (epilogue)= sum_k W[n][k] a[b][k], n < N, b < B, where a = bf16(LN(x)) (ln = 1)
// or a = x, whose values are bf16 already (ln = 0: the GELU epilogue stores them so).
//
// Weight rows are read with 16-byte loads (8 bf16), lanes striding over a row.  A warp
// takes RPW rows at a time, all their loads issued before any is used (the first step's
// before the inputs are staged: they do not depend on them); with KS > 1 each row is
// split over KS warps, each summing a K / KS slice, the partial sums joined in shared
// memory.  The B input rows a sit in shared memory as fp32 in two planes, the first and
// second four values of every group of eight: the eight inputs matching a lane's weight
// load are then one 16-byte read in each plane, consecutive lanes reading consecutive 16
// bytes (no bank conflicts), and each read serves all RPW rows.
// Epilogue: store; GELU, rounded to bf16 (the next product's operand), then store;
// y = res + W a (residual); store (when y is given) and fold the row into the greedy
// choice (amax[b], keys of lm_key); or (kLmMix, RPW = 3) the mixer step: a warp takes
// the rows d, D + d, 2D + d of the in-projection (q, k, v of channel d) and finishes
// channel d as k_lm_mixer does, writing y = u + qc y_t (y is then not the input).
// BM >= B bounds the batch rows at compile time (4 or 8): the accumulators of a warp
// are RPW x BM registers.
template <int EPI, int KS, int RPW, int BM>
__global__ void __launch_bounds__(kLmThreads, kLmCtasPerSm) k_lm_gemv(const __nv_bfloat16* __restrict__ W, int N,
                                                                     int K, const float* __restrict__ x, int B,
                                                                     int ln, float* __restrict__ y, LmEpi ep) {
    extern __shared__ float xs[];  // planes [2][B][K / 2]
    __shared__ float part[kLmThreads / 32][RPW][BM];
    constexpr int nw = kLmThreads / 32;
    constexpr bool MIX = EPI == kLmMix;
    static_assert(!MIX || RPW == 3, "the mixer epilogue takes the q, k, v rows of a channel in one warp");
    // units: rows, or (MIX) channels whose three rows KS warps share
    constexpr int UPC = MIX ? nw / KS : (nw / KS) * RPW;  // units per CTA per step
    const int NU = MIX ? ep.D : N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KH = K / 2, K8 = K / 8;
    const int Kw = K / KS;  // this warp's slice of a row
    const int j0 = (KS > 1 ? warp % KS : 0) * (Kw / 8);
    const int S8 = Kw / 8;
    auto row_of = [&](int u0, int r) -> int {  // weight row r of this warp at step u0, or -1
        if (MIX) {
            const int ch = u0 + warp / KS;
            return ch < NU ? r * ep.D + ch : -1;
        }
        const int n = u0 + (warp / KS) * RPW + r;
        return n < N ? n : -1;
    };
    uint4 pk[RPW][kLmUnroll];
    auto load_w = [&](int u0, int v0) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int n = row_of(u0, r);
            const uint4* wr = reinterpret_cast<const uint4*>(W + (long long)max(n, 0) * K) + j0;
#pragma unroll
            for (int u = 0; u < kLmUnroll; ++u) {
                const int v8 = v0 + 32 * u;
                pk[r][u] = (v8 < S8 && n >= 0) ? __ldg(wr + v8) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // the weight rows of this CTA into L2 (128-byte lines), and the first step's loads,
    // before waiting for the input
    {
        const int lines = K * 2 / 128;  // whole 128-byte lines of a row (a partial last one is left out)
        constexpr int nseg = MIX ? 3 : 1;
        for (int u0 = blockIdx.x * UPC; u0 < NU; u0 += gridDim.x * UPC) {
            const int units = min(UPC, NU - u0);
            for (int sg = 0; sg < nseg; ++sg) {
                const long long r0 = MIX ? (long long)sg * ep.D + u0 : u0;
                const char* base = reinterpret_cast<const char*>(W + r0 * K);
                for (int i = threadIdx.x; i < units * lines; i += kLmThreads)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(base + (long long)i * 128));
            }
        }
    }
    load_w(blockIdx.x * UPC, lane);
    grid_dep_wait();
    grid_dep_launch();
    // mixer epilogue: lane b < B of a channel's first warp finishes (b, channel); its
    // operands for the first step are loaded now, in the shadow of the staging
    long long t = ep.t;
    MixOps mo;
    // (the owner of value (q, b) of the reduce-scatter below: lane b << SHM)
    constexpr int SHM = RPW * BM <= 4 ? 3 : RPW * BM <= 8 ? 2 : RPW * BM <= 16 ? 1 : 0;
    const int mix_b = lane >> SHM;
    const bool mix_lane = MIX && (lane & ((1 << SHM) - 1)) == 0 && mix_b < B && (KS == 1 || warp % KS == 0);
    if (MIX) {
        if (ep.io) t = ep.io->t;
        const int d = blockIdx.x * UPC + warp / KS;
        if (mix_lane && d < NU) mo = lm_mixer_load(mix_b, d, ep.zr, ep.conv, ep.h, ep.L, B, ep.D, t, ep.Y, x);
    }
    {
        // the inputs into the two planes, twelve 16-byte loads a thread in flight at once
        constexpr int SB = 12;
        const float4* x4 = reinterpret_cast<const float4*>(x);
        float4* xs4 = reinterpret_cast<float4*>(xs);
        const int n4 = B * K / 4, K4 = K / 4;
        for (int e0 = threadIdx.x; e0 < n4; e0 += SB * kLmThreads) {
            float4 v[SB];
#pragma unroll
            for (int i = 0; i < SB; ++i)
                if (e0 + i * kLmThreads < n4) v[i] = __ldcg(x4 + e0 + i * kLmThreads);
#pragma unroll
            for (int i = 0; i < SB; ++i) {
                const int e = e0 + i * kLmThreads;
                if (e < n4) {
                    const int b = e / K4, q = e - b * K4;  // q: the 4-group within the row
                    xs4[(q & 1) * (B * K8) + b * K8 + (q >> 1)] = v[i];
                }
            }
        }
    }
    __syncthreads();
    if (ln) {
        // warp b normalises row b: mean, then variance about it (two passes), then
        // bf16((x - mean) / sqrt(var + eps)); row b is the KH values at xs[b KH] and at
        // xs[B KH + b KH], read as float4 (KH = K / 2 is a multiple of 4)
        const int KQ = KH / 4;
        for (int b = warp; b < B; b += nw) {
            float4* p0 = reinterpret_cast<float4*>(xs + b * KH);
            float4* p1 = reinterpret_cast<float4*>(xs + B * KH + b * KH);
            float s = 0.f;
            for (int i = lane; i < KQ; i += 32) {
                const float4 a = p0[i], c = p1[i];
                s += ((a.x + a.y) + (a.z + a.w)) + ((c.x + c.y) + (c.z + c.w));
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const float mean = s / (float)K;
            float v = 0.f;
            for (int i = lane; i < KQ; i += 32) {
                const float4 a = p0[i], c = p1[i];
                v = fmaf(a.x - mean, a.x - mean, v);
                v = fmaf(a.y - mean, a.y - mean, v);
                v = fmaf(a.z - mean, a.z - mean, v);
                v = fmaf(a.w - mean, a.w - mean, v);
                v = fmaf(c.x - mean, c.x - mean, v);
                v = fmaf(c.y - mean, c.y - mean, v);
                v = fmaf(c.z - mean, c.z - mean, v);
                v = fmaf(c.w - mean, c.w - mean, v);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            const float rstd = 1.0f / sqrtf(v / (float)K + kLmLnEps);
            auto nrm = [&](float t) { return __bfloat162float(__float2bfloat16_rn((t - mean) * rstd)); };
            for (int i = lane; i < KQ; i += 32) {
                float4 a = p0[i], c = p1[i];
                a = make_float4(nrm(a.x), nrm(a.y), nrm(a.z), nrm(a.w));
                c = make_float4(nrm(c.x), nrm(c.y), nrm(c.z), nrm(c.w));
                p0[i] = a;
                p1[i] = c;
            }
        }
        __syncthreads();
    }
    const float4* xlo = reinterpret_cast<const float4*>(xs);
    const float4* xhi = xlo + B * K8;
    // greedy choice: each writing warp's running best per batch row (lane 0 owns it)
    __shared__ unsigned long long sbest[nw][BM];
    if (EPI == kLmArgmax && lane == 0)
#pragma unroll
        for (int b = 0; b < BM; ++b) sbest[warp][b] = 0ull;
    bool have = true;  // pk holds the first step's first loads
    for (int u0 = blockIdx.x * UPC; u0 < NU; u0 += gridDim.x * UPC) {
        float acc[RPW][BM];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int b = 0; b < BM; ++b) acc[r][b] = 0.f;
        for (int v0 = lane; v0 < S8; v0 += 32 * kLmUnroll) {
            if (!have) load_w(u0, v0);
            have = false;
#pragma unroll
            for (int u = 0; u < kLmUnroll; ++u) {
                const int v8 = v0 + 32 * u;
                if (v8 < S8) {
                    float w[RPW][8];
#pragma unroll
                    for (int r = 0; r < RPW; ++r) {
                        const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&pk[r][u]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(w2[i]);
                            w[r][2 * i] = f.x;
                            w[r][2 * i + 1] = f.y;
                        }
                    }
#pragma unroll
                    for (int b = 0; b < BM; ++b) {
                        if (b < B) {
                            const float4 x0 = xlo[b * K8 + j0 + v8], x1 = xhi[b * K8 + j0 + v8];
#pragma unroll
                            for (int r = 0; r < RPW; ++r) {
                                float a = acc[r][b];
                                a = fmaf(w[r][0], x0.x, a);
                                a = fmaf(w[r][1], x0.y, a);
                                a = fmaf(w[r][2], x0.z, a);
                                a = fmaf(w[r][3], x0.w, a);
                                a = fmaf(w[r][4], x1.x, a);
                                a = fmaf(w[r][5], x1.y, a);
                                a = fmaf(w[r][6], x1.z, a);
                                a = fmaf(w[r][7], x1.w, a);
                                acc[r][b] = a;
                            }
                        }
                    }
                }
            }
        }
        // sums over the lanes as a reduce-scatter: value v = r BM + b (RPW BM of them,
        // padded to NP, a power of two); at the level of offset 2^k a lane keeps the half
        // of its values that bit k of its id selects and adds its partner's copy of it,
        // until one value is left (v = lane >> SH); the lanes that share it then add
        // across the remaining low bits.  NP - 1 + SH shuffles instead of 5 per value.
        constexpr int NP = RPW * BM <= 4 ? 4 : RPW * BM <= 8 ? 8 : RPW * BM <= 16 ? 16 : 32;
        constexpr int SH = NP == 4 ? 3 : NP == 8 ? 2 : NP == 16 ? 1 : 0;
        float vals[NP];
#pragma unroll
        for (int v = 0; v < NP; ++v) vals[v] = v < RPW * BM ? acc[v / BM][v % BM] : 0.f;
#pragma unroll
        for (int k = 4; k >= SH; --k) {
            const int half = 1 << (k - SH);
            const bool up = (lane >> k) & 1;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = up ? vals[i] : vals[i + half];
                const float keep = up ? vals[i + half] : vals[i];
                vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << k);
            }
        }
        float a = vals[0];
#pragma unroll
        for (int o = (1 << SH) >> 1; o >= 1; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        // the lane with low bits zero owns value v = lane >> SH: row rl = v / BM of the
        // step, batch row bl = v % BM; with KS > 1 the writing warp adds the partial sums
        // of the warps sharing its rows
        const int v = lane >> SH;
        const int rl = v / BM, bl = v % BM;
        const bool pair = (lane & ((1 << SH) - 1)) == 0 && rl < RPW && bl < B;
        if (KS > 1) {
            if (pair) part[warp][rl][bl] = a;
            __syncthreads();
            if (warp % KS == 0 && pair) {
                a = 0.f;
                for (int w = 0; w < KS; ++w) a += part[warp + w][rl][bl];
            }
            __syncthreads();
        }
        if (MIX) {
            // the owner of (q, b) gathers k and v of batch row b from the owners of (k, b), (v, b)
            const float zk = __shfl_sync(0xffffffffu, a, (lane + (BM << SH)) & 31);
            const float zv = __shfl_sync(0xffffffffu, a, (lane + (2 * BM << SH)) & 31);
            const int d = u0 + warp / KS;
            if (mix_lane && d < NU) {
                if (u0 != blockIdx.x * UPC)
                    mo = lm_mixer_load(mix_b, d, ep.zr, ep.conv, ep.h, ep.L, B, ep.D, t, ep.Y, x);
                lm_mixer_finish(mo, a, zk, zv, mix_b, d, ep.zr, ep.L, B, ep.D, t, ep.X, ep.Y, y);
            }
            continue;
        }
        const bool writer = KS == 1 || warp % KS == 0;
        const int n = u0 + (warp / KS) * RPW + rl;
        const bool own = writer && pair && n < N;
        if (own) {
            if (EPI == kLmGelu) a = __bfloat162float(__float2bfloat16_rn(0.5f * a * (1.0f + erff(a * 0.70710678118654752f))));
            if (EPI == kLmAdd) y[(long long)bl * N + n] = __ldcg(ep.res + (long long)bl * N + n) + a;
            else if (EPI != kLmArgmax || y) y[(long long)bl * N + n] = a;
        }
        if (EPI == kLmArgmax) {
            // the step's best per batch row: a maximum over the lanes of equal bl
            unsigned long long k = own ? lm_key(a, n) : 0ull;
#pragma unroll
            for (int o = BM << SH; o < (RPW * BM) << SH; o <<= 1) {
                const unsigned long long q = __shfl_xor_sync(0xffffffffu, k, o);
                k = q > k ? q : k;
            }
            if (writer && rl == 0 && bl < B && k > sbest[warp][bl]) sbest[warp][bl] = k;
        }
    }
    if (EPI == kLmArgmax) {
        // the CTA's best per row, then one atomic per row and CTA
        __syncthreads();
        if (threadIdx.x < B) {
            unsigned long long k = 0ull;
#pragma unroll
            for (int w = 0; w < nw; ++w) k = sbest[w][threadIdx.x] > k ? sbest[w][threadIdx.x] : k;
            if (k) atomicMax(ep.amax + threadIdx.x, k);
        }
    }
}

// The mixer step as a kernel of its own, one thread per (b, d), reading q, k, v from
// z [B][3D] (the traced path launches it separately, so that it can be timed).  With io
// (a replayed per-token graph) the token index comes from the step record.
__global__ void k_lm_mixer(const float* __restrict__ z, float* __restrict__ zr, const float* __restrict__ conv,
                           const float* __restrict__ h, long long L, int B, int D, long long t, float* X,
                           float* Y, const float* u, float* r, const TokIO* io) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    grid_dep_wait();
    grid_dep_launch();
    if (e >= B * D) return;
    const int b = e / D, d = e - b * D;
    const float* zb = z + (long long)b * 3 * D + d;
    const float zq = __ldcg(zb), zk = __ldcg(zb + D), zv = __ldcg(zb + 2 * D);
    if (io) t = io->t;
    const MixOps o = lm_mixer_load(b, d, zr, conv, h, L, B, D, t, Y, u);
    lm_mixer_finish(o, zq, zk, zv, b, d, zr, L, B, D, t, X, Y, r);
}

// next[b] = the greedy choice the LM head folded into amax[b] (largest logit, lowest id
// among equal maxima); also written to out[b] when given, and used as the next input
// token.  With io (a replayed per-token graph) out is the record's choice array at the
// record's token, and with advance this launch closes the token.
__global__ void k_lm_pick(const unsigned long long* __restrict__ amax, int B, int* next, int* out, TokIO* io,
                          int advance) {
    grid_dep_wait();
    grid_dep_launch();
    const int b = threadIdx.x;
    if (b < B) {
        const int idx = lm_key_id(__ldcg(amax + b));
        next[b] = idx;
        if (io) out = io->itok + (io->t - io->tx) * B;
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

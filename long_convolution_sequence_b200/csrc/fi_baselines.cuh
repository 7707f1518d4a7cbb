// fi_baselines.cuh -- the two evaluations of the same stack that the relaxed tiling is
// measured against (Flash Inference summary, "Kern-Algorithmus: Relaxierte
// Polynominterpolation", section 1, and the baselines of "Vergleichsmethoden"):
//
//  * Lazy: each position's mixer output is summed when it is needed,
//    y^l_t = sum_{i<=t} h^l[t-i] a^{l-1}_i, O(t) work at token t;
//  * Eager: as soon as a^{l-1}_t is known, its contribution h^l[t'-t] a^{l-1}_t is added
//    to every later position t' of layer l, O(L-t) work at token t.
//
// Both are the parallel versions the pages compare against: the part of token t that
// does not depend on token t's own chain (Lazy: the sums over the history; Eager: the
// pushes) runs for every layer at once, and only the layer chain of token t
// (y = running sum + h[0] a, a = tanh(y), layer after layer) is sequential.  Lazy: one
// launch per token, one CTA per chain g = (b, c); Eager: the chains, then one launch
// pushing every (chain, layer) pair.  The buffers are the context's halved layout
// act[(M+1)][G][L] (Eager keeps its running sums at the positions after t, as the tiled
// path does, but with every earlier input applied).
//
// The non-parallel versions ("NP" in "Vergleichsmethoden") take no advantage of the
// layers' independence: per token, layer after layer, one launch does that layer's whole
// share (Lazy: its full sum including the newest input, then tanh; Eager: its red cell,
// then the push of its input onto the later positions), so M launches run per token.
#pragma once

namespace fi {

struct BaseArgs {
    float* act;
    const float* h;
    int M, D;
    long long G, L;
    long long t;     // token of this launch
    long long tx;    // token of x[0] / out[0]
    const float* x;  // teacher: [.][G]; closed loop: the start token [G] (first launch) or null
    float* out;      // [.][G] y^M
    int closed;
    int first;       // first token of the call
};

// a^0_t of chain g: the teacher token, or the closed loop's start token on the call's
// first launch (otherwise the previous launch stored it)
__device__ __forceinline__ float base_input(const BaseArgs& a, long long g) {
    float* p = a.act + g * a.L + a.t;
    if (!a.closed) *p = a.x[(a.t - a.tx) * a.G + g];
    else if (a.first && a.x) *p = a.x[g];
    return *p;
}

// the red cells of token t, layers in order, from the running sums s[l-1] (thread 0);
// leaves a^0..a^M of token t in av[0..M] when av is given
__device__ __forceinline__ void base_chain(const BaseArgs& a, long long g, int c, float a0, const float* s,
                                           float* av) {
    const long long L = a.L, t = a.t;
    float v = a0, y = 0.f;
    if (av) av[0] = v;
    for (int l = 1; l <= a.M; ++l) {
        const float h0 = a.h[((long long)(l - 1) * a.D + c) * L];
        y = fmaf(h0, v, s[l - 1]);
        v = act_tanh(y);
        a.act[((long long)l * a.G + g) * L + t] = v;
        if (av) av[l] = v;
    }
    a.out[(t - a.tx) * a.G + g] = y;
    if (a.closed && t + 1 < L) a.act[g * L + t + 1] = v;
}

// Lazy: warp w sums the history of layers w+1, w+1+nw, ...; thread 0 runs the chain.
__global__ void k_lazy_token(BaseArgs a) {
    extern __shared__ float bsm[];  // [M] history sums
    const long long g = blockIdx.x;
    const int c = (int)(g % a.D);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const long long t = a.t, L = a.L;
    float a0 = 0.f;
    if (threadIdx.x == 0) a0 = base_input(a, g);  // position t: read by no warp below
    for (int l = 1 + warp; l <= a.M; l += nw) {
        const float* in = a.act + ((long long)(l - 1) * a.G + g) * L;
        const float* hl = a.h + ((long long)(l - 1) * a.D + c) * L + t;  // hl[-i] = h^l[t-i]
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        long long i = lane;
        for (; i + 96 < t; i += 128) {
            s0 = fmaf(in[i], hl[-i], s0);
            s1 = fmaf(in[i + 32], hl[-i - 32], s1);
            s2 = fmaf(in[i + 64], hl[-i - 64], s2);
            s3 = fmaf(in[i + 96], hl[-i - 96], s3);
        }
        for (; i < t; i += 32) s0 = fmaf(in[i], hl[-i], s0);
        float s = (s0 + s1) + (s2 + s3);
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) bsm[l - 1] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) base_chain(a, g, c, a0, bsm, nullptr);
}

// Eager, in two launches per token: the red cells of token t, layer after layer, one
// thread per chain, from the running sums at position t (every earlier input pushed)...
__global__ void k_eager_chain(BaseArgs a) {
    const long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (g >= a.G) return;
    const int c = (int)(g % a.D);
    const long long t = a.t, L = a.L;
    float v = base_input(a, g), y = 0.f;
    for (int l = 1; l <= a.M; ++l) {
        float* slot = a.act + ((long long)l * a.G + g) * L + t;  // running sum of y^l_t
        y = fmaf(a.h[((long long)(l - 1) * a.D + c) * L], v, *slot);
        v = act_tanh(y);
        *slot = v;
    }
    a.out[(t - a.tx) * a.G + g] = y;
    if (a.closed && t + 1 < L) a.act[g * L + t + 1] = v;
}

// ...then every layer's push at once: CTA (g, l) adds h^l[d] a^{l-1}_t onto position
// t + d of layer l, d >= 1.
__global__ void k_eager_push(BaseArgs a) {
    const long long g = blockIdx.x;
    const int l = 1 + (int)blockIdx.y;
    const int c = (int)(g % a.D);
    const long long t = a.t, L = a.L;
    const float v = a.act[((long long)(l - 1) * a.G + g) * L + t];  // a^{l-1}_t, final
    float* acc = a.act + ((long long)l * a.G + g) * L + t;          // acc[d] = position t + d
    const float* hl = a.h + ((long long)(l - 1) * a.D + c) * L;     // hl[d] = h^l[d]
    for (long long d = 1 + threadIdx.x; d < L - t; d += blockDim.x) acc[d] = fmaf(hl[d], v, acc[d]);
}

// Lazy, non-parallel: layer l of token t alone, y^l_t = sum_{i<=t} h^l[t-i] a^{l-1}_i over
// the whole history (a^{l-1}_t was finished by the previous launch), then a^l_t = tanh(y).
__global__ void k_lazy_layer(BaseArgs a, int l) {
    extern __shared__ float bsm[];  // [warps] partial sums
    const long long g = blockIdx.x;
    const int c = (int)(g % a.D);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const long long t = a.t, L = a.L;
    if (l == 1) {
        if (threadIdx.x == 0) base_input(a, g);
        __syncthreads();
    }
    const float* in = a.act + ((long long)(l - 1) * a.G + g) * L;
    const float* hl = a.h + ((long long)(l - 1) * a.D + c) * L + t;  // hl[-i] = h^l[t-i]
    const long long nt = blockDim.x;
    float s0 = 0.f, s1 = 0.f;
    long long i = threadIdx.x;
    for (; i + nt <= t; i += 2 * nt) {
        s0 = fmaf(in[i], hl[-i], s0);
        s1 = fmaf(in[i + nt], hl[-i - nt], s1);
    }
    for (; i <= t; i += nt) s0 = fmaf(in[i], hl[-i], s0);
    float s = s0 + s1;
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) bsm[warp] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float y = 0.f;
        for (int w = 0; w < nw; ++w) y += bsm[w];
        const float v = act_tanh(y);
        a.act[((long long)l * a.G + g) * L + t] = v;
        if (l == a.M) {
            a.out[(t - a.tx) * a.G + g] = y;
            if (a.closed && t + 1 < L) a.act[g * L + t + 1] = v;
        }
    }
}

// Eager, non-parallel: layer l of token t alone: its red cell from the running sum at t
// (every earlier input already pushed), then the push of its input a^{l-1}_t onto the
// later positions of layer l.
__global__ void k_eager_layer(BaseArgs a, int l) {
    __shared__ float a_in;
    const long long g = blockIdx.x;
    const int c = (int)(g % a.D);
    const long long t = a.t, L = a.L;
    float* acc = a.act + ((long long)l * a.G + g) * L + t;  // acc[d] = position t + d of layer l
    const float* hl = a.h + ((long long)(l - 1) * a.D + c) * L;  // hl[d] = h^l[d]
    if (threadIdx.x == 0) {
        const float v0 = l == 1 ? base_input(a, g) : a.act[((long long)(l - 1) * a.G + g) * L + t];
        const float y = fmaf(hl[0], v0, acc[0]);
        const float v = act_tanh(y);
        acc[0] = v;
        if (l == a.M) {
            a.out[(t - a.tx) * a.G + g] = y;
            if (a.closed && t + 1 < L) a.act[g * L + t + 1] = v;
        }
        a_in = v0;
    }
    __syncthreads();
    const float v0 = a_in;
    for (long long d = 1 + threadIdx.x; d < L - t; d += blockDim.x) acc[d] = fmaf(hl[d], v0, acc[d]);
}

}  // namespace fi

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
// (y = running sum + h[0] a, a = tanh(y), layer after layer) is sequential.  One launch
// per token, one CTA per chain g = (b, c); the buffers are the context's halved layout
// act[(M+1)][G][L] (Eager keeps its running sums at the positions after t, as the tiled
// path does, but with every earlier input applied).
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

// Eager: thread 0 finishes token t from the running sums at position t, then every
// thread pushes token t's activations onto the later positions of every layer.
__global__ void k_eager_token(BaseArgs a) {
    extern __shared__ float bsm[];  // [M] running sums, then [M + 1] activations
    float* s = bsm;
    float* av = bsm + a.M;
    const long long g = blockIdx.x;
    const int c = (int)(g % a.D);
    const long long t = a.t, L = a.L;
    if (threadIdx.x == 0) {
        const float a0 = base_input(a, g);
        for (int l = 1; l <= a.M; ++l) s[l - 1] = a.act[((long long)l * a.G + g) * L + t];
        base_chain(a, g, c, a0, s, av);
    }
    __syncthreads();
    for (int l = 1; l <= a.M; ++l) {
        const float v = av[l - 1];
        float* acc = a.act + ((long long)l * a.G + g) * L + t;  // acc[d] = position t + d
        const float* hl = a.h + ((long long)(l - 1) * a.D + c) * L;  // hl[d] = h^l[d]
        for (long long d = 1 + threadIdx.x; d < L - t; d += blockDim.x) acc[d] = fmaf(hl[d], v, acc[d]);
    }
}

}  // namespace fi

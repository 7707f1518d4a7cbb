// fi_cluster.cuh -- FFT convolution of gray blocks too large for one SM (sm_100a
// thread-block clusters, distributed shared memory).
//
// A block of edge U = N = NC * N2 (N2 = 2^LOGN2 points per CTA) is one cluster of NC
// CTAs; CTA rank k1 of the cluster owns the frequencies k = k1 + NC k2, k2 < N2.
// With n = n1 N2 + n2 and k = k1 + NC k2 the N-point DFT factors as
//   Z[k1 + NC k2] = sum_{n2} W_N2^{n2 k2} W_N^{n2 k1} sum_{n1} z[n1 N2 + n2] W_NC^{n1 k1},
// so each CTA forms the inner radix-NC sums for its k1 straight from global memory
// (the packed block is zero for n1 >= NC/2) and finishes with a local N2-point FFT in
// its shared memory (the passes of fi_fft.cuh).  The spectral multiply pairs Z[k] with
// Z[N-k], which CTA NC-k1 holds (CTA 0 and CTA NC/2 pair with themselves); it reads
// the partner's shared memory.  The inverse (a forward DFT of the conjugated product)
// runs the other way round: a local N2-point FFT over k2 per CTA, twiddles
// W_N^{k1 n2}, then a radix-NC DFT over the CTA ranks that gathers one value from
// every CTA's shared memory, of which only the outputs n1 >= NC/2 (real samples
// [U, 2U)) are formed and added onto the block's outputs.
//
// Spectra of these sizes are stored per (layer, channel) in CTA order:
// Hc[k1 N2 + k2] = H[k1 + NC k2] for k < N, then Hc[N] = H[N], stride N + 2.
#pragma once
#include <cooperative_groups.h>
#include <cuda_runtime.h>

namespace fi {

template <int LOGNC, int LOGN2>
struct ClusterTile {
    static constexpr int NC = 1 << LOGNC;
    static constexpr int N2 = 1 << LOGN2;
    static constexpr int LOGN = LOGNC + LOGN2;
    static constexpr int N = 1 << LOGN;
    static constexpr int NP = LOGN2 / 4;                   // radix-16 passes of the local FFT
    static constexpr int R0 = 1 << (LOGN2 - 4 * NP);       // extra local radix (1 or 2)
    static constexpr int T = N2 / 16;                      // threads per CTA
    static constexpr int SME = N2 + N2 / 16;
    static constexpr int HST = 2 * N2 + 2;                 // staged spectrum: own row, partner row, H[N]
    static constexpr size_t smem = (size_t)(SME + HST) * sizeof(float2);
    static constexpr int MINB = T <= 256 ? 2 : 1;
};

// Forward half of a cluster transform, shared by the block kernel and the spectrum
// kernel: on return this CTA's Z[k1 + NC k2], k2 = t + m N2/16, are in v[0][omap(m)]
// and in X (natural order over k2).  HALF: the input is zero for n1 >= NC/2.
template <int LOGNC, int LOGN2, int TWLOG, bool HALF>
__device__ __forceinline__ void cluster_forward(const float2* __restrict__ z, float2* X, float2 (*v)[16], int k1,
                                                int t, const float2* __restrict__ tw) {
    using G = ClusterTile<LOGNC, LOGN2>;
    constexpr int NC = G::NC, N2 = G::N2, LOGN = G::LOGN, T = G::T, R0 = G::R0, NP = G::NP;
    constexpr int NIN = HALF ? NC / 2 : NC;
    float2 wn1[NIN];  // W_NC^{n1 k1}
#pragma unroll
    for (int n1 = 0; n1 < NIN; ++n1) wn1[n1] = fft::tw_at<TWLOG>(tw, ((n1 * k1) & (NC - 1)) << (TWLOG - LOGNC));
    // y[n2] = W_N^{n2 k1} sum_{n1} z[n1 N2 + n2] W_NC^{n1 k1}, n2 = b + r NB: the twiddle
    // is W_N^{b k1} (one table entry per butterfly) times W_N^{r NB k1} (the same for
    // every thread of the CTA)
    auto y_of = [&](const float2 (&zz)[NIN], int r, int NB, float2 wb) {
        float2 y = zz[0];
#pragma unroll
        for (int n1 = 1; n1 < NIN; ++n1)
            y = make_float2(y.x + (zz[n1].x * wn1[n1].x - zz[n1].y * wn1[n1].y),
                            y.y + (zz[n1].x * wn1[n1].y + zz[n1].y * wn1[n1].x));
        return fft::cm(y, fft::cm(wb, fft::tw_at<TWLOG>(tw, (r * NB * k1) << (TWLOG - LOGN))));
    };
    auto y_at = [&](int b, int r, int NB, float2 wb) {
        float2 zz[NIN];
#pragma unroll
        for (int n1 = 0; n1 < NIN; ++n1) zz[n1] = __ldg(z + n1 * N2 + b + r * NB);
        return y_of(zz, r, NB, wb);
    };
    if constexpr (R0 > 1) {
        // radix-R0 first pass (Ns = 1): butterfly b reads y[b + r N2/R0]
        constexpr int BPT = 16 / R0, NB = N2 / R0;
#pragma unroll
        for (int u = 0; u < BPT; ++u) {
            const int b = t + u * T;
            const float2 wb = fft::tw_at<TWLOG>(tw, (b * k1) << (TWLOG - LOGN));
            float2 w[R0];
#pragma unroll
            for (int r = 0; r < R0; ++r) w[r] = y_at(b, r, NB, wb);
            fft::dft<R0>(w);
#pragma unroll
            for (int m = 0; m < R0; ++m) X[fft::pad(b * R0 + m)] = w[fft::omap<R0>(m)];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < NP; ++j) fft::pass<LOGN2, 16, 1, TWLOG>(X, v, t, T, (LOGN2 - 4 * NP) + 4 * j, tw);
    } else {
        constexpr int NB = N2 / 16;
        const float2 wb = fft::tw_at<TWLOG>(tw, (t * k1) << (TWLOG - LOGN));
        // the inputs of RB outputs are loaded before any is combined: the loads of a
        // batch are in flight together (the sums are bound by global-memory latency)
        constexpr int RB = NIN >= 32 ? 1 : (32 / NIN > 16 ? 16 : 32 / NIN);
#pragma unroll
        for (int r0 = 0; r0 < 16; r0 += RB) {
            float2 zz[RB][NIN];
#pragma unroll
            for (int i = 0; i < RB; ++i)
#pragma unroll
                for (int n1 = 0; n1 < NIN; ++n1) zz[i][n1] = __ldg(z + n1 * N2 + t + (r0 + i) * NB);
#pragma unroll
            for (int i = 0; i < RB; ++i) v[0][r0 + i] = y_of(zz[i], r0 + i, NB, wb);
        }
        fft::dft<16>(v[0]);
#pragma unroll
        for (int m = 0; m < 16; ++m) X[fft::pad(t * 16 + m)] = v[0][fft::omap<16>(m)];
        __syncthreads();
#pragma unroll
        for (int j = 1; j < NP; ++j) fft::pass<LOGN2, 16, 1, TWLOG>(X, v, t, T, 4 * j, tw);
    }
}

// Partner of this CTA's element k = k1 + NC k2 under k -> N - k (mod N): CTA rank and
// local index.
template <int NC, int N2>
__device__ __forceinline__ void cluster_partner(int k1, int k2, int* pk1, int* pk2) {
    if (k1 == 0) {
        *pk1 = 0;
        *pk2 = (N2 - k2) & (N2 - 1);
    } else {
        *pk1 = NC - k1;
        *pk2 = N2 - 1 - k2;
    }
}

template <int LOGNC, int LOGN2, int TWLOG>
__global__ void __launch_bounds__(ClusterTile<LOGNC, LOGN2>::T, ClusterTile<LOGNC, LOGN2>::MINB)
    k_block_fft_cluster(TileArgs a0) {
    const TileArgs a = with_step(a0);
    namespace cg = cooperative_groups;
    using G = ClusterTile<LOGNC, LOGN2>;
    constexpr int NC = G::NC, N2 = G::N2, N = G::N, LOGN = G::LOGN, T = G::T, R0 = G::R0, NP = G::NP;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) float2 csm[];
    float2* X = csm;
    const int k1 = (int)cluster.block_rank();
    const long long item = blockIdx.x / NC;
    const int t = threadIdx.x;
    const TilePtrs p = tile_ptrs(a, item);
    float2 v[1][16];
    const int pk1 = k1 == 0 ? 0 : NC - k1;

    // the two spectrum rows this CTA's multiply reads stream into shared memory
    // during the forward transform: Hs[k2] = H[k1 + NC k2], Hs[N2 + j] = row pk1, Hs[2 N2] = H[N]
    float2* Hs = csm + G::SME;
    {
        const float2* Hown = p.spec + (long long)k1 * N2;
        const float2* Hpar = p.spec + (long long)pk1 * N2;
        for (int c = t; c < N2 / 2; c += T) {
            cp_async16(Hs + 2 * c, Hown + 2 * c);
            cp_async16(Hs + N2 + 2 * c, Hpar + 2 * c);
        }
        if (t == 0) Hs[2 * N2] = __ldg(p.spec + N);
        cp_async_commit();
    }

    grid_dep_wait();  // the block's inputs and old outputs come from the previous launches
    cluster_forward<LOGNC, LOGN2, TWLOG, true>(reinterpret_cast<const float2*>(p.in), X, v, k1, t, a.tw);
    cp_async_wait_all();
    cluster.sync();  // every CTA's Z is in its shared memory, the staged spectrum is complete

    // ---- spectral multiply (see fi_fft.cuh): Q[k] = conj(Z[k]) (S + sin D) + Z[N-k] (i cos D)
    float2 q[16];
    {
        constexpr int NB = N2 / 16;
        const float2* Xp = cluster.map_shared_rank(X, pk1);
        const float2 wb = fft::tw_at<TWLOG>(a.tw, (k1 + NC * t) << (TWLOG - LOGN - 1));  // W_{2N}^{k1 + NC t}
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int k2 = t + m * NB;
            int qk1, qk2;
            cluster_partner<NC, N2>(k1, k2, &qk1, &qk2);
            const float2 Zk = v[0][fft::omap<16>(m)];
            const float2 Zn = Xp[fft::pad(qk2)];
            const float2 Hk = Hs[k2];
            const float2 Hn = (k1 == 0 && k2 == 0) ? Hs[2 * N2] : Hs[N2 + qk2];
            const float2 w = fft::cm(wb, fft::w32(m));  // W_{2N}^{k}, k = k1 + NC k2
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
    // The inverse runs in the spectrum area, free once this CTA's threads have read it:
    // X keeps this CTA's Z, which the partner CTA may still be reading, so no cluster
    // barrier is needed here.
    __syncthreads();
    grid_dep_launch();
    float2* X2 = Hs;
    // this CTA's old outputs (runs [k1 PER, (k1+1) PER) + N2 i, i < NC/2) stream into
    // the rest of the spectrum area during the inverse transform
    constexpr int PER = N2 / NC;  // output n2 values of this CTA
    static_assert(PER % T == 0, "outputs per CTA must be a multiple of its threads");
    static_assert(G::SME + N2 / 2 <= G::HST, "inverse area and old outputs fit the spectrum area");
    float2* Os = Hs + G::SME;
    if (!a.overwrite) {
        const float2* o2c = reinterpret_cast<const float2*>(p.out);
#pragma unroll
        for (int i = 0; i < NC / 2; ++i)
            for (int c = t; c < PER / 2; c += T) cp_async16(Os + i * PER + 2 * c, o2c + k1 * PER + N2 * i + 2 * c);
    }
    cp_async_commit();

    // ---- inverse, local N2-point DFT over k2: first pass in registers (Ns = 1)
    fft::dft<16>(q);
#pragma unroll
    for (int m = 0; m < 16; ++m) X2[fft::pad(t * 16 + m)] = q[fft::omap<16>(m)];
    __syncthreads();
    // remaining passes; the last one multiplies its outputs n2 by W_N^{k1 n2} and
    // leaves them in natural order
    {
        constexpr int NLAST = R0 > 1 ? NP : NP - 1;  // radix-16 passes after the first
#pragma unroll
        for (int j = 1; j < NLAST; ++j) fft::pass<LOGN2, 16, 1, TWLOG>(X2, v, t, T, 4 * j, a.tw);
        if constexpr (R0 > 1) {
            // radix-R0 at Ns = N2/R0: butterfly b (< N2/R0) reads X[b + r N2/R0]
            constexpr int BPT = 16 / R0, NB = N2 / R0;
            float2 w[BPT][R0];
#pragma unroll
            for (int u = 0; u < BPT; ++u) {
                const int b = t + u * T;
#pragma unroll
                for (int r = 0; r < R0; ++r) w[u][r] = X2[fft::pad(b + r * NB)];
                fft::apply_twiddles<R0, TWLOG>(w[u], a.tw, LOGN2, b);
                fft::dft<R0>(w[u]);
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < BPT; ++u) {
                const int b = t + u * T;
                const float2 wb = fft::tw_at<TWLOG>(a.tw, (b * k1) << (TWLOG - LOGN));
#pragma unroll
                for (int m = 0; m < R0; ++m) {
                    const float2 wm = fft::cm(wb, fft::tw_at<TWLOG>(a.tw, (m * NB * k1) << (TWLOG - LOGN)));
                    X2[fft::pad(b + m * NB)] = fft::cm(w[u][fft::omap<R0>(m)], wm);
                }
            }
        } else {
            // radix-16 at Ns = N2/16: butterfly t, outputs t + m N2/16
            constexpr int NB = N2 / 16;
            float2 w[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) w[r] = X2[fft::pad(t + r * NB)];
            fft::apply_twiddles<16, TWLOG>(w, a.tw, LOGN2, t);
            fft::dft<16>(w);
            __syncthreads();
            const float2 wb = fft::tw_at<TWLOG>(a.tw, (t * k1) << (TWLOG - LOGN));
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float2 wm = fft::cm(wb, fft::tw_at<TWLOG>(a.tw, (m * NB * k1) << (TWLOG - LOGN)));
                X2[fft::pad(t + m * NB)] = fft::cm(w[fft::omap<16>(m)], wm);
            }
        }
    }
    cp_async_wait_all();
    cluster.sync();  // every CTA's twiddled local result is in its shared memory

    // ---- radix-NC over the CTA ranks; this CTA forms the outputs n2 in its share,
    // all remote loads first
    {
        constexpr int NPT = PER / T;
        float2* o2 = reinterpret_cast<float2*>(p.out);
        float2 g[NPT][NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const float2* Xc = cluster.map_shared_rank(X2, c);
#pragma unroll
            for (int u = 0; u < NPT; ++u) g[u][c] = Xc[fft::pad(k1 * PER + t + u * T)];
        }

        float dep = 0.f;
#pragma unroll
        for (int u = 0; u < NPT; ++u) {
            fft::dft<NC>(g[u]);
            dep += g[u][0].x;  // every DFT output depends on every value loaded for it
        }
        // every value read from the other CTAs' shared memory has arrived (the arrival
        // takes an operand computed from all of them), so this CTA no longer reads them
        // and a relaxed arrival suffices; the wait, before exit, overlaps the stores
        asm volatile("barrier.cluster.arrive.relaxed.aligned; // %0\n" ::"f"(dep) : "memory");
#pragma unroll
        for (int u = 0; u < NPT; ++u) {
            const int j = t + u * T;
#pragma unroll
            for (int n1 = NC / 2; n1 < NC; ++n1) {
                const float2 F = g[u][fft::omap<NC>(n1)];
                const int i = n1 - NC / 2;
                const float2 y = make_float2(F.x, -F.y);
                float2* o = o2 + k1 * PER + j + N2 * i;
                if (a.overwrite) *o = y;
                else {
                    const float2 old = Os[i * PER + j];
                    *o = make_float2(old.x + y.x, old.y + y.y);
                }
            }
        }
    }
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");  // no CTA leaves while another reads it
    if (a.io && a.advance) tok_advance_if_last(a.io);
}

// Spectra of the cluster sizes: H = scale * DFT_{2N}(taps[0, 2N)), k = 0..N, in CTA
// order (see above), one cluster per (layer, channel) item; taps packed as complex
// pairs (the full 2N samples, no zero half).
template <int LOGNC, int LOGN2, int TWLOG>
__global__ void __launch_bounds__(ClusterTile<LOGNC, LOGN2>::T, ClusterTile<LOGNC, LOGN2>::MINB)
    k_spectra_cluster(const float* __restrict__ taps, long long ld, float2* spec, long long hstride,
                      const float2* __restrict__ tw, float scale) {
    namespace cg = cooperative_groups;
    using G = ClusterTile<LOGNC, LOGN2>;
    constexpr int NC = G::NC, N2 = G::N2, N = G::N, LOGN = G::LOGN;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) float2 csm[];
    float2* X = csm;
    const int k1 = (int)cluster.block_rank();
    const long long item = blockIdx.x / NC;
    const int t = threadIdx.x;
    float2 v[1][16];
    cluster_forward<LOGNC, LOGN2, TWLOG, false>(reinterpret_cast<const float2*>(taps + item * ld), X, v, k1, t, tw);
    cluster.sync();
    constexpr int NB = N2 / 16;
    const int pk1 = k1 == 0 ? 0 : NC - k1;
    const float2* Xp = cluster.map_shared_rank(X, pk1);
    float2* H = spec + item * hstride;
    const float2 wb = fft::tw_at<TWLOG>(tw, (k1 + NC * t) << (TWLOG - LOGN - 1));
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const int k2 = t + m * NB;
        int qk1, qk2;
        cluster_partner<NC, N2>(k1, k2, &qk1, &qk2);
        const float2 Zk = v[0][fft::omap<16>(m)];
        const float2 Zn = Xp[fft::pad(qk2)];
        const float2 w = fft::cm(wb, fft::w32(m));
        // 2X[k] = A - i w B,  2X[N-k] = conj(A + i w B),  A = Zk + conj Zn, B = Zk - conj Zn
        const float2 A = make_float2(Zk.x + Zn.x, Zk.y - Zn.y);
        const float2 Bv = make_float2(Zk.x - Zn.x, Zk.y + Zn.y);
        const float2 P = fft::mul_pi(fft::cm(w, Bv));
        const float h = 0.5f * scale;
        H[k1 * N2 + k2] = make_float2(h * (A.x - P.x), h * (A.y - P.y));
        if (k1 == 0 && k2 == 0) H[N] = make_float2(h * (A.x + P.x), -h * (A.y + P.y));
    }
    cluster.sync();
}

}  // namespace fi

// fi_api.cu -- host side of the C-ABI (include/fi.h): context lifetime, the
// lowbit schedule, the Hybrid tau table, launch sequencing for the window and
// per-token paths, CUDA-graph capture and replay, host/device staging.
//
// Passages followed (web summary of arXiv 2410.12982, "Flash Inference: Near Linear
// Time Inference for Long Convolution Sequence Models and Beyond"):
//   section "Kachelung-Strategie (Algorithmus 1)"   -- which block follows which token
//   section "LCSM-Inferenz-Algorithmus (Algorithmus 2)" -- red cells, blocks, sampler
//   section "Schicht-uebergreifende Parallelisierung (Algorithmus 3)" -- one launch
//           carries the blocks of every layer
//   section "Implementierungsdetails" -- CUDA graphs, FFT precompute, Hybrid tau
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "fi.h"
#include "fi_kernels.cuh"
#include "fi_lm.cuh"
#include "fi_dd.cuh"

using namespace fi;

// Fixed device scratch of fi_tau_fft_noalloc (8 MiB, in every device that loads the
// library, until the process exits).  Host code must not use the symbol as a device
// address: the address comes from cudaGetSymbolAddress at set-up.
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

thread_local char g_err[1024] = "";

int set_err(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

#define CK(call)                                                                               \
    do {                                                                                       \
        cudaError_t e_ = (call);                                                               \
        if (e_ != cudaSuccess)                                                                 \
            return set_err(e_ == cudaErrorMemoryAllocation ? FI_ENOMEM : FI_ECUDA,             \
                           "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__,   \
                           __LINE__);                                                          \
    } while (0)

constexpr unsigned kMagic = 0xF1C7A5E5u;
constexpr int kTwLog = 18;          // twiddle table e^{-2 pi i k / 2^18}
constexpr int kFusedQLimit = 14;    // largest block size whose FFT one CTA can hold (U = 16384)
constexpr int kFftQMax = 17;        // largest block size served by FFT (clusters of CTAs beyond 2^12)
constexpr int kFftQMin = 3;         // smallest block size served by FFT (U = 8)
constexpr int kDirectQMax = 12;     // largest block size served by the direct kernel
constexpr int kFuseQMax = 4;        // per-token path: blocks up to U = 16 run inside the step kernel
constexpr int kStepNT = 128;
constexpr int kDirectNT = 128;
constexpr size_t kSmemMax = 227 * 1024;
constexpr int kGraphCache = 8;

struct GraphKey {
    int path, mode;  // mode: 0 teacher, 1 closed
    long long t0, steps;
    const void* x;
    const void* y;
    bool operator<(const GraphKey& o) const {
        return std::tie(path, mode, t0, steps, x, y) < std::tie(o.path, o.mode, o.t0, o.steps, o.x, o.y);
    }
};

struct TraceRec {
    int cls;
    int q;  // block size 2^q of block launches, -1 otherwise
    cudaEvent_t a, b;
};

struct GraphEntry {
    cudaGraphExec_t exec = nullptr;
    std::vector<TraceRec> trace;
    long long launches = 0;
};

}  // namespace

struct fi_ctx {
    unsigned magic = kMagic;
    int M = 0, B = 0, D = 0, L = 0, P = 0;
    long long G = 0;
    int dev = 0, nsm = 0;
    cudaStream_t stream = nullptr;   // user stream (nullptr = legacy default)
    cudaStream_t cap = nullptr;      // private stream used to capture graphs
    float* act = nullptr;            // [(M+1)][G][L]
    float* yout = nullptr;           // language model: the mixers' outputs [M][G][L] (blocks read act[l], add onto yout[l])
    float* h = nullptr;              // [M][D][L]
    float2* tw = nullptr;            // [2^kTwLog]
    float2* spec[32] = {};           // per block size 2^q
    long long spec_stride[32] = {};  // complex entries per (layer, channel)
    int tau[32] = {}, tau_user[32] = {};
    float tau_us[32][2] = {};
    int W = 0, kch = 0, win_ncta = 0;
    size_t win_smem = 0;
    int path = FI_PATH_WINDOW, graphs = 1;
    int pdl = 1;  // window-path launches overlap their start with the predecessor's end
    int layer_split = 0;  // ablation (FI_LAYER_SPLIT=1): one block launch per layer instead of one for all
    long long t = 0;
    float* sx = nullptr;  // staging for host inputs
    size_t sx_n = 0;
    float* sy = nullptr;  // staging for host outputs
    size_t sy_n = 0;
    float* pre = nullptr;  // prompt-prefill scratch, grown on demand
    size_t pre_n = 0;
    float2* pre_spec = nullptr;  // prefill: spectra of the shifted taps [M][D][U+2] of one prompt size
    int pre_spec_q = -1;         // its block size 2^q (-1: none)
    size_t pre_spec_n = 0;
    std::map<GraphKey, GraphEntry> gcache;
    std::vector<GraphKey> gorder;
    // per-token path: one graph per (mode, block size 2^q released after the token;
    // index 32 = the last token, which releases none), replayed per token
    TokIO* tio = nullptr;
    cudaGraphExec_t tokg[2][33] = {};
    long long tokg_nodes[2][33] = {};
    size_t bytes = 0;
    // tracing: per-launch event pairs grouped by kernel class
    int trace_on = 0;
    std::vector<TraceRec>* rec = nullptr;        // list being filled by enqueue
    std::vector<TraceRec> eager_trace;           // list of the last eager run
    const std::vector<TraceRec>* last_trace = nullptr;
    std::vector<cudaEvent_t> event_pool;
    size_t event_next = 0;
    long long launches = 0;                      // kernels launched by runs so far
    long long enq_launches = 0;                  // kernels enqueued by the current enqueue()
};

namespace {

bool is_device_ptr(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

int ctz64(long long v) {
    int q = 0;
    while (!((v >> q) & 1)) ++q;
    return q;
}

// Live contexts: a pointer that was never returned by fi_create, or was destroyed,
// is rejected without being dereferenced.
std::mutex g_live_mu;
std::set<const fi_ctx*> g_live;

int check_ctx(const fi_ctx* c) {
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        if (!c || !g_live.count(c)) return set_err(FI_ESTATE, "null or destroyed context");
    }
    if (c->magic != kMagic) return set_err(FI_ESTATE, "null or destroyed context");
    return FI_OK;
}

cudaEvent_t pool_event(fi_ctx* c) {
    if (c->event_next == c->event_pool.size()) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) {
            cudaGetLastError();  // out of events: the launch goes untraced, no error is left behind
            return nullptr;
        }
        c->event_pool.push_back(e);
    }
    return c->event_pool[c->event_next++];
}

// Record an event on st: as an external event node while st is being captured into a
// graph (so that the event is recorded at every replay), as a plain record otherwise.
void trace_record(cudaEvent_t e, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) cudaGetLastError();
    if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    else cudaEventRecord(e, st);
}

// Bracket one launch with events when tracing (also inside graph capture).
struct LaunchScope {
    fi_ctx* c;
    cudaStream_t st;
    TraceRec r;
    bool on;
    LaunchScope(fi_ctx* c_, int cls, cudaStream_t st_, int q = -1)
        : c(c_), st(st_), on(c_->trace_on && c_->rec) {
        c->enq_launches++;
        if (on) {
            r.cls = cls;
            r.q = q;
            r.a = pool_event(c);
            r.b = pool_event(c);
            on = r.a && r.b;
            if (on) trace_record(r.a, st);
        }
    }
    ~LaunchScope() {
        if (on) {
            trace_record(r.b, st);
            c->rec->push_back(r);
        }
    }
};

template <typename T>
int dev_alloc(fi_ctx* c, T** p, size_t count) {
    const char* f = getenv("FI_FAULT");
    if (f && strstr(f, "alloc")) return set_err(FI_ENOMEM, "injected allocation failure (FI_FAULT=alloc)");
    cudaError_t e = cudaMalloc((void**)p, count * sizeof(T));
    if (e != cudaSuccess) {
        *p = nullptr;
        cudaGetLastError();
        return set_err(e == cudaErrorMemoryAllocation ? FI_ENOMEM : FI_ECUDA,
                       "cudaMalloc(%zu bytes) failed: %s", count * sizeof(T), cudaGetErrorString(e));
    }
    c->bytes += count * sizeof(T);
    return FI_OK;
}

size_t win_smem_bytes(int W, int M, int B, int kch) {
    // slot, tap and shifted-copy rows plus the leading zero row, each W + kWinPad floats,
    // and the speculative chain values of two tokens (M x 32 float2 each)
    return (size_t)((M + 1) * kch * B + M * kch + M * kch * B + 1) * (W + kWinPad) * sizeof(float) +
           (size_t)2 * M * 32 * sizeof(float2);
}

// chain registers of the window kernel are unrolled up to MAXM layers (18: exact)
int win_maxm(int M) { return M <= 8 ? 8 : (M == 18 ? 18 : (M <= 20 ? 20 : (M <= 40 ? 40 : 0))); }

// ---------------------------------------------------------------- kernel launchers
// Launches of the generation path may overlap their start with the predecessor's
// end (programmatic dependent launch): the kernels read nothing the predecessor
// writes before griddepcontrol.wait.
void set_pdl(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* at, int pdl) {
    if (!pdl) return;
    at[cfg->numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[cfg->numAttrs].val.programmaticStreamSerializationAllowed = 1;
    cfg->attrs = at;
    cfg->numAttrs += 1;
}

template <int LOGN>
int launch_fft_tile_t(const TileArgs& a, cudaStream_t st, int pdl) {
    using G = FftTile<LOGN>;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)((a.count + G::TPC - 1) / G::TPC));
    cfg.blockDim = dim3(G::NT);
    cfg.dynamicSmemBytes = G::smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    set_pdl(&cfg, at, pdl);
    CK(cudaLaunchKernelEx(&cfg, k_block_fft<LOGN, kTwLog>, a));
    return FI_OK;
}

int launch_fft_tile(int logn, const TileArgs& a, cudaStream_t st, int pdl) {
    switch (logn) {
        case 3: return launch_fft_tile_t<3>(a, st, pdl);
        case 4: return launch_fft_tile_t<4>(a, st, pdl);
        case 5: return launch_fft_tile_t<5>(a, st, pdl);
        case 6: return launch_fft_tile_t<6>(a, st, pdl);
        case 7: return launch_fft_tile_t<7>(a, st, pdl);
        case 8: return launch_fft_tile_t<8>(a, st, pdl);
        case 9: return launch_fft_tile_t<9>(a, st, pdl);
        case 10: return launch_fft_tile_t<10>(a, st, pdl);
        case 11: return launch_fft_tile_t<11>(a, st, pdl);
        case 12: return launch_fft_tile_t<12>(a, st, pdl);
        case 13: return launch_fft_tile_t<13>(a, st, pdl);
        case 14: return launch_fft_tile_t<14>(a, st, pdl);
        default: return set_err(FI_EINVAL, "no single-CTA FFT for 2^%d points", logn);
    }
}

// Blocks beyond one CTA: one cluster of NC = 2^LOGNC CTAs per block, 2^LOGN2 points
// per CTA (U = 2^13 .. 2^17 -> (2, 4096), (4, 4096), (8, 4096), (16, 4096), (16, 8192);
// clusters of 16 are a non-portable size that B200 supports).
template <int LOGNC, int LOGN2>
cudaLaunchConfig_t cluster_config(long long count, cudaStream_t st, cudaLaunchAttribute* at) {
    using G = ClusterTile<LOGNC, LOGN2>;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(count * G::NC));
    cfg.blockDim = dim3(G::T);
    cfg.dynamicSmemBytes = G::smem;
    cfg.stream = st;
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = G::NC;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cfg;
}

template <int LOGNC, int LOGN2>
int launch_cluster_t(const TileArgs& a, cudaStream_t st, int pdl) {
    cudaLaunchAttribute at[2];
    cudaLaunchConfig_t cfg = cluster_config<LOGNC, LOGN2>(a.count, st, at);
    set_pdl(&cfg, at, pdl);
    CK(cudaLaunchKernelEx(&cfg, k_block_fft_cluster<LOGNC, LOGN2, kTwLog>, a));
    return FI_OK;
}

int launch_cluster_tile(int q, const TileArgs& a, cudaStream_t st, int pdl) {
    switch (q) {
        case 13: return launch_cluster_t<1, 12>(a, st, pdl);
        case 14: return launch_cluster_t<2, 12>(a, st, pdl);
        case 15: return launch_cluster_t<3, 12>(a, st, pdl);
        case 16: return launch_cluster_t<4, 12>(a, st, pdl);
        case 17: return launch_cluster_t<4, 13>(a, st, pdl);
        default: return set_err(FI_EINVAL, "no cluster FFT for 2^%d points", q);
    }
}

template <int LOGNC, int LOGN2>
int launch_spectra_cluster_t(const float* taps, long long ld, int count, float2* spec, long long hstride,
                             const float2* tw, cudaStream_t st, float scale) {
    cudaLaunchAttribute at[1];
    cudaLaunchConfig_t cfg = cluster_config<LOGNC, LOGN2>(count, st, at);
    CK(cudaLaunchKernelEx(&cfg, k_spectra_cluster<LOGNC, LOGN2, kTwLog>, taps, ld, spec, hstride, tw, scale));
    return FI_OK;
}

int launch_spectra_cluster(int q, const float* taps, long long ld, int count, float2* spec, long long hstride,
                           const float2* tw, cudaStream_t st, float scale) {
    switch (q) {
        case 13: return launch_spectra_cluster_t<1, 12>(taps, ld, count, spec, hstride, tw, st, scale);
        case 14: return launch_spectra_cluster_t<2, 12>(taps, ld, count, spec, hstride, tw, st, scale);
        case 15: return launch_spectra_cluster_t<3, 12>(taps, ld, count, spec, hstride, tw, st, scale);
        case 16: return launch_spectra_cluster_t<4, 12>(taps, ld, count, spec, hstride, tw, st, scale);
        case 17: return launch_spectra_cluster_t<4, 13>(taps, ld, count, spec, hstride, tw, st, scale);
        default: return set_err(FI_EINVAL, "no cluster spectrum kernel for 2^%d points", q);
    }
}

int launch_direct_tile(const TileArgs& a, cudaStream_t st) {
    if (a.U <= 8 && (a.U & (a.U - 1)) == 0) {
        const unsigned grid = (unsigned)((a.count + 127) / 128);
        switch (a.U) {
            case 1: k_tile_direct_small<1><<<grid, 128, 0, st>>>(a); break;
            case 2: k_tile_direct_small<2><<<grid, 128, 0, st>>>(a); break;
            case 4: k_tile_direct_small<4><<<grid, 128, 0, st>>>(a); break;
            default: k_tile_direct_small<8><<<grid, 128, 0, st>>>(a); break;
        }
        CK(cudaGetLastError());
        return FI_OK;
    }
    const size_t smem = (size_t)3 * a.U * sizeof(float);
    k_tile_direct<kDirectNT, 4><<<a.count, kDirectNT, smem, st>>>(a);
    CK(cudaGetLastError());
    return FI_OK;
}

// Spectra of the FFT tau carry the kernels' 1/(2U) scale (fused_scale).  Complex
// entries per (layer, channel) spectrum: bins 0..U plus one pad entry, so that every
// spectrum starts on a 16-byte boundary (async copies).
float fused_scale(int q) { return 1.0f / (2.0f * (float)(1LL << q)); }
long long fused_stride(long long U) { return U + 2; }

template <int LOGN>
int launch_spectra_t(const float* taps, long long ld, int count, int nspec, long long offstep,
                     float2* spec, const float2* tw, cudaStream_t st, float scale, long long hstride) {
    constexpr int NT = (1 << LOGN) / 4 < 32 ? 32 : ((1 << LOGN) / 4 > 1024 ? 1024 : (1 << LOGN) / 4);
    const size_t smem = sizeof(float2) << LOGN;
    k_spectra<LOGN, NT><<<count * nspec, NT, smem, st>>>(taps, ld, nspec, offstep, spec, tw, kTwLog, scale, hstride);
    CK(cudaGetLastError());
    return FI_OK;
}

int launch_spectra(int logn, const float* taps, long long ld, int count, int nspec, long long offstep,
                   float2* spec, const float2* tw, cudaStream_t st, float scale, long long hstride) {
    switch (logn) {
        case 3: return launch_spectra_t<3>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 4: return launch_spectra_t<4>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 5: return launch_spectra_t<5>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 6: return launch_spectra_t<6>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 7: return launch_spectra_t<7>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 8: return launch_spectra_t<8>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 9: return launch_spectra_t<9>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 10: return launch_spectra_t<10>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 11: return launch_spectra_t<11>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 12: return launch_spectra_t<12>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 13: return launch_spectra_t<13>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        case 14: return launch_spectra_t<14>(taps, ld, count, nspec, offstep, spec, tw, st, scale, hstride);
        default: return set_err(FI_EINVAL, "no spectrum kernel for 2^%d points", logn);
    }
}

// Largest block size served by the one-CTA FFT tile kernel; larger ones run on a
// cluster of CTAs.  The choice is fixed per process (FI_FUSED_QMAX overrides it).
int fused_qmax() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("FI_FUSED_QMAX");
        const int x = e ? atoi(e) : 14;
        v = std::max(12, std::min(kFusedQLimit, x));
    }
    return v;
}

// Filter spectra of `count` tap rows (row i at taps + i * ld) for block size 2^q, in
// the layout the FFT tau of that size reads (natural order for one CTA, CTA order
// for clusters), stride fused_stride(2^q).
int make_spectra(int q, const float* taps, long long ld, int count, float2* spec, const float2* tw,
                 cudaStream_t st) {
    if (q <= fused_qmax())
        return launch_spectra(q, taps, ld, count, 1, 0, spec, tw, st, fused_scale(q), fused_stride(1LL << q));
    return launch_spectra_cluster(q, taps, ld, count, spec, fused_stride(1LL << q), tw, st, fused_scale(q));
}

// The FFT tau of block size 2^q over a.count tiles.
int launch_fft(int q, const TileArgs& a, cudaStream_t st, int pdl = 0) {
    return q <= fused_qmax() ? launch_fft_tile(q, a, st, pdl) : launch_cluster_tile(q, a, st, pdl);
}

// chains per CTA fixed at compile time for the 18-layer stack at B = 1 with 6 channels
// per CTA (864 or fewer channels over 148 SMs), W = 128
constexpr int kWinCPBT = 6;
bool win_fixed_geom(const fi_ctx* c, int W) {
    return W == 128 && c->M == 18 && c->B == 1 && c->kch == kWinCPBT;
}

template <int W, int MAXM>
int launch_window_t(const fi_ctx* c, const WinArgs& a, cudaStream_t st, int pdl) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)c->win_ncta);
    cfg.blockDim = dim3(kWinThreads);
    cfg.dynamicSmemBytes = c->win_smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    set_pdl(&cfg, at, pdl);
    if constexpr (W == 128 && MAXM == 18) {
        if (win_fixed_geom(c, W)) {
            CK(cudaLaunchKernelEx(&cfg, k_window<W, MAXM, true, kWinCPBT>, a));
            return FI_OK;
        }
    }
    CK(cudaLaunchKernelEx(&cfg, k_window<W, MAXM, MAXM == 18, 0>, a));
    return FI_OK;
}

template <int W>
int launch_window_w(const fi_ctx* c, const WinArgs& a, cudaStream_t st, int pdl) {
    switch (win_maxm(c->M)) {
        case 8: return launch_window_t<W, 8>(c, a, st, pdl);
        case 18: return launch_window_t<W, 18>(c, a, st, pdl);
        case 20: return launch_window_t<W, 20>(c, a, st, pdl);
        case 40: return launch_window_t<W, 40>(c, a, st, pdl);
        default: return set_err(FI_EINVAL, "window kernel supports at most 40 layers");
    }
}

int launch_window(const fi_ctx* c, const WinArgs& a, cudaStream_t st, int pdl) {
    switch (c->W) {
        case 32: return launch_window_w<32>(c, a, st, pdl);
        case 64: return launch_window_w<64>(c, a, st, pdl);
        case 128: return launch_window_w<128>(c, a, st, pdl);
        case 256: return launch_window_w<256>(c, a, st, pdl);
        default: return set_err(FI_EINVAL, "unsupported window %d", c->W);
    }
}

// Dynamic shared memory above 48 KB must be enabled per kernel before the first
// launch (and before any graph capture); done once per process.
template <int LOGN>
int attr_fft() {
    constexpr int NT = (1 << LOGN) / 4 < 32 ? 32 : ((1 << LOGN) / 4 > 1024 ? 1024 : (1 << LOGN) / 4);
    const int smem = (int)(sizeof(float2) << LOGN);
    CK(cudaFuncSetAttribute(k_block_fft<LOGN, kTwLog>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)FftTile<LOGN>::smem));
    CK(cudaFuncSetAttribute(k_spectra<LOGN, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    return FI_OK;
}

template <int LOGNC, int LOGN2>
int attr_cluster() {
    using G = ClusterTile<LOGNC, LOGN2>;
    CK(cudaFuncSetAttribute(k_block_fft_cluster<LOGNC, LOGN2, kTwLog>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)G::smem));
    CK(cudaFuncSetAttribute(k_spectra_cluster<LOGNC, LOGN2, kTwLog>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)G::smem));
    if (G::NC > 8) {
        CK(cudaFuncSetAttribute(k_block_fft_cluster<LOGNC, LOGN2, kTwLog>,
                                cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
        CK(cudaFuncSetAttribute(k_spectra_cluster<LOGNC, LOGN2, kTwLog>,
                                cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    }
    return FI_OK;
}

template <int W>
int attr_window() {
    CK(cudaFuncSetAttribute(k_window<W, 8, false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax));
    CK(cudaFuncSetAttribute(k_window<W, 18, true, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax));
    CK(cudaFuncSetAttribute(k_window<W, 20, false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax));
    CK(cudaFuncSetAttribute(k_window<W, 40, false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax));
    if constexpr (W == 128)
        CK(cudaFuncSetAttribute(k_window<W, 18, true, kWinCPBT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemMax));
    return FI_OK;
}

int set_all_attrs() {
    static int done = 0;
    if (done) return FI_OK;
    int rc = 0;
    rc |= attr_fft<3>() | attr_fft<4>() | attr_fft<5>() | attr_fft<6>() | attr_fft<7>() | attr_fft<8>();
    rc |= attr_fft<9>() | attr_fft<10>() | attr_fft<11>() | attr_fft<12>() | attr_fft<13>() | attr_fft<14>();
    rc |= attr_cluster<1, 12>() | attr_cluster<2, 12>() | attr_cluster<3, 12>() | attr_cluster<4, 12>();
    rc |= attr_cluster<4, 13>();
    rc |= attr_window<32>() | attr_window<64>() | attr_window<128>() | attr_window<256>();
    if (rc) return FI_ECUDA;
    CK(cudaFuncSetAttribute(k_tile_direct<kDirectNT, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)(3 * (1 << kDirectQMax) * sizeof(float))));
    done = 1;
    return FI_OK;
}

TileArgs stack_tile_args(const fi_ctx* c, long long n) {
    TileArgs a;
    memset(&a, 0, sizeof(a));
    a.act = c->act;
    a.act_out = c->yout ? c->yout : c->act + c->G * c->L;
    a.h = c->h;
    a.L = c->L;
    a.G = c->G;
    a.D = c->D;
    a.n = n;
    a.U = (int)lowbit(n);
    a.count = (int)(c->M * c->G);
    a.overwrite = is_pow2(n) ? 1 : 0;
    a.tw = c->tw;
    a.twlog = kTwLog;
    return a;
}

// The gray blocks of every layer released after the n-th token, one launch
// (section "Schicht-uebergreifende Parallelisierung (Algorithmus 3)").
int launch_block(fi_ctx* c, long long n, int impl, cudaStream_t st, int pdl = 0, int force_acc = 0,
                 TokIO* io = nullptr) {
    TileArgs a = stack_tile_args(c, n);
    if (force_acc) a.overwrite = 0;
    a.io = io;  // replayed per-token graph: the kernels take n from the step record
    a.advance = io ? 1 : 0;  // and this launch closes the token
    const int q = ctz64(n);
    const int cls = impl == FI_TAU_DIRECT ? FI_K_BLOCK_DIRECT
                    : (q <= fused_qmax() ? FI_K_BLOCK_FFT : FI_K_BLOCK_CLUSTER);
    if (impl != FI_TAU_DIRECT) {
        a.spec = c->spec[q];
        a.spec_stride = c->spec_stride[q];
    }
    auto one = [&](const TileArgs& b) {
        LaunchScope scope(c, cls, st, q);
        return impl == FI_TAU_DIRECT ? launch_direct_tile(b, st) : launch_fft(q, b, st, pdl);
    };
    if (!c->layer_split) return one(a);
    // ablation: the same blocks as M launches of one layer each (the layer's buffers,
    // filters and spectra addressed as layer 0 of a one-layer stack)
    for (int l = 0; l < c->M; ++l) {
        TileArgs b = a;
        b.act = a.act + (long long)l * c->G * c->L;
        b.act_out = a.act_out + (long long)l * c->G * c->L;
        b.h = a.h + (long long)l * c->D * c->L;
        if (b.spec) b.spec = a.spec + (long long)l * c->D * a.spec_stride;
        b.count = (int)c->G;
        b.advance = (l == c->M - 1) ? a.advance : 0;  // only the last launch closes the token
        int rc = one(b);
        if (rc) return rc;
    }
    return FI_OK;
}

int upload_twiddles(fi_ctx* c) {
    const int nt = 1 << kTwLog;
    std::vector<float2> tw(nt);
    for (int k = 0; k < nt; ++k) {
        double ang = -2.0 * M_PI * (double)k / (double)nt;
        tw[k] = make_float2((float)cos(ang), (float)sin(ang));
    }
    int rc = dev_alloc(c, &c->tw, (size_t)nt);
    if (rc) return rc;
    CK(cudaMemcpy(c->tw, tw.data(), sizeof(float2) * nt, cudaMemcpyHostToDevice));
    return FI_OK;
}

int tau_impl(fi_ctx* tmp, int impl, int U, int q, int count, const float* blocks, const float* taps, int ldt,
             float* out, int accumulate) {
    TileArgs a;
    memset(&a, 0, sizeof(a));
    a.flat = 1;
    a.fin = blocks;
    a.fout = out;
    a.ftaps = taps;
    a.ldt = ldt;
    a.U = U;
    a.count = count;
    a.overwrite = accumulate ? 0 : 1;
    cudaStream_t st = nullptr;
    int rc;
    if (impl == FI_TAU_DIRECT) {
        rc = launch_direct_tile(a, st);
    } else {
        if ((rc = upload_twiddles(tmp))) return rc;
        a.tw = tmp->tw;
        a.twlog = kTwLog;
        if ((rc = dev_alloc(tmp, &tmp->spec[0], (size_t)count * fused_stride(U)))) return rc;
        if ((rc = make_spectra(q, taps, ldt, count, tmp->spec[0], tmp->tw, st))) return rc;
        a.spec = tmp->spec[0];
        a.spec_stride = fused_stride(U);
        rc = launch_fft(q, a, st);
    }
    if (rc) return rc;
    CK(cudaStreamSynchronize(st));
    return FI_OK;
}

// ---------------------------------------------------------------- allocation-free FFT tau
// Scratch of fi_tau_fft_noalloc: one fixed array per device, part of the library's
// device image, so it exists from module load to process exit and needs no
// cudaMalloc.  Layout (complex64 entries): [0, 2^kTwLog) twiddles, written once per
// device at set-up; then the filter spectra of one chunk of items.
constexpr int kNoAllocMaxDevices = 64;
constexpr int kNoAllocQMax = 16;  // largest block (U = 65536) the fixed array serves
std::mutex g_noalloc_mu;
float2* g_noalloc_base[kNoAllocMaxDevices] = {};
void* g_noalloc_ctx[kNoAllocMaxDevices] = {};  // context the set-up was made in

// The calling thread's current context (the driver's handle), looked up through the
// runtime's driver entry point so that the library needs no link against libcuda.
// A device reset or a context teardown gives the device a new context, in which the
// module (and the fixed array) is loaded afresh: the cached address and the twiddle
// table written into the old one no longer hold.
int current_context(void** out) {
    typedef int (*GetCurrent)(void**);
    static GetCurrent fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
            cudaGetLastError();
            return set_err(FI_ECUDA, "fi_tau_fft_noalloc: cuCtxGetCurrent entry point unavailable");
        }
        fn = (GetCurrent)p;
    }
    *out = nullptr;
    if (fn(out) != 0 || !*out) return set_err(FI_ECUDA, "fi_tau_fft_noalloc: no current CUDA context");
    return FI_OK;
}

// Once per device and context, with that device current: resolve the array's device
// address (the host-side symbol is only a stand-in) and store the twiddle table in it.
int noalloc_setup(int dev, float2** base) {
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return set_err(FI_EINVAL, "fi_tau_fft_noalloc: device ordinal %d above %d", dev, kNoAllocMaxDevices - 1);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    CK(cudaSetDevice(dev));  // makes the device's primary context current (creating it if needed)
    void* ctx = nullptr;
    int rc = current_context(&ctx);
    if (rc) return rc;
    if (!g_noalloc_base[dev] || g_noalloc_ctx[dev] != ctx) {
        g_noalloc_base[dev] = nullptr;
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return set_err(FI_ECUDA, "fi_tau_fft_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        }
        const int nt = 1 << kTwLog;
        std::vector<float2> tw(nt);
        for (int k = 0; k < nt; ++k) {
            const double ang = -2.0 * M_PI * (double)k / (double)nt;
            tw[k] = make_float2((float)cos(ang), (float)sin(ang));
        }
        e = cudaMemcpy(p, tw.data(), sizeof(float2) * nt, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return set_err(FI_ECUDA, "fi_tau_fft_noalloc: twiddle upload failed: %s", cudaGetErrorString(e));
        }
        g_noalloc_base[dev] = (float2*)p;
        g_noalloc_ctx[dev] = ctx;
    }
    *base = g_noalloc_base[dev];
    return FI_OK;
}

// The FFT tau of fi_tau, with every temporary carved out of the fixed array and the
// items processed in chunks small enough to fit it.
int tau_fft_noalloc_impl(int U, int q, int count, const float* blocks, const float* taps, int ldt, float* out,
                         int accumulate) {
    int dev = 0;
    CK(cudaGetDevice(&dev));
    float2* base = nullptr;
    int rc = noalloc_setup(dev, &base);
    if (rc) return rc;
    const long long ntw = 1LL << kTwLog;
    float2* spec = base + ntw;
    const long long avail = (long long)(kNoAllocScratchBytes / sizeof(float2)) - ntw;
    cudaStream_t st = nullptr;
    TileArgs a;
    memset(&a, 0, sizeof(a));
    a.flat = 1;
    a.ldt = ldt;
    a.U = U;
    a.overwrite = accumulate ? 0 : 1;
    a.tw = base;
    a.twlog = kTwLog;
    const long long per_item = fused_stride(U);
    const int chunk = (int)std::min<long long>(count, avail / per_item);
    for (int i0 = 0; i0 < count; i0 += chunk) {
        const int n = std::min(chunk, count - i0);
        const float* tp = taps + (long long)i0 * ldt;
        if ((rc = make_spectra(q, tp, ldt, n, spec, base, st))) return rc;
        a.fin = blocks + (long long)i0 * U;
        a.fout = out + (long long)i0 * U;
        a.ftaps = tp;
        a.count = n;
        a.spec = spec;
        a.spec_stride = per_item;
        if ((rc = launch_fft(q, a, st))) return rc;
    }
    CK(cudaStreamSynchronize(st));
    return FI_OK;
}

int tau_of(const fi_ctx* c, int q) { return c->tau_user[q] ? c->tau_user[q] : c->tau[q]; }

// ---------------------------------------------------------------- launch sequences
int enqueue_token(fi_ctx* c, long long t, const float* x, float* y, int closed, cudaStream_t st,
                  TokIO* io = nullptr) {
    StepArgs a;
    a.io = io;
    a.advance = 0;
    a.act = c->act;
    a.h = c->h;
    a.M = c->M;
    a.D = c->D;
    a.L = c->L;
    a.G = c->G;
    a.t = t;
    a.x = x;
    a.y = y;
    a.closed = closed;
    a.fuseU = 0;
    const long long n = t + 1;
    int q = -1, impl = 0;
    if (n < c->L) {
        q = ctz64(n);
        impl = tau_of(c, q);
        if (q <= kFuseQMax && impl == FI_TAU_DIRECT) a.fuseU = 1 << q;
    }
    const int grid = (int)((c->G + 31) / 32);
    const bool block_follows = n < c->L && a.fuseU == 0;
    a.advance = (io && !block_follows) ? 1 : 0;  // the step kernel closes the token itself
    {
        LaunchScope scope(c, FI_K_TOKEN_STEP, st);
        k_token_step<kStepNT><<<grid, kStepNT, 0, st>>>(a);
        CK(cudaGetLastError());
    }
    if (block_follows) return launch_block(c, n, impl, st, 0, 0, io);
    return FI_OK;
}

// The launches of one token step with the token taken from the step record: the step
// kernel and the block released after it (edge 2^q; none for the last token), the last
// of them advancing the record.  Captured once per (mode, q) into a graph.
int capture_token_graph(fi_ctx* c, int closed, int idx) {
    const long long t = idx == 32 ? c->L - 1 : (1LL << idx) - 1;  // a token releasing edge 2^idx
    c->enq_launches = 0;
    CK(cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed));
    int rc = enqueue_token(c, t, nullptr, nullptr, closed, c->cap, c->tio);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->cap, &graph);
    if (!rc && e == cudaSuccess) e = cudaGetLastError();
    if (rc || e != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return rc ? rc : set_err(FI_ECUDA, "token graph capture failed: %s", cudaGetErrorString(e));
    }
    const char* f = getenv("FI_FAULT");
    if (f && strstr(f, "capture")) {
        cudaGraphDestroy(graph);
        return set_err(FI_ECUDA, "injected graph capture failure (FI_FAULT=capture)");
    }
    e = cudaGraphInstantiate(&c->tokg[closed][idx], graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
        c->tokg[closed][idx] = nullptr;
        return set_err(FI_ECUDA, "token graph instantiate failed: %s", cudaGetErrorString(e));
    }
    c->tokg_nodes[closed][idx] = c->enq_launches;
    return FI_OK;
}

// The per-token path from captured graphs: the step record is set once for the call,
// then one graph replay per token, the graph of the block size the token releases.
int run_token_graphs(fi_ctx* c, long long t0, long long steps, const float* x, float* out, int closed) {
    for (long long t = t0; t < t0 + steps; ++t) {  // capture what this call needs first
        const long long n = t + 1;
        const int idx = n < c->L ? ctz64(n) : 32;
        if (!c->tokg[closed][idx]) {
            int rc = capture_token_graph(c, closed, idx);
            if (rc) return rc;
        }
    }
    TokIO v;
    memset(&v, 0, sizeof(v));
    v.x = x;
    v.y = out;
    v.tx = t0;
    v.t = t0;
    v.closed = closed;
    v.done = 0;
    k_set_step<<<1, 1, 0, c->stream>>>(c->tio, v);
    CK(cudaGetLastError());
    long long nl = 1;
    for (long long t = t0; t < t0 + steps; ++t) {
        const long long n = t + 1;
        const int idx = n < c->L ? ctz64(n) : 32;
        CK(cudaGraphLaunch(c->tokg[closed][idx], c->stream));
        nl += c->tokg_nodes[closed][idx];
    }
    c->launches += nl;
    c->last_trace = nullptr;
    return FI_OK;
}

int enqueue_window_path(fi_ctx* c, long long t0, long long steps, const float* x, float* out, int closed,
                        cudaStream_t st) {
    const long long W = c->W, L = c->L, end = t0 + steps;
    long long t = t0;
    while (t < end) {
        const long long k = t / W;
        const long long wend = std::min((k + 1) * W, L);
        const long long t1 = std::min(end, wend);
        WinArgs a;
        a.act = c->act;
        a.h = c->h;
        a.M = c->M;
        a.B = c->B;
        a.D = c->D;
        a.L = L;
        a.G = c->G;
        a.t0 = t;
        a.t1 = t1;
        a.tx = t0;
        a.x = closed ? (t == t0 ? x : nullptr) : x;
        a.out = out;
        a.closed = closed;
        a.kch = c->kch;
        int rc;
        {
            LaunchScope scope(c, FI_K_WINDOW, st);
            // the call's first launch follows the staging copies of its inputs, which
            // griddepcontrol.wait does not wait for: no programmatic dependent launch
            rc = launch_window(c, a, st, t == t0 ? 0 : c->pdl);
        }
        if (rc) return rc;
        if (t1 == (k + 1) * W && t1 < L) {
            rc = launch_block(c, t1, tau_of(c, ctz64(t1)), st, c->pdl);
            if (rc) return rc;
        }
        t = t1;
    }
    return FI_OK;
}

int enqueue(fi_ctx* c, long long t0, long long steps, const float* x, float* out, int closed, cudaStream_t st) {
    if (c->path == FI_PATH_WINDOW && c->W > 0) return enqueue_window_path(c, t0, steps, x, out, closed, st);
    for (long long k = 0; k < steps; ++k) {
        const float* xk = closed ? (k == 0 ? x : nullptr) : x + k * c->G;
        int rc = enqueue_token(c, t0 + k, xk, out + k * c->G, closed, st);
        if (rc) return rc;
    }
    return FI_OK;
}

void drop_graphs(fi_ctx* c) {
    if (c->last_trace != &c->eager_trace) c->last_trace = nullptr;
    for (auto& kv : c->gcache) cudaGraphExecDestroy(kv.second.exec);
    c->gcache.clear();
    c->gorder.clear();
    for (int m = 0; m < 2; ++m)
        for (int i = 0; i < 33; ++i) {
            if (c->tokg[m][i]) cudaGraphExecDestroy(c->tokg[m][i]);
            c->tokg[m][i] = nullptr;
        }
}

// Run a launch sequence, from a captured graph when enabled (section
// "Implementierungsdetails": CUDA graphs remove the per-launch CPU overhead).
// The Lazy / Eager baselines: one launch per token, one CTA per chain.
int run_baseline(fi_ctx* c, long long t0, long long steps, const float* x, float* out, int closed) {
    const bool eager = c->path == FI_PATH_EAGER || c->path == FI_PATH_EAGER_NP;
    const bool np = c->path == FI_PATH_LAZY_NP || c->path == FI_PATH_EAGER_NP;
    if (eager && t0 == 0)  // running sums of layers 1..M start at zero
        CK(cudaMemsetAsync(c->act + c->G * c->L, 0, sizeof(float) * c->M * c->G * c->L, c->stream));
    BaseArgs a;
    a.act = c->act;
    a.h = c->h;
    a.M = c->M;
    a.D = c->D;
    a.G = c->G;
    a.L = c->L;
    a.tx = t0;
    a.x = x;
    a.out = out;
    a.closed = closed;
    const int threads = 32 * std::min(c->M, 32);
    const size_t smem = (size_t)(2 * c->M + 1) * sizeof(float);
    const int np_threads = eager ? 512 : 256;
    for (long long t = t0; t < t0 + steps; ++t) {
        a.t = t;
        a.first = t == t0;
        if (np) {
            // one launch per layer, in layer order: no two layers' work side by side
            for (int l = 1; l <= c->M; ++l) {
                if (eager) k_eager_layer<<<(unsigned)c->G, np_threads, 0, c->stream>>>(a, l);
                else k_lazy_layer<<<(unsigned)c->G, np_threads, (np_threads / 32) * sizeof(float), c->stream>>>(a, l);
            }
        } else if (eager) {
            k_eager_chain<<<(unsigned)((c->G + 127) / 128), 128, 0, c->stream>>>(a);
            k_eager_push<<<dim3((unsigned)c->G, (unsigned)c->M), 256, 0, c->stream>>>(a);
        } else {
            k_lazy_token<<<(unsigned)c->G, threads, smem, c->stream>>>(a);
        }
    }
    CK(cudaGetLastError());
    c->launches += np ? steps * c->M : (eager ? 2 * steps : steps);
    c->last_trace = nullptr;
    return FI_OK;
}

int run(fi_ctx* c, long long t0, long long steps, const float* x, float* out, int closed) {
    if (c->path >= FI_PATH_LAZY) return run_baseline(c, t0, steps, x, out, closed);
    const bool window = c->path == FI_PATH_WINDOW && c->W > 0;
    if (!window && c->graphs && !c->trace_on) return run_token_graphs(c, t0, steps, x, out, closed);
    c->enq_launches = 0;
    if (!c->graphs || !window) {
        c->eager_trace.clear();
        c->event_next = 0;
        c->rec = &c->eager_trace;
        int rc = enqueue(c, t0, steps, x, out, closed, c->stream);
        c->rec = nullptr;
        c->last_trace = &c->eager_trace;
        c->launches += c->enq_launches;
        return rc;
    }
    GraphKey key{c->path, closed, t0, steps, x, out};
    auto it = c->gcache.find(key);
    if (it == c->gcache.end()) {
        if ((int)c->gorder.size() >= kGraphCache) {
            GraphKey old = c->gorder.front();
            c->gorder.erase(c->gorder.begin());
            if (c->last_trace == &c->gcache[old].trace) c->last_trace = nullptr;
            cudaGraphExecDestroy(c->gcache[old].exec);
            c->gcache.erase(old);
        }
        GraphEntry ent;
        CK(cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed));
        c->rec = &ent.trace;
        int rc = enqueue(c, t0, steps, x, out, closed, c->cap);
        c->rec = nullptr;
        cudaGraph_t graph = nullptr;
        cudaError_t e = cudaStreamEndCapture(c->cap, &graph);
        if (rc) {
            if (graph) cudaGraphDestroy(graph);
            return rc;
        }
        if (e != cudaSuccess) return set_err(FI_ECUDA, "graph capture failed: %s", cudaGetErrorString(e));
        const char* f = getenv("FI_FAULT");
        if (f && strstr(f, "capture")) {
            cudaGraphDestroy(graph);
            return set_err(FI_ECUDA, "injected graph capture failure (FI_FAULT=capture)");
        }
        e = cudaGraphInstantiate(&ent.exec, graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) return set_err(FI_ECUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
        ent.launches = c->enq_launches;
        it = c->gcache.emplace(key, std::move(ent)).first;
        c->gorder.push_back(key);
    }
    CK(cudaGraphLaunch(it->second.exec, c->stream));
    c->last_trace = &it->second.trace;
    c->launches += it->second.launches;
    return FI_OK;
}

int ensure_stage(fi_ctx* c, float** buf, size_t* cap, size_t n) {
    if (*cap >= n) return FI_OK;
    if (*buf) {
        CK(cudaStreamSynchronize(c->stream));
        cudaFree(*buf);
        c->bytes -= *cap * sizeof(float);
        *buf = nullptr;
        *cap = 0;
        drop_graphs(c);  // graphs may reference the old staging buffer
    }
    int rc = dev_alloc(c, buf, n);
    if (rc) return rc;
    *cap = n;
    return FI_OK;
}

// ---------------------------------------------------------------- setup
int choose_window(fi_ctx* c) {
    const char* env = getenv("FI_WINDOW");
    int forced = env ? atoi(env) : 0;
    if (c->B > 32) return FI_OK;  // chain lanes: one warp per CTA
    if (!win_maxm(c->M)) return FI_OK;
    int kch0 = (int)((c->D + c->nsm - 1) / c->nsm);
    if (kch0 * c->B > 32) kch0 = std::max(1, 32 / c->B);
    // The window kernel holds one CTA per SM (its registers) and its CTAs never wait on
    // one another, so a launch may take several waves.  Per window W, the most channels
    // per CTA whose rows fit gives the fewest waves; a wave costs about the same per
    // token at any W, plus a per-launch overhead (~16 tokens' worth) that W amortises.
    const int cand[] = {128, 64, 256, 32};
    double best = 1e300;
    for (int W : cand) {
        if (forced && W != forced) continue;
        if (W > c->L) continue;
        for (int kch = kch0; kch >= 1; --kch) {
            const size_t sm = win_smem_bytes(W, c->M, c->B, kch);
            if (sm > kSmemMax) continue;
            const int ncta = (c->D + kch - 1) / kch;
            const int waves = (ncta + c->nsm - 1) / c->nsm;
            const double cost = waves * (1.0 + 16.0 / W);
            if (cost < best - 1e-9) {
                best = cost;
                c->W = W;
                c->kch = kch;
                c->win_ncta = ncta;
                c->win_smem = sm;
            }
            break;
        }
    }
    return FI_OK;  // W = 0: window path unavailable, per-token path only
}

// Device time of one launch of the blocks released at n with implementation impl:
// one warm-up launch, then `reps` launches each between its own pair of events; the
// median (robust to a launch that met a clock or scheduling hiccup).
float time_launch(fi_ctx* c, long long n, int impl, int reps) {
    if (launch_block(c, n, impl, c->cap)) return -1.f;
    std::vector<cudaEvent_t> ev(reps + 1);
    for (auto& e : ev) cudaEventCreate(&e);
    bool ok = cudaEventRecord(ev[0], c->cap) == cudaSuccess;
    for (int r = 0; r < reps && ok; ++r) {
        if (launch_block(c, n, impl, c->cap)) ok = false;
        if (ok) ok = cudaEventRecord(ev[r + 1], c->cap) == cudaSuccess;
    }
    std::vector<float> us;
    if (ok && cudaEventSynchronize(ev[reps]) == cudaSuccess) {
        for (int r = 0; r < reps; ++r) {
            float ms = 0.f;
            cudaEventElapsedTime(&ms, ev[r], ev[r + 1]);
            us.push_back(1000.f * ms);
        }
    }
    for (auto& e : ev) cudaEventDestroy(e);
    if (us.size() != (size_t)reps) return -1.f;
    std::sort(us.begin(), us.end());
    return us[reps / 2];
}

// Hybrid tau: time each implementation able to serve block size 2^q and keep the
// faster (ties go to direct).  The timing launches write into positions that the
// first real block onto them overwrites, so they leave no trace.
int autotune(fi_ctx* c) {
    const char* env = getenv("FI_TAU");  // "q:impl,q:impl" with impl d|f
    for (int q = 0; q < c->P; ++q) {
        const long long U = 1LL << q;
        const bool can_d = q <= kDirectQMax;
        const bool can_f = c->spec[q] != nullptr;
        float td = 0.f, tf = 0.f;
        if (can_d && can_f) {
            td = time_launch(c, U, FI_TAU_DIRECT, 7);
            tf = time_launch(c, U, FI_TAU_FFT, 7);
            if (td < 0 || tf < 0) return FI_ECUDA;
        }
        c->tau_us[q][0] = td;
        c->tau_us[q][1] = tf;
        if (can_d && can_f) c->tau[q] = (tf < td) ? FI_TAU_FFT : FI_TAU_DIRECT;
        else c->tau[q] = can_f ? FI_TAU_FFT : FI_TAU_DIRECT;
        (void)U;
    }
    if (env) {
        const char* p = env;
        while (*p) {
            int q = atoi(p);
            const char* colon = strchr(p, ':');
            if (!colon) break;
            char k = colon[1];
            if (q >= 0 && q < c->P) {
                if (k == 'd' && q <= kDirectQMax) c->tau[q] = FI_TAU_DIRECT;
                if (k == 'f' && c->spec[q]) c->tau[q] = FI_TAU_FFT;
            }
            const char* comma = strchr(colon, ',');
            if (!comma) break;
            p = comma + 1;
        }
    }
    return FI_OK;
}

void free_ctx(fi_ctx* c) {
    if (!c) return;
    cudaStreamSynchronize(c->stream);
    drop_graphs(c);
    cudaFree(c->act);
    cudaFree(c->h);
    cudaFree(c->tw);
    for (int q = 0; q < 32; ++q) cudaFree(c->spec[q]);
    cudaFree(c->sx);
    cudaFree(c->sy);
    cudaFree(c->pre);
    cudaFree(c->pre_spec);
    cudaFree(c->tio);
    for (cudaEvent_t e : c->event_pool) cudaEventDestroy(e);
    if (c->cap) cudaStreamDestroy(c->cap);
    c->magic = 0;
    delete c;
}

int create_impl(fi_ctx* c, const float* filters) {
    int rc0 = set_all_attrs();
    if (rc0) return rc0;
    CK(cudaGetDevice(&c->dev));
    CK(cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, c->dev));
    CK(cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking));
    if (const char* e = getenv("FI_PDL")) c->pdl = atoi(e) ? 1 : 0;
    if (const char* e = getenv("FI_LAYER_SPLIT")) c->layer_split = atoi(e) ? 1 : 0;
    const long long M = c->M, D = c->D, L = c->L, G = c->G;
    int rc;
    if ((rc = dev_alloc(c, &c->act, (size_t)(M + 1) * G * L))) return rc;
    if ((rc = dev_alloc(c, &c->h, (size_t)M * D * L))) return rc;
    if ((rc = dev_alloc(c, &c->tio, 1))) return rc;
    CK(cudaMemcpyAsync(c->h, filters, sizeof(float) * M * D * L, cudaMemcpyDefault, c->cap));
    // twiddles from fp64 host trigonometry
    if ((rc = upload_twiddles(c))) return rc;
    // filter spectra for every FFT-served block size
    for (int q = kFftQMin; q < c->P && q <= kFftQMax; ++q) {
        const long long U = 1LL << q;
        c->spec_stride[q] = fused_stride(U);
        if ((rc = dev_alloc(c, &c->spec[q], (size_t)(M * D) * fused_stride(U)))) return rc;
        if ((rc = make_spectra(q, c->h, L, (int)(M * D), c->spec[q], c->tw, c->cap))) return rc;
    }
    CK(cudaStreamSynchronize(c->cap));
    if ((rc = choose_window(c))) return rc;
    if ((rc = autotune(c))) return rc;
    CK(cudaStreamSynchronize(c->cap));
    return FI_OK;
}


}  // namespace

// ====================================================================== C-ABI
// Prompt prefill (x, y device pointers): the prompt's activations layer by layer, one
// FFT convolution per layer (U = the power of two >= p), then the state the tiled path
// expects at t = p: the running sum of every position >= p holds the blocks released
// up to p.  Those are the blocks n <= p whose outputs reach past p (n + lowbit(n) > p);
// the largest power of two n0 <= p is the first and widest, its outputs [n0, 2 n0)
// cover every other's.  They are replayed through the ordinary block launches onto
// zeroed positions [p, 2 n0), accumulating, in decreasing n: a block writes only at
// positions >= its own n, so no replayed block clobbers the inputs of one still to
// come.  Their outputs below p, already final activations, are saved before and
// restored after.
int prefill_impl(fi_ctx* c, const float* x, int p, float* y) {
    const long long G = c->G, L = c->L;
    const int M = c->M;
    int U = 1 << kFftQMin;
    while (U < p) U <<= 1;
    const int q = ctz64(U);
    cudaStream_t st = c->stream;
    long long n0 = 1;
    while (2 * n0 <= p) n0 <<= 1;  // the first open block: the largest power of two <= p
    // scratch (kept by the context): blocks [G][U], out [G][U] (together the shifted taps
    // [D][2U] while the spectra are made), the saved activations [M][G][p - n0]
    const size_t nb = (size_t)G * U;
    const size_t need = 2 * nb + (size_t)M * G * (size_t)(p - n0);
    int rc;
    if ((rc = ensure_stage(c, &c->pre, &c->pre_n, need))) return rc;
    float* blocks = c->pre;
    float* out = blocks + nb;
    float* saved_area = out + nb;
    const int grid = 4 * c->nsm, nt = 256;
    const long long sstride = fused_stride(U);
    // the spectra of the shifted taps of every layer and channel, once per prompt size
    // (the FFT precompute of section "Speicheroptimierung" for the prompt's block size);
    // the batch rows of a channel share them
    if (c->pre_spec_q != q) {
        const size_t ns = (size_t)M * c->D * sstride;
        if (c->pre_spec_n < ns) {
            CK(cudaStreamSynchronize(st));
            cudaFree(c->pre_spec);
            c->bytes -= c->pre_spec_n * sizeof(float2);
            c->pre_spec = nullptr;
            c->pre_spec_n = 0;
            c->pre_spec_q = -1;
            if ((rc = dev_alloc(c, &c->pre_spec, ns))) return rc;
            c->pre_spec_n = ns;
        }
        float* taps = blocks;  // [D][2U]: within blocks and out, 2 G U >= 2 D U floats
        for (int l = 1; l <= M; ++l) {
            k_prefill_taps<<<grid, nt, 0, st>>>(c->h, l, c->D, c->D, L, U, taps);
            if ((rc = make_spectra(q, taps, 2 * U, c->D, c->pre_spec + (size_t)(l - 1) * c->D * sstride, c->tw,
                                   st)))
                return rc;
        }
        CK(cudaGetLastError());
        c->pre_spec_q = q;
    }
    k_prefill_input<<<grid, nt, 0, st>>>(x, G, L, p, c->act);
    long long nl = 1;
    for (int l = 1; l <= M; ++l) {
        k_prefill_gather<<<grid, nt, 0, st>>>(c->act, l - 1, G, L, p, U, blocks);
        TileArgs a;
        memset(&a, 0, sizeof(a));
        a.flat = 1;
        a.fin = blocks;
        a.fout = out;
        a.ftaps = blocks;  // not read: the FFT tau reads only the spectra
        a.ldt = 2 * U;
        a.U = U;
        a.count = (int)G;
        a.overwrite = 1;
        a.tw = c->tw;
        a.twlog = kTwLog;
        a.spec = c->pre_spec + (size_t)(l - 1) * c->D * sstride;
        a.spec_stride = sstride;
        a.spec_mod = c->D;  // chain g = b D + c reads channel c's row
        if ((rc = launch_fft(q, a, st))) return rc;
        k_prefill_scatter<<<grid, nt, 0, st>>>(out, l, G, L, p, U, c->act, l == M ? y : nullptr);
        nl += 3;
    }
    CK(cudaGetLastError());
    float* saved = nullptr;
    if (n0 < p) {
        saved = saved_area;
        k_prefill_rows<<<grid, nt, 0, st>>>(c->act, saved, M, G, L, (int)n0, p, 1);
    }
    const long long zend = std::min<long long>(2 * n0, L);
    if (zend > p)
        CK(cudaMemset2DAsync(c->act + G * L + p, sizeof(float) * L, 0, sizeof(float) * (zend - p), (size_t)M * G, st));
    for (long long n = std::min<long long>(p, L - 1); n >= n0; --n) {
        if (n + lowbit(n) <= p) continue;
        if ((rc = launch_block(c, n, tau_of(c, ctz64(n)), st, 0, 1))) return rc;
        ++nl;
    }
    if (saved) k_prefill_rows<<<grid, nt, 0, st>>>(c->act, saved, M, G, L, (int)n0, p, 0);
    CK(cudaGetLastError());
    c->launches += nl;
    c->last_trace = nullptr;
    return FI_OK;
}

// ====================================================================== language model
// The Hyena-like model around the mixer (fi_lm.cuh has the layer it computes): one
// mixer context holds the long convolutions (act = the mixer inputs x of every layer,
// yout = their outputs y, filters and spectra), the rest are bf16 weights and small
// per-token buffers.  A token is a host-issued launch sequence: embedding; per layer
// the in-projection, the mixer step, the MLP; the LM head and the greedy choice; then
// the gray blocks of every layer in one launch (section "Schicht-uebergreifende
// Parallelisierung (Algorithmus 3)").
constexpr unsigned kLmMagic = 0xF1C71A11u;

struct fi_lm {
    unsigned magic = kLmMagic;
    fi_ctx* mix = nullptr;
    int M = 0, B = 0, D = 0, L = 0, V = 0;
    long long t = 0;
    __nv_bfloat16 *E = nullptr, *Wlm = nullptr, *Win = nullptr, *W1 = nullptr, *W2 = nullptr;
    float* conv = nullptr;                       // [M][3][3D]
    float *u = nullptr, *z = nullptr, *zr = nullptr, *m1 = nullptr;
    float* r = nullptr;                          // [B][D]: u + qc y_t, the MLP's input and residual
    int *tok = nullptr, *next = nullptr;         // [B]: the next input token, the latest choice
    unsigned long long* amax = nullptr;          // [B]: the LM head's running greedy choice (keys of lm_key)
    int* stage_i = nullptr;                      // host token arrays staged on the device
    size_t stage_i_n = 0;
    float* stage_f = nullptr;
    size_t stage_f_n = 0;
    // tracing: events around the mixer's block launches (every token) and mixer steps
    // (every kTraceEvery-th token), and around each whole call
    int trace_on = 0;
    std::vector<cudaEvent_t> ev;
    std::vector<std::pair<int, int>> ev_blocks, ev_steps;  // event index pairs
    int ev_call0 = -1, ev_call1 = -1;
    long long traced_tokens = 0, sampled_tokens = 0;
    // greedy generation from captured graphs: one per block size released (32: none)
    int graphs = 1;
    cudaGraphExec_t gen_graph[33] = {};
};

namespace {

std::mutex g_lm_mu;
std::set<const fi_lm*> g_lm_live;
constexpr int kTraceEvery = 64;

int check_lm(const fi_lm* m) {
    std::lock_guard<std::mutex> lk(g_lm_mu);
    if (!m || !g_lm_live.count(m) || m->magic != kLmMagic) return set_err(FI_ESTATE, "null or destroyed model");
    return FI_OK;
}

template <typename T>
int lm_alloc(fi_lm* m, T** p, size_t count) {
    return dev_alloc(m->mix, p, count);
}

// fp32 host or device weights -> bf16 device array
int lm_upload_bf16(fi_lm* m, const float* src, size_t n, __nv_bfloat16** dst) {
    int rc = lm_alloc(m, dst, n);
    if (rc) return rc;
    float* tmp = nullptr;
    CK(cudaMalloc((void**)&tmp, n * sizeof(float)));
    cudaError_t e = cudaMemcpy(tmp, src, n * sizeof(float), cudaMemcpyDefault);
    if (e == cudaSuccess) {
        k_to_bf16<<<1184, 256>>>(tmp, (long long)n, *dst);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    cudaFree(tmp);
    if (e != cudaSuccess) return set_err(FI_ECUDA, "weight upload failed: %s", cudaGetErrorString(e));
    return FI_OK;
}

int lm_event(fi_lm* m, cudaStream_t st) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    cudaEventRecord(e, st);
    m->ev.push_back(e);
    return (int)m->ev.size() - 1;
}

void lm_clear_trace(fi_lm* m) {
    for (cudaEvent_t e : m->ev) cudaEventDestroy(e);
    m->ev.clear();
    m->ev_blocks.clear();
    m->ev_steps.clear();
    m->ev_call0 = m->ev_call1 = -1;
    m->traced_tokens = m->sampled_tokens = 0;
}

// Launch with programmatic dependent launch (the model's kernels wait for their
// predecessors themselves, after prefetching what does not depend on them).
template <typename... KArgs, typename... Args>
int lm_launch(int pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args... args) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    set_pdl(&cfg, at, pdl);
    CK(cudaLaunchKernelEx(&cfg, kernel, args...));
    return FI_OK;
}

// Matrix-vector shapes: a warp per row slice of K / KS, RPW rows a warp at a time.
// W_in and W1 (K = D) take two rows a warp, the LM head (K = D, N = V rows) four; W2
// (K = 4D) splits each row over 4 warps, two rows a warp, so that either way a lane has
// all of its loads for a step in flight together and each shared-memory read of the
// inputs serves two or four rows.  At most kLmCtasPerSm CTAs an SM (one wave).
template <int EPI, int KS, int RPW>
int lm_gemv(int pdl, int nsm, const __nv_bfloat16* W, int N, int K, const float* x, int B, int ln, float* y,
            const LmEpi& ep, cudaStream_t st) {
    // units: rows, or (mixer epilogue) channels, one a warp
    const int units = EPI == kLmMix ? ep.D : N;
    const int per_cta = EPI == kLmMix ? (kLmThreads / 32) / KS : ((kLmThreads / 32) / KS) * RPW;
    const int grid = std::min((units + per_cta - 1) / per_cta, kLmCtasPerSm * nsm);
    const size_t smem = (size_t)B * K * sizeof(float);
    if (B <= 4)
        return lm_launch(pdl, k_lm_gemv<EPI, KS, RPW, 4>, dim3(grid), dim3(kLmThreads), smem, st, W, N, K, x, B, ln, y,
                         ep);
    return lm_launch(pdl, k_lm_gemv<EPI, KS, RPW, kLmMaxB>, dim3(grid), dim3(kLmThreads), smem, st, W, N, K, x, B, ln,
                     y, ep);
}

template <int EPI, int KS, int RPW>
int lm_gemv_attrs() {
    CK(cudaFuncSetAttribute(k_lm_gemv<EPI, KS, RPW, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)kSmemMax - 1024));
    CK(cudaFuncSetAttribute(k_lm_gemv<EPI, KS, RPW, kLmMaxB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)kSmemMax - 1024));
    return FI_OK;
}

// One token t: tok_src [B] (device) is its input; logits_out [B][V] (device) or null;
// next_out [B] (device) receives the greedy choice, also kept as the next input.
// first: the token's first launch follows copies or a memset of the call's set-up, which
// griddepcontrol.wait does not wait for, so it is launched without programmatic
// dependent launch; tracing also turns it off (overlapping launches blur the events).
int lm_token(fi_lm* m, long long t, const int* tok_src, float* logits_out, int* next_out, cudaStream_t st,
             TokIO* io = nullptr, bool first = false) {
    const int M = m->M, B = m->B, D = m->D, V = m->V;
    const long long L = m->L, G = (long long)B * D;
    fi_ctx* c = m->mix;
    // Programmatic dependent launch: each kernel releases its successor once its own
    // wait has returned, so at most one launch waits behind the running one (its weight
    // rows already streaming into L2).  Tracing turns it off.
    const int pdl = m->trace_on ? 0 : 1;
    int rc;
    if ((rc = lm_launch(first ? 0 : pdl, k_lm_embed, dim3((B * D + 255) / 256), dim3(256), 0, st, (const __nv_bfloat16*)m->E,
                        tok_src, B, D, m->u, m->amax)))
        return rc;
    const bool sample = m->trace_on && (t % kTraceEvery == 0);
    const LmEpi none = {};
    for (int l = 0; l < M; ++l) {
        // in-projection and mixer step: r = u + qc y_t (fused; traced runs launch the
        // mixer step on its own, to time it)
        LmEpi mx = {};
        mx.zr = m->zr + (size_t)l * 2 * B * 3 * D;
        mx.conv = m->conv + (size_t)l * 9 * D;
        mx.h = c->h + (size_t)l * D * L;
        mx.L = L;
        mx.t = t;
        mx.X = c->act + (size_t)l * G * L;
        mx.Y = c->yout + (size_t)l * G * L;
        mx.io = io;
        mx.D = D;
        const __nv_bfloat16* Win = m->Win + (size_t)l * 3 * D * D;
        if (!m->trace_on) {
            // a channel's three rows split over two warps (16-byte slices need D % 16 == 0)
            rc = (D % 16 == 0) ? lm_gemv<kLmMix, 2, 3>(pdl, c->nsm, Win, 3 * D, D, m->u, B, 1, m->r, mx, st)
                               : lm_gemv<kLmMix, 1, 3>(pdl, c->nsm, Win, 3 * D, D, m->u, B, 1, m->r, mx, st);
            if (rc) return rc;
        } else {
            // the same row split as the fused kernel: the same sums, bit for bit
            rc = (D % 16 == 0) ? lm_gemv<kLmStore, 2, 2>(pdl, c->nsm, Win, 3 * D, D, m->u, B, 1, m->z, none, st)
                               : lm_gemv<kLmStore, 1, 2>(pdl, c->nsm, Win, 3 * D, D, m->u, B, 1, m->z, none, st);
            if (rc) return rc;
            const int e0 = sample ? lm_event(m, st) : -1;
            if ((rc = lm_launch(pdl, k_lm_mixer, dim3((B * D + 127) / 128), dim3(128), 0, st, (const float*)m->z, mx.zr,
                                mx.conv, mx.h, L, B, D, t, mx.X, mx.Y, (const float*)m->u, m->r, (const TokIO*)io)))
                return rc;
            if (sample) m->ev_steps.push_back({e0, lm_event(m, st)});
        }
        // MLP: u = r + W2 bf16(GELU(W1 bf16(LN(r))))
        if ((rc = lm_gemv<kLmGelu, 1, 2>(pdl, c->nsm, m->W1 + (size_t)l * 4 * D * D, 4 * D, D, m->r, B, 1, m->m1, none,
                                         st)))
            return rc;
        LmEpi ad = {};
        ad.res = m->r;
        if ((rc = lm_gemv<kLmAdd, 4, 2>(pdl, c->nsm, m->W2 + (size_t)l * 4 * D * D, D, 4 * D, m->m1, B, 0, m->u, ad,
                                        st)))
            return rc;
    }
    // the LM head stores the logits only when they are asked for; its epilogue folds
    // every row into the greedy choice, which the pick kernel reads
    LmEpi hd = {};
    hd.amax = m->amax;
    if ((rc = lm_gemv<kLmArgmax, 1, 4>(pdl, c->nsm, m->Wlm, V, D, m->u, B, 1, logits_out, hd, st))) return rc;
    const bool block_follows = t + 1 < L;
    if ((rc = lm_launch(pdl, k_lm_pick, dim3(1), dim3(32), 0, st, (const unsigned long long*)m->amax, B, m->tok,
                        next_out, io, (io && !block_follows) ? 1 : 0)))
        return rc;
    if (block_follows) {
        const int e0 = m->trace_on ? lm_event(m, st) : -1;
        if ((rc = launch_block(c, t + 1, tau_of(c, ctz64(t + 1)), st, 0, 0, io))) return rc;  // the block kernels read through L1: no early start
        if (m->trace_on) m->ev_blocks.push_back({e0, lm_event(m, st)});
    }
    if (m->trace_on) {
        m->traced_tokens++;
        if (sample) m->sampled_tokens++;
    }
    return FI_OK;
}

int lm_run_graphs(fi_lm* m, int steps, int* next_d, cudaStream_t st) {
    fi_ctx* c = m->mix;
    const long long t0 = m->t;
    for (long long t = t0; t < t0 + steps; ++t) {  // capture what this call needs first
        const int idx = t + 1 < m->L ? ctz64(t + 1) : 32;
        if (m->gen_graph[idx]) continue;
        const long long tr = idx == 32 ? m->L - 1 : (1LL << idx) - 1;  // a token releasing 2^idx
        CK(cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed));
        int rc = lm_token(m, tr, m->tok, nullptr, nullptr, c->cap, c->tio, true);
        cudaGraph_t graph = nullptr;
        cudaError_t e = cudaStreamEndCapture(c->cap, &graph);
        if (rc || e != cudaSuccess) {
            if (graph) cudaGraphDestroy(graph);
            cudaGetLastError();
            return rc ? rc : set_err(FI_ECUDA, "model graph capture failed: %s", cudaGetErrorString(e));
        }
        e = cudaGraphInstantiate(&m->gen_graph[idx], graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) {
            m->gen_graph[idx] = nullptr;
            return set_err(FI_ECUDA, "model graph instantiate failed: %s", cudaGetErrorString(e));
        }
    }
    TokIO v;
    memset(&v, 0, sizeof(v));
    v.tx = t0;
    v.t = t0;
    v.itok = next_d;
    k_set_step<<<1, 1, 0, st>>>(c->tio, v);
    CK(cudaGetLastError());
    for (long long t = t0; t < t0 + steps; ++t) {
        const int idx = t + 1 < m->L ? ctz64(t + 1) : 32;
        CK(cudaGraphLaunch(m->gen_graph[idx], st));
    }
    return FI_OK;
}

int lm_stage(fi_lm* m, const int* src, size_t n, const int** out) {
    if (is_device_ptr(src)) {
        *out = src;
        return FI_OK;
    }
    if (m->stage_i_n < n) {
        cudaFree(m->stage_i);
        m->stage_i = nullptr;
        m->stage_i_n = 0;
        int rc = lm_alloc(m, &m->stage_i, n);
        if (rc) return rc;
        m->stage_i_n = n;
    }
    CK(cudaMemcpyAsync(m->stage_i, src, n * sizeof(int), cudaMemcpyHostToDevice, m->mix->stream));
    *out = m->stage_i;
    return FI_OK;
}

// a run of tokens: teacher (tokens [steps][B]) or closed loop (tok0 [B] at t = 0, or
// continuing from the last choice); outputs logits [steps][B][V] (or null) and the
// greedy choices [steps][B]
int lm_run(fi_lm* m, const int* tokens, const int* tok0, int steps, float* logits, int* next) {
    if (steps < 0) return set_err(FI_EINVAL, "steps must be >= 0");
    if (m->t + steps > m->L) return set_err(FI_ECAPACITY, "t=%lld + steps=%d exceeds capacity L=%d", m->t, steps, m->L);
    if (steps == 0) return FI_OK;
    if (!next) return set_err(FI_EINVAL, "the output token array is NULL");
    cudaStream_t st = m->mix->stream;
    const int B = m->B, V = m->V;
    int rc;
    const int* tok_d = nullptr;
    if (tokens) {
        if ((rc = lm_stage(m, tokens, (size_t)steps * B, &tok_d))) return rc;
    } else if (tok0) {
        const int* t0d = nullptr;
        if ((rc = lm_stage(m, tok0, (size_t)B, &t0d))) return rc;
        CK(cudaMemcpyAsync(m->tok, t0d, B * sizeof(int), cudaMemcpyDeviceToDevice, st));
    } else if (m->t == 0) {
        return set_err(FI_EINVAL, "closed loop at t=0 needs the start tokens");
    }
    const bool n_host = !is_device_ptr(next);
    const bool l_host = logits && !is_device_ptr(logits);
    int* next_d = next;
    float* logits_d = logits;
    const size_t need_f = (n_host ? (size_t)steps * B : 0) + (l_host ? (size_t)steps * B * V : 0);
    if (need_f > m->stage_f_n) {
        cudaFree(m->stage_f);
        m->stage_f = nullptr;
        m->stage_f_n = 0;
        if ((rc = lm_alloc(m, &m->stage_f, need_f))) return rc;
        m->stage_f_n = need_f;
    }
    if (n_host) next_d = reinterpret_cast<int*>(m->stage_f);
    if (l_host) logits_d = m->stage_f + (n_host ? (size_t)steps * B : 0);
    if (m->t == 0) CK(cudaMemsetAsync(m->zr, 0, sizeof(float) * (size_t)m->M * 2 * B * 3 * m->D, st));
    if (m->trace_on) {
        lm_clear_trace(m);
        m->ev_call0 = lm_event(m, st);
    }
    if (!tokens && m->graphs && !m->trace_on) {
        // greedy generation: one captured graph per block size, the token from the record
        if ((rc = lm_run_graphs(m, steps, next_d, st))) return rc;
    } else {
        for (int k = 0; k < steps; ++k) {
            const int* src = tokens ? tok_d + (size_t)k * B : m->tok;
            if ((rc = lm_token(m, m->t + k, src, logits ? logits_d + (size_t)k * B * V : nullptr,
                               next_d + (size_t)k * B, st, nullptr, k == 0)))
                return rc;
        }
    }
    if (m->trace_on) m->ev_call1 = lm_event(m, st);
    m->t += steps;
    if (n_host) CK(cudaMemcpyAsync(next, next_d, sizeof(int) * steps * B, cudaMemcpyDeviceToHost, st));
    if (l_host) CK(cudaMemcpyAsync(logits, logits_d, sizeof(float) * steps * B * V, cudaMemcpyDeviceToHost, st));
    if (n_host || l_host) CK(cudaStreamSynchronize(st));
    return FI_OK;
}

void lm_free(fi_lm* m) {
    if (!m) return;
    lm_clear_trace(m);
    for (int i = 0; i < 33; ++i)
        if (m->gen_graph[i]) cudaGraphExecDestroy(m->gen_graph[i]);
    if (m->mix) {
        cudaStreamSynchronize(m->mix->stream);
        cudaFree(m->mix->yout);
        m->mix->yout = nullptr;
        free_ctx(m->mix);
    }
    cudaFree(m->E);
    cudaFree(m->Wlm);
    cudaFree(m->Win);
    cudaFree(m->W1);
    cudaFree(m->W2);
    cudaFree(m->conv);
    cudaFree(m->u);
    cudaFree(m->z);
    cudaFree(m->zr);
    cudaFree(m->m1);
    cudaFree(m->r);
    cudaFree(m->amax);
    cudaFree(m->tok);
    cudaFree(m->next);
    cudaFree(m->stage_i);
    cudaFree(m->stage_f);
    m->magic = 0;
    delete m;
}

int lm_create_impl(fi_lm* m, const float* E, const float* Wlm, const float* Win, const float* conv,
                   const float* W1, const float* W2, const float* filters) {
    const int M = m->M, B = m->B, D = m->D, V = m->V;
    fi_ctx* c = new fi_ctx();
    m->mix = c;
    c->M = M;
    c->B = B;
    c->D = D;
    c->L = m->L;
    c->G = (long long)B * D;
    while ((1 << c->P) < c->L) ++c->P;
    int rc = create_impl(c, filters);
    if (rc) return rc;
    if ((rc = dev_alloc(c, &c->yout, (size_t)M * c->G * c->L))) return rc;
    if ((rc = lm_gemv_attrs<kLmStore, 1, 2>()) || (rc = lm_gemv_attrs<kLmStore, 2, 2>()) || (rc = lm_gemv_attrs<kLmMix, 1, 3>()) || (rc = lm_gemv_attrs<kLmMix, 2, 3>()) ||
        (rc = lm_gemv_attrs<kLmGelu, 1, 2>()) || (rc = lm_gemv_attrs<kLmAdd, 4, 2>()) ||
        (rc = lm_gemv_attrs<kLmArgmax, 1, 4>()))
        return rc;
    const size_t DD = (size_t)D * D;
    if ((rc = lm_upload_bf16(m, E, (size_t)V * D, &m->E))) return rc;
    if ((rc = lm_upload_bf16(m, Wlm, (size_t)V * D, &m->Wlm))) return rc;
    if ((rc = lm_upload_bf16(m, Win, (size_t)M * 3 * DD, &m->Win))) return rc;
    if ((rc = lm_upload_bf16(m, W1, (size_t)M * 4 * DD, &m->W1))) return rc;
    if ((rc = lm_upload_bf16(m, W2, (size_t)M * 4 * DD, &m->W2))) return rc;
    if ((rc = lm_alloc(m, &m->conv, (size_t)M * 9 * D))) return rc;
    CK(cudaMemcpy(m->conv, conv, sizeof(float) * M * 9 * D, cudaMemcpyDefault));
    if ((rc = lm_alloc(m, &m->u, (size_t)B * D))) return rc;
    if ((rc = lm_alloc(m, &m->z, (size_t)B * 3 * D))) return rc;
    if ((rc = lm_alloc(m, &m->zr, (size_t)M * 2 * B * 3 * D))) return rc;
    if ((rc = lm_alloc(m, &m->m1, (size_t)B * 4 * D))) return rc;
    if ((rc = lm_alloc(m, &m->r, (size_t)B * D))) return rc;
    if ((rc = lm_alloc(m, &m->tok, (size_t)B))) return rc;
    if ((rc = lm_alloc(m, &m->next, (size_t)B))) return rc;
    if ((rc = lm_alloc(m, &m->amax, (size_t)B))) return rc;
    CK(cudaDeviceSynchronize());
    return FI_OK;
}

}  // namespace

extern "C" {

const char* fi_last_error(void) { return g_err; }

const char* fi_version(void) { return "fi-b200 0.1 (sm_100a)"; }

fi_ctx* fi_create(int layers, int B, int D, int L, const float* filters) {
    g_err[0] = 0;
    if (layers < 1 || B < 1 || D < 1 || L < 2 || (L & (L - 1)) || !filters) {
        set_err(FI_EINVAL, "fi_create: need layers, B, D >= 1, L a power of two >= 2, filters != NULL "
                           "(got %d, %d, %d, %d, %p)", layers, B, D, L, (const void*)filters);
        return nullptr;
    }
    const long long G = (long long)B * D;
    if (L > (1 << (kFftQMax + 1))) {
        set_err(FI_EINVAL, "fi_create: L = %d above %d, the longest sequence whose blocks the FFT tau serves",
                L, 1 << (kFftQMax + 1));
        return nullptr;
    }
    if ((long long)(layers + 1) * G * L > (1LL << 40)) {
        set_err(FI_EINVAL, "fi_create: buffers too large");
        return nullptr;
    }
    fi_ctx* c = new fi_ctx();
    c->M = layers;
    c->B = B;
    c->D = D;
    c->L = L;
    c->G = G;
    while ((1 << c->P) < L) ++c->P;
    int rc = create_impl(c, filters);
    if (rc) {
        std::string msg = g_err;
        free_ctx(c);
        cudaGetLastError();
        set_err(rc, "%s", msg.c_str());
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_live_mu);
    g_live.insert(c);
    return c;
}

void fi_destroy(fi_ctx* ctx) {
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        if (!ctx || !g_live.count(ctx)) return;
        g_live.erase(ctx);
    }
    free_ctx(ctx);
}

int fi_reset(fi_ctx* ctx) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    ctx->t = 0;
    return FI_OK;
}

static int run_call(fi_ctx* c, const float* x, int steps, float* out, int closed) {
    int rc = check_ctx(c);
    if (rc) return rc;
    if (steps < 0) return set_err(FI_EINVAL, "steps must be >= 0");
    if (c->t + steps > c->L)
        return set_err(FI_ECAPACITY, "t=%lld + steps=%d exceeds capacity L=%d", c->t, steps, c->L);
    if (steps == 0) return FI_OK;
    if (!out) return set_err(FI_EINVAL, "output pointer is NULL");
    if (!closed && !x) return set_err(FI_EINVAL, "input pointer is NULL");
    if (closed && !x && c->t == 0) return set_err(FI_EINVAL, "closed loop at t=0 needs x0");
    const long long G = c->G;
    const float* xd = x;
    float* od = out;
    const bool x_host = x && !is_device_ptr(x);
    const bool o_host = !is_device_ptr(out);
    if (x_host) {
        const size_t nx = closed ? (size_t)G : (size_t)G * steps;
        if ((rc = ensure_stage(c, &c->sx, &c->sx_n, nx))) return rc;
        CK(cudaMemcpyAsync(c->sx, x, nx * sizeof(float), cudaMemcpyHostToDevice, c->stream));
        xd = c->sx;
    }
    if (o_host) {
        if ((rc = ensure_stage(c, &c->sy, &c->sy_n, (size_t)G * steps))) return rc;
        od = c->sy;
    }
    rc = run(c, c->t, steps, xd, od, closed);
    if (rc) return rc;
    c->t += steps;
    if (o_host) {
        CK(cudaMemcpyAsync(out, od, sizeof(float) * G * steps, cudaMemcpyDeviceToHost, c->stream));
        CK(cudaStreamSynchronize(c->stream));
    }
    return FI_OK;
}

int fi_step(fi_ctx* ctx, const float* x_t, float* y_t) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (!x_t || !y_t) return set_err(FI_EINVAL, "fi_step: x_t and y_t must be non-NULL");
    // one token: the per-token sequence is the natural form
    const int saved = ctx->path;
    ctx->path = FI_PATH_TOKEN;
    rc = run_call(ctx, x_t, 1, y_t, 0);
    ctx->path = saved;
    return rc;
}

int fi_generate(fi_ctx* ctx, const float* x0, int steps, float* out) { return run_call(ctx, x0, steps, out, 1); }

int fi_forward(fi_ctx* ctx, const float* x, int steps, float* y) { return run_call(ctx, x, steps, y, 0); }

int fi_prefill(fi_ctx* ctx, const float* x, int p, float* y) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (ctx->t != 0) return set_err(FI_EINVAL, "fi_prefill starts a sequence: call it at t = 0 (fi_reset)");
    if (p < 1 || p > ctx->L) return set_err(FI_EINVAL, "fi_prefill: need 1 <= p <= L = %d", ctx->L);
    if (p > (1 << kFftQMax))
        return set_err(FI_EINVAL, "fi_prefill: p = %d above %d, the longest prompt one FFT convolution serves",
                       p, 1 << kFftQMax);
    if (!x || !y) return set_err(FI_EINVAL, "fi_prefill: x and y must be non-NULL");
    if (ctx->path >= FI_PATH_LAZY) return set_err(FI_EINVAL, "fi_prefill serves the tiled paths only");
    if (p < (1 << kFftQMin)) return run_call(ctx, x, p, y, 0);  // a few tokens: the online path
    const long long G = ctx->G;
    const float* xd = x;
    float* yd = y;
    const bool x_host = !is_device_ptr(x), y_host = !is_device_ptr(y);
    if (x_host) {
        if ((rc = ensure_stage(ctx, &ctx->sx, &ctx->sx_n, (size_t)G * p))) return rc;
        CK(cudaMemcpyAsync(ctx->sx, x, sizeof(float) * G * p, cudaMemcpyHostToDevice, ctx->stream));
        xd = ctx->sx;
    }
    if (y_host) {
        if ((rc = ensure_stage(ctx, &ctx->sy, &ctx->sy_n, (size_t)G * p))) return rc;
        yd = ctx->sy;
    }
    if ((rc = prefill_impl(ctx, xd, p, yd))) return rc;
    ctx->t = p;
    if (y_host) {
        CK(cudaMemcpyAsync(y, yd, sizeof(float) * G * p, cudaMemcpyDeviceToHost, ctx->stream));
        CK(cudaStreamSynchronize(ctx->stream));
    }
    return FI_OK;
}

int fi_read_layer(fi_ctx* ctx, int layer, int t0, int t1, float* dst) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (layer < 0 || layer > ctx->M || t0 < 0 || t1 < t0 || t1 > ctx->t || !dst)
        return set_err(FI_EINVAL, "fi_read_layer: need 0 <= layer <= %d, 0 <= t0 <= t1 <= t=%lld", ctx->M,
                       ctx->t);
    if (t1 == t0) return FI_OK;
    const size_t n = (size_t)(t1 - t0) * ctx->G;
    const bool host = !is_device_ptr(dst);
    float* d = dst;
    if (host) {
        if ((rc = ensure_stage(ctx, &ctx->sy, &ctx->sy_n, n))) return rc;
        d = ctx->sy;
    }
    const int grid = (int)std::min<size_t>((n + 255) / 256, 65535);
    k_read_layer<<<grid, 256, 0, ctx->stream>>>(ctx->act, ctx->L, ctx->G, layer, t0, t1, d);
    CK(cudaGetLastError());
    if (host) {
        CK(cudaMemcpyAsync(dst, d, n * sizeof(float), cudaMemcpyDeviceToHost, ctx->stream));
        CK(cudaStreamSynchronize(ctx->stream));
    }
    return FI_OK;
}

int fi_set_stream(fi_ctx* ctx, void* stream) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    ctx->stream = (cudaStream_t)stream;
    return FI_OK;
}

int fi_set_path(fi_ctx* ctx, int path) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (path < FI_PATH_WINDOW || path > FI_PATH_EAGER_NP) return set_err(FI_EINVAL, "unknown path %d", path);
    if (path == FI_PATH_WINDOW && ctx->W == 0)
        return set_err(FI_EINVAL, "window path unavailable for this shape (shared memory)");
    const bool base_new = path >= FI_PATH_LAZY, base_old = ctx->path >= FI_PATH_LAZY;
    if (path != ctx->path && ctx->t != 0 && (base_new || base_old))
        return set_err(FI_EINVAL, "the lazy and eager paths keep their own state: switch to or from them at t = 0");
    if (base_new && base_old && path != ctx->path && ctx->t != 0)
        return set_err(FI_EINVAL, "switch between the baselines at t = 0");
    ctx->path = path;
    return FI_OK;
}

int fi_set_graphs(fi_ctx* ctx, int on) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    ctx->graphs = on ? 1 : 0;
    return FI_OK;
}

int fi_set_tau(fi_ctx* ctx, int q, int impl) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (q < 0 || q >= ctx->P) return set_err(FI_EINVAL, "block size 2^%d out of range", q);
    if (impl == FI_TAU_DIRECT && q > kDirectQMax)
        return set_err(FI_EINVAL, "direct tau limited to U <= %d", 1 << kDirectQMax);
    if (impl == FI_TAU_FFT && !ctx->spec[q]) return set_err(FI_EINVAL, "no spectrum for U = %d", 1 << q);
    if (impl != FI_TAU_AUTO && impl != FI_TAU_DIRECT && impl != FI_TAU_FFT)
        return set_err(FI_EINVAL, "unknown tau implementation %d", impl);
    ctx->tau_user[q] = impl;
    drop_graphs(ctx);
    return FI_OK;
}

int fi_get_info(const fi_ctx* ctx, fi_info* info) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (!info) return set_err(FI_EINVAL, "info is NULL");
    memset(info, 0, sizeof(*info));
    info->layers = ctx->M;
    info->B = ctx->B;
    info->D = ctx->D;
    info->L = ctx->L;
    info->t = (int)ctx->t;
    info->window = ctx->W;
    info->chains_per_cta = ctx->kch * ctx->B;
    info->path = ctx->path >= FI_PATH_LAZY ? ctx->path
                 : ((ctx->path == FI_PATH_WINDOW && ctx->W) ? FI_PATH_WINDOW : FI_PATH_TOKEN);
    info->graphs = ctx->graphs;
    for (int q = 0; q < ctx->P && q < 32; ++q) {
        info->tau[q] = tau_of(ctx, q);
        info->tau_us[q][0] = ctx->tau_us[q][0];
        info->tau_us[q][1] = ctx->tau_us[q][1];
    }
    info->device_bytes = ctx->bytes;
    info->sm_count = ctx->nsm;
    info->launches = ctx->launches;
    return FI_OK;
}

int fi_set_trace(fi_ctx* ctx, int on) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if ((on ? 1 : 0) != ctx->trace_on) drop_graphs(ctx);  // recapture with or without events
    ctx->trace_on = on ? 1 : 0;
    return FI_OK;
}

int fi_trace_read(fi_ctx* ctx, fi_trace* out) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (!out) return set_err(FI_EINVAL, "fi_trace_read: out is NULL");
    memset(out, 0, sizeof(*out));
    if (!ctx->last_trace) return FI_OK;
    CK(cudaStreamSynchronize(ctx->stream));
    for (const TraceRec& r : *ctx->last_trace) {
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, r.a, r.b));
        if (r.cls < 0 || r.cls >= FI_K_CLASSES) continue;
        out->launches[r.cls] += 1;
        out->total_us[r.cls] += 1000.0 * ms;
        if (1000.0 * ms > out->max_us[r.cls]) out->max_us[r.cls] = 1000.0 * ms;
        if (r.q >= 0 && r.q < 32) {
            out->block_launches[r.q] += 1;
            out->block_us[r.q] += 1000.0 * ms;
        }
    }
    return FI_OK;
}

int fi_trace_launches(fi_ctx* ctx, int max, int* cls, int* q, float* us) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (max < 0 || (max > 0 && (!cls || !q || !us)))
        return set_err(FI_EINVAL, "fi_trace_launches: need max >= 0 and non-NULL arrays");
    if (!ctx->last_trace) return 0;
    CK(cudaStreamSynchronize(ctx->stream));
    const int n = (int)ctx->last_trace->size();
    for (int i = 0; i < n && i < max; ++i) {
        const TraceRec& r = (*ctx->last_trace)[i];
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, r.a, r.b));
        cls[i] = r.cls;
        q[i] = r.q;
        us[i] = 1000.f * ms;
    }
    return n;
}

int fi_debug_schedule(const fi_ctx* ctx, int n, int* U, int* impl, int* src_lo, int* dst_lo, int* dst_hi) {
    int rc = check_ctx(ctx);
    if (rc) return rc;
    if (n < 1 || n > ctx->L - 1) return set_err(FI_EINVAL, "n must be in [1, L-1]");
    const long long u = lowbit(n);
    if (U) *U = (int)u;
    if (impl) *impl = tau_of(ctx, ctz64(n));
    if (src_lo) *src_lo = (int)(n - u);
    if (dst_lo) *dst_lo = n;
    if (dst_hi) *dst_hi = (int)std::min<long long>(n + u - 1, ctx->L - 1);
    return FI_OK;
}

int fi_tau(int impl, int U, int count, const float* blocks, const float* taps, int ldt, float* out,
           int accumulate) {
    if (U < 1 || (U & (U - 1)) || count < 1 || !blocks || !taps || !out || ldt < 2 * U)
        return set_err(FI_EINVAL, "fi_tau: need U a power of two, count >= 1, ldt >= 2U, non-NULL pointers");
    const int q = ctz64(U);
    if (impl != FI_TAU_DIRECT && impl != FI_TAU_FFT) return set_err(FI_EINVAL, "fi_tau: unknown impl %d", impl);
    if (impl == FI_TAU_DIRECT && q > kDirectQMax)
        return set_err(FI_EINVAL, "fi_tau: direct tau limited to U <= %d", 1 << kDirectQMax);
    if (impl == FI_TAU_FFT && (ldt & 1))
        return set_err(FI_EINVAL, "fi_tau: FFT tau reads taps in pairs; ldt must be even");
    if (impl == FI_TAU_FFT && (((uintptr_t)out & 15) || ((uintptr_t)blocks & 7) || ((uintptr_t)taps & 7)))
        return set_err(FI_EINVAL, "fi_tau: FFT tau needs out 16-byte and blocks, taps 8-byte aligned");
    if (impl == FI_TAU_FFT && (q < kFftQMin || q > kFftQMax))
        return set_err(FI_EINVAL, "fi_tau: FFT tau needs %d <= U <= %d", 1 << kFftQMin, 1 << kFftQMax);
    int rc = set_all_attrs();
    if (rc) return rc;
    fi_ctx tmp;  // holds this call's temporary allocations
    rc = tau_impl(&tmp, impl, U, q, count, blocks, taps, ldt, out, accumulate);
    cudaFree(tmp.tw);
    cudaFree(tmp.spec[0]);
    tmp.magic = 0;
    return rc;
}

int fi_tau_fft_noalloc(int U, int count, const float* blocks, const float* taps, int ldt, float* out,
                       int accumulate) {
    if (U < 1 || (U & (U - 1)) || count < 1 || !blocks || !taps || !out || ldt < 2 * U || (ldt & 1))
        return set_err(FI_EINVAL, "fi_tau_fft_noalloc: need U a power of two, count >= 1, ldt >= 2U and even, "
                                  "non-NULL pointers");
    if (((uintptr_t)out & 15) || ((uintptr_t)blocks & 7) || ((uintptr_t)taps & 7))
        return set_err(FI_EINVAL, "fi_tau_fft_noalloc: needs out 16-byte and blocks, taps 8-byte aligned");
    const int q = ctz64(U);
    if (q < kFftQMin || q > kNoAllocQMax)
        return set_err(FI_EINVAL, "fi_tau_fft_noalloc: U = %d outside [%d, %d], the largest block its fixed "
                                  "%zu-byte scratch serves", U, 1 << kFftQMin, 1 << kNoAllocQMax,
                       kNoAllocScratchBytes);
    int rc = set_all_attrs();
    if (rc) return rc;
    return tau_fft_noalloc_impl(U, q, count, blocks, taps, ldt, out, accumulate);
}


// ---------------------------------------------------------------- language model
fi_lm* fi_lm_create(int layers, int B, int D, int L, int V, const float* E, const float* W_lm, const float* W_in,
                    const float* conv, const float* W1, const float* W2, const float* filters) {
    g_err[0] = 0;
    if (layers < 1 || B < 1 || B > kLmMaxB || D < 8 || (D % 8) || L < 2 || (L & (L - 1)) || V < 1 || !E ||
        !W_lm || !W_in || !conv || !W1 || !W2 || !filters) {
        set_err(FI_EINVAL, "fi_lm_create: need layers >= 1, 1 <= B <= %d, D a multiple of 8, L a power of two "
                           ">= 2, V >= 1 and non-NULL weights", kLmMaxB);
        return nullptr;
    }
    if (L > (1 << (kFftQMax + 1))) {
        set_err(FI_EINVAL, "fi_lm_create: L = %d above %d", L, 1 << (kFftQMax + 1));
        return nullptr;
    }
    fi_lm* m = new fi_lm();
    m->M = layers;
    m->B = B;
    m->D = D;
    m->L = L;
    m->V = V;
    int rc = lm_create_impl(m, E, W_lm, W_in, conv, W1, W2, filters);
    if (rc) {
        std::string msg = g_err;
        lm_free(m);
        cudaGetLastError();
        set_err(rc, "%s", msg.c_str());
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_lm_mu);
    g_lm_live.insert(m);
    return m;
}

void fi_lm_destroy(fi_lm* m) {
    {
        std::lock_guard<std::mutex> lk(g_lm_mu);
        if (!m || !g_lm_live.count(m)) return;
        g_lm_live.erase(m);
    }
    lm_free(m);
}

int fi_lm_reset(fi_lm* m) {
    int rc = check_lm(m);
    if (rc) return rc;
    m->t = 0;
    m->mix->t = 0;
    return FI_OK;
}

int fi_lm_forward(fi_lm* m, const int* tokens, int steps, float* logits, int* next) {
    int rc = check_lm(m);
    if (rc) return rc;
    if (!tokens && steps > 0) return set_err(FI_EINVAL, "fi_lm_forward: tokens is NULL");
    return lm_run(m, tokens, nullptr, steps, logits, next);
}

int fi_lm_generate(fi_lm* m, const int* tok0, int steps, int* next) {
    int rc = check_lm(m);
    if (rc) return rc;
    return lm_run(m, nullptr, tok0, steps, nullptr, next);
}

int fi_lm_set_graphs(fi_lm* m, int on) {
    int rc = check_lm(m);
    if (rc) return rc;
    m->graphs = on ? 1 : 0;
    return FI_OK;
}

int fi_lm_set_trace(fi_lm* m, int on) {
    int rc = check_lm(m);
    if (rc) return rc;
    m->trace_on = on ? 1 : 0;
    if (!on) lm_clear_trace(m);
    return FI_OK;
}

int fi_lm_split(fi_lm* m, double* mixer_us, double* total_us) {
    int rc = check_lm(m);
    if (rc) return rc;
    if (!mixer_us || !total_us) return set_err(FI_EINVAL, "fi_lm_split: NULL output");
    *mixer_us = *total_us = 0.0;
    if (m->ev_call0 < 0 || m->ev_call1 < 0) return FI_OK;
    CK(cudaStreamSynchronize(m->mix->stream));
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, m->ev[m->ev_call0], m->ev[m->ev_call1]));
    *total_us = 1000.0 * ms;
    double blocks = 0.0, steps = 0.0;
    for (auto& pr : m->ev_blocks) {
        CK(cudaEventElapsedTime(&ms, m->ev[pr.first], m->ev[pr.second]));
        blocks += 1000.0 * ms;
    }
    for (auto& pr : m->ev_steps) {
        CK(cudaEventElapsedTime(&ms, m->ev[pr.first], m->ev[pr.second]));
        steps += 1000.0 * ms;
    }
    const double scale = m->sampled_tokens ? (double)m->traced_tokens / (double)m->sampled_tokens : 0.0;
    *mixer_us = blocks + steps * scale;
    return FI_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- data-dependent filter
// The long convolution with a filter that arrives online with the data (fi.h,
// fi_dd_create): red cells per step (k_dd_step, which also adds the blocks of U <= 8
// on the direct tau; k_dd_window for a whole aligned window given at once), then the
// larger blocks released after the step's token: two of the same size U = lowbit(n) at a step n that is not a power of
// two (x against rho's prefix, rho against x's prefix), one at n = U (x against rho
// with its unknown tail still zero).  The FFT form uses the spectra of the prefixes
// x[0, 2U) and rho[0, 2U), made at step 2U; the power-of-two block uses the spectrum
// of rho[0, 2U) made at its own step.

constexpr unsigned kDdMagic = 0xDD5EED01u;

struct fi_dd {
    unsigned magic = kDdMagic;
    fi_ctx* c = nullptr;                 // device, stream, twiddles, allocation count
    int G = 0, L = 0, P = 0;
    long long t = 0;
    float *xb = nullptr, *rb = nullptr;  // [G][L]: x and rho as they arrive (zero beyond t)
    float* acc = nullptr;                // [G][L]: running sums of the products i, j >= 1
    float2* spx[32] = {};                // per q: spectra of x[0, 2^(q+1)), stride 2^q + 2
    float2* spr[32] = {};                // per q: spectra of rho[0, 2^(q+1))
    float2* spz = nullptr;               // spectra of rho[0, 2U) at the power-of-two step U
    int tau_user[32] = {};
    float* stage = nullptr;              // host arrays staged on the device
    size_t stage_n = 0;
};

namespace {

std::mutex g_dd_mu;
std::set<const fi_dd*> g_dd_live;

int check_dd(const fi_dd* d) {
    std::lock_guard<std::mutex> lk(g_dd_mu);
    if (!d || !g_dd_live.count(d) || d->magic != kDdMagic) return set_err(FI_ESTATE, "null or destroyed context");
    return FI_OK;
}

// Blocks of size 2^q: the direct tau up to U = 8 (one thread per tile), the FFT tau
// above, unless set otherwise.
int dd_tau(const fi_dd* d, int q) {
    if (d->tau_user[q]) return d->tau_user[q];
    return q <= 3 ? FI_TAU_DIRECT : FI_TAU_FFT;
}

// Algorithm 1's block released after the n-th token over all channels: input x (or
// rho) at [n - U, n), taps rho (or x) from index 0, added onto the running sums.
int dd_block(fi_dd* d, long long n, bool x_input, const float2* spec, cudaStream_t st) {
    TileArgs a;
    memset(&a, 0, sizeof(a));
    a.act = x_input ? d->xb : d->rb;
    a.act_out = d->acc;
    a.h = x_input ? d->rb : d->xb;
    a.L = d->L;
    a.G = d->G;
    a.D = d->G;
    a.n = n;
    a.U = (int)lowbit(n);
    a.count = d->G;
    a.overwrite = 0;
    a.tw = d->c->tw;
    a.twlog = kTwLog;
    const int q = ctz64(n);
    if (dd_tau(d, q) == FI_TAU_DIRECT) return launch_direct_tile(a, st);
    a.spec = spec;
    a.spec_stride = fused_stride(a.U);
    return launch_fft(q, a, st);
}

// The blocks released after the n-th token (n < L): two of size U = lowbit(n), or at a
// power of two one, preceded by the spectra that become final there.
int dd_release(fi_dd* d, long long n, cudaStream_t st) {
    const int G = d->G;
    const long long L = d->L;
    const int q = ctz64(n);
    int rc;
    if (is_pow2(n)) {
        // the prefixes of length n are final: spectra for the blocks of size n / 2
        // still to come (steps 3n/2, 5n/2, ...)
        if (q >= 1) {
            const int q2 = q - 1;
            if (dd_tau(d, q2) == FI_TAU_FFT && (3LL << q2) < L) {
                if ((rc = make_spectra(q2, d->xb, L, G, d->spx[q2], d->c->tw, st))) return rc;
                if ((rc = make_spectra(q2, d->rb, L, G, d->spr[q2], d->c->tw, st))) return rc;
            }
        }
        if (dd_tau(d, q) == FI_TAU_FFT && (rc = make_spectra(q, d->rb, L, G, d->spz, d->c->tw, st))) return rc;
        return dd_block(d, n, true, d->spz, st);
    }
    if ((rc = dd_block(d, n, true, d->spr[q], st))) return rc;
    return dd_block(d, n, false, d->spx[q], st);
}

// Steps d->t .. d->t + steps - 1.  A whole aligned window of kDdWin steps at kW >= kDdWin
// runs as one k_dd_window launch (the blocks of U < kDdWin inside it folded in), then
// the blocks released at its end; every other step runs on its own (k_dd_step, with
// the blocks of U <= 8 inside it), then its larger blocks.
int dd_run(fi_dd* d, const float* x, const float* rho, int steps, float* y, cudaStream_t st) {
    const int G = d->G;
    const long long L = d->L;
    constexpr int W = kDdWin;
    int rc;
    const long long t0 = d->t, t_end = d->t + steps;
    long long t = t0;
    while (t < t_end) {
        const size_t k = (size_t)(t - t0);
        const float *xk = x + k * G, *rk = rho + k * G;
        float* yk = y + k * G;
        if (t >= W && t % W == 0 && t + W <= t_end) {
            k_dd_window<W><<<(G + kDdWinCh - 1) / kDdWinCh, 256, dd_window_smem<W>(), st>>>(d->xb, d->rb, d->acc, xk,
                                                                                          rk, yk, t, G, L);
            CK(cudaGetLastError());
            if (t + W < L && (rc = dd_release(d, t + W, st))) return rc;
            t += W;
            continue;
        }
        const long long n = t + 1;
        const int q = n < L ? ctz64(n) : -1;
        // blocks of U <= 8 on the direct tau run inside the step kernel
        const int fused = (q >= 0 && q <= 3 && dd_tau(d, q) == FI_TAU_DIRECT) ? (1 << q) : 0;
        const dim3 grid((G + 127) / 128), blk(128);
        switch (fused) {
            case 1: k_dd_step<1><<<grid, blk, 0, st>>>(d->xb, d->rb, d->acc, xk, rk, yk, t, G, L); break;
            case 2: k_dd_step<2><<<grid, blk, 0, st>>>(d->xb, d->rb, d->acc, xk, rk, yk, t, G, L); break;
            case 4: k_dd_step<4><<<grid, blk, 0, st>>>(d->xb, d->rb, d->acc, xk, rk, yk, t, G, L); break;
            case 8: k_dd_step<8><<<grid, blk, 0, st>>>(d->xb, d->rb, d->acc, xk, rk, yk, t, G, L); break;
            default: k_dd_step<0><<<grid, blk, 0, st>>>(d->xb, d->rb, d->acc, xk, rk, yk, t, G, L); break;
        }
        CK(cudaGetLastError());
        if (n < L && !fused && (rc = dd_release(d, n, st))) return rc;
        ++t;
    }
    return FI_OK;
}

void dd_free(fi_dd* d) {
    if (!d) return;
    if (d->c) cudaStreamSynchronize(d->c->stream);
    cudaFree(d->xb);
    cudaFree(d->rb);
    cudaFree(d->acc);
    for (int q = 0; q < 32; ++q) {
        cudaFree(d->spx[q]);
        cudaFree(d->spr[q]);
    }
    cudaFree(d->spz);
    cudaFree(d->stage);
    free_ctx(d->c);
    d->magic = 0;
    delete d;
}

int dd_create_impl(fi_dd* d) {
    int rc = set_all_attrs();
    if (rc) return rc;
    CK(cudaFuncSetAttribute(k_dd_window<kDdWin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)dd_window_smem<kDdWin>()));
    fi_ctx* c = new fi_ctx();
    d->c = c;
    CK(cudaGetDevice(&c->dev));
    CK(cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, c->dev));
    if ((rc = upload_twiddles(c))) return rc;
    const size_t GL = (size_t)d->G * d->L;
    if ((rc = dev_alloc(c, &d->xb, GL)) || (rc = dev_alloc(c, &d->rb, GL)) || (rc = dev_alloc(c, &d->acc, GL)))
        return rc;
    // prefix spectra for every size of the blocks at steps that are not powers of two
    // (3U < L), the power-of-two block's spectrum for U up to L / 2
    for (int q = kFftQMin; q <= d->P - 2; ++q) {
        const size_t n = (size_t)d->G * fused_stride(1LL << q);
        if ((rc = dev_alloc(c, &d->spx[q], n)) || (rc = dev_alloc(c, &d->spr[q], n))) return rc;
    }
    if (d->P - 1 >= kFftQMin && (rc = dev_alloc(c, &d->spz, (size_t)d->G * fused_stride(1LL << (d->P - 1)))))
        return rc;
    CK(cudaMemset(d->xb, 0, GL * sizeof(float)));
    CK(cudaMemset(d->rb, 0, GL * sizeof(float)));
    CK(cudaMemset(d->acc, 0, GL * sizeof(float)));
    CK(cudaDeviceSynchronize());
    return FI_OK;
}

// A host array of n floats on the device (device arrays pass through).
int dd_stage(fi_dd* d, const float* src, size_t n, size_t off, const float** out, cudaStream_t st) {
    if (is_device_ptr(src)) {
        *out = src;
        return FI_OK;
    }
    CK(cudaMemcpyAsync(d->stage + off, src, n * sizeof(float), cudaMemcpyHostToDevice, st));
    *out = d->stage + off;
    return FI_OK;
}

}  // namespace

extern "C" {

fi_dd* fi_dd_create(int G, int L) {
    g_err[0] = 0;
    if (G < 1 || L < 2 || (L & (L - 1)) || L > (1 << kFftQMax)) {
        set_err(FI_EINVAL, "fi_dd_create: need G >= 1 and L a power of two in [2, %d] (G=%d, L=%d)",
                1 << kFftQMax, G, L);
        return nullptr;
    }
    fi_dd* d = new fi_dd();
    d->G = G;
    d->L = L;
    while ((1 << d->P) < L) ++d->P;
    const int rc = dd_create_impl(d);
    if (rc) {
        const std::string msg = g_err;
        dd_free(d);
        cudaGetLastError();
        set_err(rc, "%s", msg.c_str());
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_dd_mu);
    g_dd_live.insert(d);
    return d;
}

void fi_dd_destroy(fi_dd* d) {
    {
        std::lock_guard<std::mutex> lk(g_dd_mu);
        if (!d || !g_dd_live.count(d)) return;
        g_dd_live.erase(d);
    }
    dd_free(d);
}

int fi_dd_reset(fi_dd* d) {
    int rc = check_dd(d);
    if (rc) return rc;
    const size_t GL = (size_t)d->G * d->L;
    cudaStream_t st = d->c->stream;
    CK(cudaMemsetAsync(d->xb, 0, GL * sizeof(float), st));
    CK(cudaMemsetAsync(d->rb, 0, GL * sizeof(float), st));
    CK(cudaMemsetAsync(d->acc, 0, GL * sizeof(float), st));
    CK(cudaStreamSynchronize(st));
    d->t = 0;
    return FI_OK;
}

int fi_dd_set_tau(fi_dd* d, int q, int impl) {
    int rc = check_dd(d);
    if (rc) return rc;
    if (q < 0 || q >= d->P) return set_err(FI_EINVAL, "fi_dd_set_tau: q=%d outside [0, %d)", q, d->P);
    if (impl != FI_TAU_AUTO && impl != FI_TAU_DIRECT && impl != FI_TAU_FFT)
        return set_err(FI_EINVAL, "fi_dd_set_tau: unknown implementation %d", impl);
    if (impl == FI_TAU_DIRECT && q > kDirectQMax)
        return set_err(FI_EINVAL, "fi_dd_set_tau: the direct tau serves U <= %d", 1 << kDirectQMax);
    if (impl == FI_TAU_FFT && q < kFftQMin)
        return set_err(FI_EINVAL, "fi_dd_set_tau: the FFT tau serves U >= %d", 1 << kFftQMin);
    if (d->t > 0) return set_err(FI_ESTATE, "fi_dd_set_tau: only before the first step (t=%lld)", d->t);
    d->tau_user[q] = impl;
    return FI_OK;
}

int fi_dd_forward(fi_dd* d, const float* x, const float* rho, int steps, float* y) {
    int rc = check_dd(d);
    if (rc) return rc;
    if (steps < 0) return set_err(FI_EINVAL, "steps must be >= 0");
    if (d->t + steps > d->L)
        return set_err(FI_ECAPACITY, "t=%lld + steps=%d exceeds capacity L=%d", d->t, steps, d->L);
    if (steps == 0) return FI_OK;
    if (!x || !rho || !y) return set_err(FI_EINVAL, "fi_dd_forward: NULL array");
    const size_t n = (size_t)steps * d->G;
    const bool xh = !is_device_ptr(x), rh = !is_device_ptr(rho), yh = !is_device_ptr(y);
    const size_t need = n * ((xh ? 1 : 0) + (rh ? 1 : 0) + (yh ? 1 : 0));
    if (need > d->stage_n) {
        cudaFree(d->stage);
        d->stage = nullptr;
        d->stage_n = 0;
        if ((rc = dev_alloc(d->c, &d->stage, need))) return rc;
        d->stage_n = need;
    }
    cudaStream_t st = d->c->stream;
    size_t off = 0;
    const float *xd = nullptr, *rd = nullptr;
    if ((rc = dd_stage(d, x, n, off, &xd, st))) return rc;
    off += xh ? n : 0;
    if ((rc = dd_stage(d, rho, n, off, &rd, st))) return rc;
    off += rh ? n : 0;
    float* yd = yh ? d->stage + off : y;
    if ((rc = dd_run(d, xd, rd, steps, yd, st))) return rc;
    d->t += steps;
    if (yh) CK(cudaMemcpyAsync(y, yd, n * sizeof(float), cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    return FI_OK;
}

}  // extern "C"

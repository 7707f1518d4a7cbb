"""Benchmark: closed-loop generation through the mixer stack (mixer tokens/s).

One "step" = one whole L-token closed-loop generation (fi_reset + fi_generate from
t = 0) of the stack of 18 long-convolution layers, B=1, D=864, L=2^17, fp32,
synthetic seeded filters: every block, red cell, sampler and tanh of the path runs
inside it.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank generates its own sequence
(independent start token) with the same model; no data-path collective.  Weak
scaling; value = all ranks' tokens / max-over-ranks time.
--impl reference times the CPU oracle (plain fp64 lazy evaluation) on the host.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "mixer tokens/s (B·L/time) at 18L×D864×L=2^17; % of HBM/fp32 roofline"
WORKLOADS = {
    # name: (layers, B, D, L)
    "headline": (18, 1, 864, 1 << 17),
    "hyena_shape": (18, 4, 768, 1 << 15),
    "tiny": (1, 1, 16, 1 << 10),
    # the headline stack at a shorter length: a few GB on the device, every launch
    # still larger than L2 (used for profiler captures)
    "short": (18, 1, 864, 1 << 14),
    # the headline length with fewer channels: every block size up to 2^16 in a few GB
    # (used for profiler captures of the largest blocks)
    "narrow": (18, 1, 96, 1 << 17),
}
FALLBACK_HBM_GBS = 6650.0
FP32_LANES_PER_SM = 128


# ------------------------------------------------------------------ cost model
def model_bytes_flops(M, B, D, L):
    """Algorithmic work of one L-token generation (whole stack).

    Per (layer, channel) and tile of edge U: block read B*U, output read-modify-write
    2*B*U, taps or spectrum 2U (shared over the batch), all fp32; per token the red
    cell reads/writes 2B+1 values.  FLOPs per tile and batch row: the cheaper of the
    direct 2U^2 and two real 2U-point FFTs (2.5 N log2 N each) + complex product +
    accumulate; per token 2 flops of red cell."""
    P = L.bit_length() - 1
    byts = 0
    flops = 0
    for q in range(P):
        U = 1 << q
        ntile = 1 << (P - 1 - q)
        byts += ntile * 4 * (3 * B * U + 2 * U)
        flops += ntile * B * min(2 * U * U, 10 * U * math.log2(2 * U) + 6 * (U + 1) + U)
    byts += L * 4 * (2 * B + 1)
    flops += B * 2 * L
    return byts * M * D, flops * M * D


def level_bytes(M, B, D, L, q):
    """Algorithmic bytes of one launch of the blocks of edge 2^q (all layers/channels)."""
    U = 1 << q
    return M * D * 4 * (3 * B * U + 2 * U)


def window_bytes(M, B, D, L, W):
    """Algorithmic bytes of one window-kernel launch: W tokens of red cells plus every
    block of edge < W released inside the window (same per-tile model)."""
    w = W.bit_length() - 1
    per_token = w * 2 * (3 * B + 2) + 4 * (2 * B + 1)
    return M * D * W * per_token


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for f in ("fi_kernels.cuh", "fi_fft.cuh", "fi_cluster.cuh"):
        h.update((ROOT / "long_convolution_sequence_b200" / "csrc" / f).read_bytes())
    return h.hexdigest()


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the ncu capture summarised under
    profiles/, or None when there is none or the kernel sources changed since."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    if d.get("kernel_sources_sha256") != kernel_sources_sha256():
        return None
    return d.get("per_launch_bytes", {}).get(kernel)


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        mhz = d.get("sm_max_mhz", 1965.0)
        return d["hbm_gbs"], "measured", mhz
    return FALLBACK_HBM_GBS, "fallback", 1965.0


# ------------------------------------------------------------------ clocks
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = Path("/tmp/fi_bench_clocks_%d.csv" % os.getpid())

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in self.path.read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        self.path.unlink(missing_ok=True)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(h, x0, T_s, G_s, M, B, D, L):
    """Time the fp64 lazy oracle on G_s chains (channels 0..G_s-1 of batch row 0), all
    layers, the first T_s closed-loop tokens; return (tokens/s for the whole workload,
    seconds, description).  The lazy oracle's work is M * chains * T(T+1)/2 MACs, so
    the whole-workload time is the measured time scaled by that count."""
    import oracle
    hs = np.ascontiguousarray(h[:, :G_s, :T_s])
    xs = np.ascontiguousarray(x0[:1, :G_s])
    t0 = time.perf_counter()
    oracle.stack(hs, xs, T=T_s, closed_loop=True, want=("y_last",))
    sec = time.perf_counter() - t0
    full = sec * (B * D / G_s) * (L * (L + 1) / 2) / (T_s * (T_s + 1) / 2)
    desc = ("%d chains x %d layers x first %d of %d tokens, closed loop; time scaled by chains "
            "(x%g) and by the lazy cost T(T+1)/2 (x%.1f)" % (G_s, M, T_s, L, B * D / G_s,
                                                            (L * (L + 1)) / (T_s * (T_s + 1))))
    return B * L / full, sec, desc


def oracle_sample_size(M, L, budget_s=15.0, rate=1.0e9):
    T_s = int(math.sqrt(2 * budget_s * rate / M))
    T_s = 1 << max(8, min(L.bit_length() - 1, T_s.bit_length() - 1))
    return min(T_s, L)


# ------------------------------------------------------------------ ranks
def rank_seed(rank):
    """Seed of rank r's start token: every replica generates its own sequence."""
    return rank


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (every rank gets it); the identity at N=1."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, B, L, ms_max):
    """Whole-job throughput: the tokens all ranks generated over the slowest rank's time."""
    return world * B * L / (ms_max / 1000.0)


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-trace", action="store_true",
                    help="skip the extra traced step that times each kernel class")
    ap.add_argument("--path", choices=("window", "token"), default="window")
    ap.add_argument("--graphs", type=int, default=1)
    ap.add_argument("--sweep", action="store_true",
                    help="the configuration sweep (18 layers; B, D, L grids): one JSON line per point")
    ap.add_argument("--sweep-b", default="1,2,4,8")
    ap.add_argument("--sweep-d", default="256,512,768,1024")
    ap.add_argument("--sweep-l", default="12,14,16,18", help="log2 L values")
    ap.add_argument("--baseline", choices=("lazy", "eager", "lazy_np", "eager_np"),
                    help="time the pages' Lazy or Eager baseline on this device next to the tiled path "
                         "(default workload: short)")
    ap.add_argument("--ablation", choices=("layers", "graphs", "tau", "latency"),
                    help="the pages' ablations on this path: one across-layer block launch against M "
                         "per-layer launches, graphs on against off, Hybrid tau against FFT-only and "
                         "direct-only, the per-token latency distribution; one JSON line per variant")
    ap.add_argument("--baseline-workload", default="short", choices=sorted(WORKLOADS),
                    help="workload of --baseline (the O(L^2) baselines take minutes at the headline length)")
    ap.add_argument("--lm", action="store_true",
                    help="the Hyena-like language model end to end (18 layers, B=4, D=768, L=2^15, vocabulary "
                         "50257, greedy decoding): tokens/s and the mixer / non-mixer split")
    ap.add_argument("--lm-profile", type=int, default=0, metavar="N",
                    help="with --lm: generate the first N tokens from host launches, untimed (for ncu launch lists)")
    ap.add_argument("--prefill", default=None,
                    help="comma-separated prompt lengths: time fi_prefill against the online "
                         "teacher-forced path over the same prompt (headline stack)")
    ap.add_argument("--dd", action="store_true",
                    help="the long convolution with a data-dependent filter (18 x 864 channels, L=2^17, "
                         "both sequences online): channel-steps/s, against a fixed filter of the same shape")
    ap.add_argument("--dd-profile", action="store_true",
                    help="with --dd: one untimed pass of the workload (for ncu launch lists)")
    args = ap.parse_args()
    if args.dd:
        return bench_dd(args)
    if args.prefill:
        return bench_prefill(args)
    if args.sweep:
        return bench_sweep(args)
    if args.baseline:
        return bench_baseline(args)
    if args.ablation:
        return bench_ablation(args)
    if args.lm:
        return bench_lm(args)
    M, B, D, L = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from long_convolution_sequence_b200 import synth
    if args.impl == "reference":
        if rank != 0:
            return 0
        return bench_reference(args, M, B, D, L, synth)

    import torch
    import torch.distributed as dist
    import datetime
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    import long_convolution_sequence_b200 as fi

    t_setup = time.perf_counter()
    h = synth.filters(M, D, L, seed=0)
    x0 = synth.start_token(B, D, seed=rank_seed(rank))
    t_gen = time.perf_counter() - t_setup
    t0 = time.perf_counter()
    ctx = fi.FlashInference(M, B, D, L, h)
    t_create = time.perf_counter() - t0
    ctx.set_path(fi.FI_PATH_WINDOW if args.path == "window" else fi.FI_PATH_TOKEN)
    ctx.set_graphs(bool(args.graphs))
    trace = not args.no_trace
    ctx.set_trace(False)  # the timed steps run the plain graph; one traced step follows
    info = ctx.info()

    x0_d = torch.from_numpy(x0).cuda()
    out_d = torch.empty((L, B, D), device="cuda")

    def one_step():
        ctx.reset()
        ctx.generate(x0_d, L, out_d)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()

    clocks = Clocks(local)
    launches0 = ctx.info().launches
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        one_step()
    ev1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    launches = ctx.info().launches - launches0
    tr, perq = {}, {}
    if trace:
        # one more step with every launch bracketed by events (per-class device times)
        ctx.set_trace(True)
        one_step()
        torch.cuda.synchronize()
        tr, perq = ctx.trace(per_block_size=True)
    classes_q = {}
    for q in perq:
        impl = info.tau[q]
        name = ("block_direct" if impl == fi.FI_TAU_DIRECT else
                ("block_cluster" if q > int(os.environ.get("FI_FUSED_QMAX", "14")) else "block_fft"))
        classes_q.setdefault(name, set()).add(q)
    ms = max_over_ranks(ms, world, "cuda")

    # end to end through the public API: host (pinned) start token in, host result out
    x0_h = torch.from_numpy(x0).pin_memory()
    out_h = torch.empty((L, B, D), pin_memory=True)
    ctx.set_trace(False)
    ctx.reset()
    ctx.generate(x0_h, L, out_h)  # capture / warm
    e2e_steps = max(1, min(args.steps, 3))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        ctx.reset()
        ctx.generate(x0_h, L, out_h)
    e2e_sec = (time.perf_counter() - t0) / e2e_steps
    e2e_sec = max_over_ranks(e2e_sec, world, "cuda")
    finite = bool(np.isfinite(out_h.numpy()).all())

    if rank != 0:
        ctx.close()
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    hbm, peak_kind, sm_mhz = peaks()
    tokens = world * B * L
    value = job_tokens_per_s(world, B, L, ms)
    byts, flops = model_bytes_flops(M, B, D, L)
    fp32_peak = info.sm_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6
    t_roof = max(byts / (hbm * 1e9), flops / fp32_peak)

    roof = None
    if tr:
        # dominant kernel class by device time in the traced step
        dom = max(tr, key=lambda k: tr[k][1])
        n_l, tot_us, max_us = tr[dom]
        if dom == "window":
            per_launch = window_bytes(M, B, D, L, info.window)
            work = per_launch * n_l
            unit_desc = ("W=%d tokens x (red cells + blocks of edge < W) x %d layers x %d channels"
                         % (info.window, M, D))
        else:
            # block launches: algorithmic bytes of each block size launched in this class
            cls_q = {q: v for q, v in perq.items() if q in classes_q.get(dom, ())}
            work = sum(v[0] * level_bytes(M, B, D, L, q) for q, v in cls_q.items())
            per_launch = work / max(1, n_l)
            unit_desc = "blocks of edge 2^q for q in %s, every layer and channel" % sorted(cls_q)
        ach = work / (tot_us * 1e-6) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": recorded_traffic(dom), "kernel": dom,
                "launches_per_step": n_l, "avg_launch_us": round(tot_us / n_l, 2),
                "bytes_per_launch": int(per_launch), "per_launch_work": unit_desc,
                "peak_source": ("measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                                else "fallback 6.65 TB/s")}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        import oracle
        T_s = oracle_sample_size(M, L)
        G_s = min(B * D, max(1, oracle.num_threads()))
        val, sec, desc = time_oracle(h, x0, T_s, G_s, M, B, D, L)
        cpu = {"value": round(val, 3), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
               "sample": desc, "sample_seconds": round(sec, 2)}

    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic: seeded decaying-exponential random filters, N(0,1) start token",
        "config": {"workload": "closed-loop generation of %d tokens through %d long-convolution layers, "
                               "B=%d, D=%d, tanh block and sampler" % (L, M, B, D),
                   "layers": M, "B": B, "D": D, "L": L, "window": info.window,
                   "path": args.path, "graphs": bool(args.graphs),
                   "tau": {str(q): ("fft" if info.tau[q] == fi.FI_TAU_FFT else "direct")
                           for q in range(L.bit_length() - 1)},
                   "l2": "inputs larger than L2: %.1f GB of buffers, filters and spectra resident per GPU"
                         % (info.device_bytes / 1e9),
                   "parallelism": "replicas x%d (one sequence per GPU)" % world},
        "e2e": {"value": round(tokens / e2e_sec, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": B * D * 4, "d2h_bytes_per_step": L * B * D * 4},
        "gpu_launches": int(launches),
        "roofline": roof,
        "job_roofline": {"model_bytes": byts, "model_flops": flops, "t_roof_ms": round(t_roof * 1e3, 3),
                         "frac": round(t_roof * 1e3 / ms, 4), "hbm_gbs": hbm,
                         "fp32_tflops": round(fp32_peak / 1e12, 1),
                         "note": "time of the slower of model bytes at HBM peak and model FLOPs at fp32 peak, "
                                 "divided by the measured step time"},
        "cpu_baseline": cpu,
        "clocks": clk,
        "kernel_time_us": {k: round(v[1], 1) for k, v in tr.items()},
        "block_time_us": {str(q): round(v[1], 1) for q, v in sorted(perq.items())},
        "setup_s": {"filters": round(t_gen, 2), "create": round(t_create, 2)},
        "outputs_finite": finite,
        "context": "pages' figures (H100/A100, precision not stated): 110x mixer and 7.8x end-to-end "
                   "speedup over lazy inference",
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def sweep_need_bytes(M, B, D, L):
    """Device memory a sweep point needs: the context's filters plus their spectra
    (about 3 M D L floats), its halved-layout buffers ((M+1) B D L floats), and the
    device copy of the filters it is created from (M D L floats)."""
    return 4 * L * D * (4 * M + (M + 1) * B)


def sweep_filters(M, D, L, seed=0):
    """Filters of the sweep drawn on the device (synth.device_filters: the headline's
    law, h[c, k] = N(0,1) exp(-a_c k) / sqrt(32), a_c ~ U(0.001, 0.05), independent per
    layer, from torch's seeded CUDA generator): the 2^18-tap filters of the largest
    points would take minutes on the host."""
    from long_convolution_sequence_b200 import synth
    return synth.device_filters(M, D, L, seed=seed)


def bench_sweep(args):
    """Configuration sweep on the synthetic mixer stack: 18 layers, B, D, L over the
    given grids.  Per point: one warm-up and one timed closed-loop generation (CUDA
    events), the tile-size histogram of the schedule, and the tau implementation
    chosen per block size.  Points whose memory need exceeds the free device memory
    are reported as not fitting."""
    import torch
    import long_convolution_sequence_b200 as fi
    M = 18
    hbm, peak_kind, sm_mhz = peaks()
    names = {fi.FI_TAU_DIRECT: "direct", fi.FI_TAU_FFT: "fft"}
    for B in [int(v) for v in args.sweep_b.split(",")]:
        for D in [int(v) for v in args.sweep_d.split(",")]:
            for P in [int(v) for v in args.sweep_l.split(",")]:
                L = 1 << P
                line = {"metric": "sweep point: mixer tokens/s", "layers": M, "B": B, "D": D, "L": L}
                need = sweep_need_bytes(M, B, D, L)
                free, _ = torch.cuda.mem_get_info()
                if need > 0.85 * free:
                    line.update({"fits": False, "need_gb": round(need / 1e9, 1), "free_gb": round(free / 1e9, 1)})
                    print(json.dumps(line), flush=True)
                    continue
                h = sweep_filters(M, D, L)
                x0 = torch.from_numpy(synth_start(B, D)).cuda()
                t0 = time.perf_counter()
                ctx = fi.FlashInference(M, B, D, L, h)
                t_create = time.perf_counter() - t0
                del h
                torch.cuda.empty_cache()
                info = ctx.info()
                out = torch.empty((L, B, D), device="cuda")
                ctx.reset()
                ctx.generate(x0, L, out)
                ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ctx.reset()
                ev0.record()
                ctx.generate(x0, L, out)
                ev1.record()
                torch.cuda.synchronize()
                ms = ev0.elapsed_time(ev1)
                byts, flops = model_bytes_flops(M, B, D, L)
                fp32_peak = info.sm_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6
                t_roof = max(byts / (hbm * 1e9), flops / fp32_peak)
                cls = ["block_cluster" if q > int(os.environ.get("FI_FUSED_QMAX", "14")) and info.tau[q] == fi.FI_TAU_FFT
                       else names.get(info.tau[q], str(info.tau[q])) for q in range(P)]
                line.update({
                    "fits": True, "ms": round(ms, 3), "value": round(B * L / (ms / 1e3), 1),
                    "roofline_frac": round(t_roof * 1e3 / ms, 4),
                    "path": "window W=%d" % info.window if info.window else "per-token",
                    "tile_histogram": {str(1 << q): 1 << (P - 1 - q) for q in range(P)},
                    "tau": {str(1 << q): cls[q] for q in range(P)},
                    "create_s": round(t_create, 2), "device_gb": round(info.device_bytes / 1e9, 2),
                    "finite": bool(torch.isfinite(out).all().item()),
                })
                print(json.dumps(line), flush=True)
                ctx.close()
                del out
                torch.cuda.empty_cache()
    return 0


def bench_baseline(args):
    """One of the pages' Lazy or Eager baselines (FI_PATH_LAZY / FI_PATH_EAGER, parallel
    across layers, or their NP forms FI_PATH_LAZY_NP / FI_PATH_EAGER_NP) timed on this
    device beside the tiled window path, same workload, same process: one closed-loop
    generation each after warm-up, CUDA events.  The baselines cost O(L^2) per
    channel-layer; the default workload (--baseline-workload) is the headline stack at
    L = 2^14, where the line also carries the baseline's time scaled to L = 2^17 by the
    L^2 law (labelled as extrapolated); --baseline-workload headline measures it."""
    import torch
    import long_convolution_sequence_b200 as fi
    from long_convolution_sequence_b200 import synth
    wl = args.baseline_workload
    M, B, D, L = WORKLOADS[wl]
    h = synth.filters(M, D, L, seed=0)
    x0 = torch.from_numpy(synth.start_token(B, D, seed=0)).cuda()
    out = torch.empty((L, B, D), device="cuda")
    ctx = fi.FlashInference(M, B, D, L, h)

    def timed(n):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for _ in range(n):
            ctx.reset()
            ctx.generate(x0, L, out)
        ev1.record()
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1) / n

    timed(3)
    fi_ms = timed(3)
    ctx.reset()
    ctx.set_path({"lazy": fi.FI_PATH_LAZY, "eager": fi.FI_PATH_EAGER, "lazy_np": fi.FI_PATH_LAZY_NP,
                  "eager_np": fi.FI_PATH_EAGER_NP}[args.baseline])
    ctx.generate(x0, min(L, 256), out)  # warm-up of the baseline's kernels
    torch.cuda.synchronize()
    base_ms = timed(1)
    finite = bool(torch.isfinite(out).all().item())
    ctx.close()
    scale = (float(1 << 17) / L) ** 2
    line = {"metric": "mixer tokens/s (B*L/time), %s baseline on this device" % args.baseline,
            "impl": args.baseline + "_gpu", "value": round(B * L / (base_ms / 1e3), 1),
            "unit": "tokens/s", "ms_per_generation": round(base_ms, 3),
            "tiled_value": round(B * L / (fi_ms / 1e3), 1), "tiled_ms_per_generation": round(fi_ms, 3),
            "tiled_speedup": round(base_ms / fi_ms, 2),
            "extrapolated_ms_at_L_2^17": round(base_ms * scale, 1) if L < (1 << 17) else None,
            "finite": finite, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl, "layers": M, "B": B, "D": D, "L": L}}
    print(json.dumps(line), flush=True)
    return 0



def bench_ablation(args):
    """The pages' ablations ("Ablationsstudien", "Implementierungsdetails", "Antwortzeit
    pro Token") measured on this path, on the workload's stack (default: headline),
    closed loop from t = 0, CUDA events, one warm-up and two timed generations per
    variant; one JSON line per variant.

    layers:  every block launch covering all M layers (Algorithm 3) against M launches
             of one layer each (FI_LAYER_SPLIT=1), on the window and per-token paths;
    graphs:  captured CUDA graphs against launches issued from the host, both paths;
    tau:     the measured Hybrid choice against FFT for every size it serves (U >= 8)
             and direct for every size it serves (U <= 4096), both paths (on the window
             path every block smaller than W runs inside the window kernel, so tau only
             chooses among the larger sizes there);
    latency: device time per token from a traced generation: per-token path, each
             token's launches; window path, each window launch spread over its W tokens
             plus the block launch at the window's end on its last token."""
    import torch
    import long_convolution_sequence_b200 as fi
    from long_convolution_sequence_b200 import synth
    M, B, D, L = WORKLOADS[args.workload]
    h = synth.filters(M, D, L, seed=0)
    x0 = torch.from_numpy(synth.start_token(B, D, seed=0)).cuda()
    out = torch.empty((L, B, D), device="cuda")
    paths = {"window": fi.FI_PATH_WINDOW, "token": fi.FI_PATH_TOKEN}

    def timed(ctx, n=2):
        ctx.reset()
        ctx.generate(x0, L, out)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for _ in range(n):
            ctx.reset()
            ctx.generate(x0, L, out)
        ev1.record()
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1) / n

    def emit(variant, path, ms, **extra):
        line = {"metric": "ablation: mixer tokens/s", "ablation": args.ablation, "variant": variant,
                "path": path, "ms_per_generation": round(ms, 3), "value": round(B * L / (ms / 1e3), 1),
                "unit": "tokens/s", "finite": bool(torch.isfinite(out).all().item()),
                "config": {"workload": args.workload, "layers": M, "B": B, "D": D, "L": L}}
        line.update(extra)
        print(json.dumps(line), flush=True)

    if args.ablation == "layers":
        for split in (0, 1):
            os.environ["FI_LAYER_SPLIT"] = str(split)
            with fi.FlashInference(M, B, D, L, h) as ctx:
                for pname, path in paths.items():
                    ctx.set_path(path)
                    n0 = ctx.info().launches
                    ms = timed(ctx)
                    emit("per-layer block launches" if split else "one launch for all layers", pname, ms,
                         launches_per_generation=(ctx.info().launches - n0) // 3)
        os.environ.pop("FI_LAYER_SPLIT", None)
        return 0
    with fi.FlashInference(M, B, D, L, h) as ctx:
        info = ctx.info()
        P = L.bit_length() - 1
        if args.ablation == "graphs":
            for pname, path in paths.items():
                ctx.set_path(path)
                for graphs in (True, False):
                    ctx.set_graphs(graphs)
                    n0 = ctx.info().launches
                    ms = timed(ctx, 1)
                    emit("graphs on" if graphs else "graphs off", pname, ms,
                         launches_per_generation=(ctx.info().launches - n0) // 2)
            return 0
        if args.ablation == "tau":
            choices = {"hybrid (measured)": {},
                       "fft everywhere": {q: fi.FI_TAU_FFT for q in range(3, P)},
                       "direct everywhere": {q: fi.FI_TAU_DIRECT for q in range(0, min(P, 13))}}
            for pname, path in paths.items():
                ctx.set_path(path)
                for name, table in choices.items():
                    for q in range(P):
                        ctx.set_tau(q, fi.FI_TAU_AUTO)
                    for q, impl in table.items():
                        ctx.set_tau(q, impl)
                    tau = {str(q): ("fft" if ctx.info().tau[q] == fi.FI_TAU_FFT else "direct") for q in range(P)}
                    emit(name, pname, timed(ctx), tau=tau)
            for q in range(P):
                ctx.set_tau(q, fi.FI_TAU_AUTO)
            return 0
        # latency
        for pname, path in paths.items():
            ctx.set_path(path)
            ctx.set_trace(True)
            ctx.reset()
            ctx.generate(x0, L, out)
            torch.cuda.synchronize()
            cls, qs, us = ctx.trace_launches()
            per_tok = np.zeros(L)
            W = info.window
            if path == fi.FI_PATH_WINDOW:
                t = 0
                for c, q, u in zip(cls, qs, us):
                    if c == fi.FI_K_WINDOW:
                        per_tok[t:t + W] += u / W
                        t += W
                    else:  # the block released at the end of the window just done
                        per_tok[t - 1] += u
            else:
                t = -1
                for c, q, u in zip(cls, qs, us):
                    if c == fi.FI_K_TOKEN_STEP:
                        t += 1
                    per_tok[t] += u
            ctx.set_trace(False)
            n = np.arange(1, L + 1)
            lowq = np.array([(int(v) & -int(v)).bit_length() - 1 for v in n])
            by_q = {str(q): round(float(per_tok[lowq == q].mean()), 3) for q in range(P + 1) if (lowq == q).any()}
            pct = {p: round(float(np.percentile(per_tok, p)), 3) for p in (50, 90, 99, 99.9)}
            emit("per-token device time", pname, float(per_tok.sum()) / 1e3,
                 us_per_token={"mean": round(float(per_tok.mean()), 3), "percentiles": pct,
                               "max": round(float(per_tok.max()), 1),
                               "mean_by_released_block_log2": by_q},
                 note="time of one traced generation (events around every launch)")
        return 0


LM_CONFIG = dict(M=18, B=4, D=768, L=1 << 15, V=50257)


def lm_model_bytes(M, B, D, L, V):
    """Algorithmic bytes of one greedy generation of L tokens: per token the bf16
    weights each GEMV streams (W_in 3D x D, W1 4D x D, W2 D x 4D per layer, the LM head
    V x D) and the embedding rows (B x D), 2 bytes each; the mixers' blocks, 20U bytes
    per block and chain (4U(3B'+2) at one row per chain) over M x B x D chains, one block
    of U = lowbit(n) after token n; and per token and chain of every layer the mixer
    step's state (the short-convolution ring, the input and running sum, 40 bytes)."""
    weights = (M * (3 * D * D + 4 * D * D + 4 * D * D) + V * D + B * D) * 2
    G = B * D
    blocks = sum(20 * (n & -n) for n in range(1, L)) * M * G
    return L * weights + blocks + L * M * G * 40


def bench_lm(args):
    """The Hyena-like model end to end (BASELINE configuration 5): greedy generation of
    L tokens from uniform random start tokens, random-init weights (bf16 GEMMs, fp32
    mixer).  One warm-up generation, then timed generations (CUDA events); a traced
    generation gives the mixers' share of the device time (the pages' mixer / non-mixer
    split, section "Hauptergebnisse"); the oracle is timed on its first tokens."""
    import torch
    import long_convolution_sequence_b200 as fi
    from long_convolution_sequence_b200 import synth
    c = LM_CONFIG
    M, B, D, L, V = c["M"], c["B"], c["D"], c["L"], c["V"]
    t0 = time.perf_counter()
    p = synth.hyena_params(M, D, L, V, seed=0)
    t_gen = time.perf_counter() - t0
    tok0 = synth.token_ids(1, B, V, seed=0)[0]
    stack = lambda k: np.ascontiguousarray(np.stack(p[k]))
    lm = fi.LanguageModel(M, B, D, L, V, p["E"], p["W_lm"], stack("W_in"), stack("c"), stack("W1"), stack("W2"),
                          stack("h"))
    tok0_d = torch.from_numpy(tok0).cuda()
    if args.lm_profile:
        # a profiling workload, not a measurement: one generation of the first
        # lm_profile tokens, every kernel launched from the host (for ncu launch lists)
        lm.set_graphs(False)
        out = torch.empty((args.lm_profile, B), dtype=torch.int32, device="cuda")
        lm.generate(tok0_d, args.lm_profile, out)
        torch.cuda.synchronize()
        lm.close()
        print(json.dumps({"lm_profile_tokens": args.lm_profile, "last_choices": out[-1].tolist()}), flush=True)
        return 0
    nxt = torch.empty((L, B), dtype=torch.int32, device="cuda")

    def gen():
        lm.reset()
        lm.generate(tok0_d, L, nxt)

    gen()
    torch.cuda.synchronize()
    clocks = Clocks(0)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, min(args.steps, 2))
    ev0.record()
    h0 = time.perf_counter()
    for _ in range(steps):
        gen()
    host_ms = (time.perf_counter() - h0) * 1e3 / steps  # time to issue the work
    ev1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / steps
    lm.set_graphs(False)
    gen()
    ev0.record()
    h0 = time.perf_counter()
    gen()
    host_ms_eager = (time.perf_counter() - h0) * 1e3
    ev1.record()
    torch.cuda.synchronize()
    ms_eager = ev0.elapsed_time(ev1)
    lm.set_graphs(True)
    lm.set_trace(True)
    gen()
    torch.cuda.synchronize()
    mix_us, tot_us = lm.split()
    lm.set_trace(False)
    toks = nxt.cpu().numpy()
    # the oracle on a bounded sample: the first T_s tokens of this generation, fed back as
    # teacher tokens; the GPU's logits on the same tokens against the oracle's
    from oracle import hyena
    T_s = 8
    inputs = np.concatenate([tok0[None, :], toks[:T_s - 1]]).astype(np.int32)
    t1 = time.perf_counter()
    ref = hyena.run(p, tokens=inputs)
    sec = time.perf_counter() - t1
    lm.reset()
    lg = np.empty((T_s, B, V), np.float32)
    tf = np.empty((T_s, B), np.int32)
    lm.forward(inputs, T_s, lg, tf)
    lm.close()
    rms = float(np.sqrt(np.mean(ref["logits"] ** 2)))
    logit_err = float(np.abs(lg - ref["logits"]).max()) / rms
    hbm, src, _ = peaks()
    nbytes = lm_model_bytes(M, B, D, L, V)
    ach = nbytes / (ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
            "traffic": None, "kernel": "whole generation", "model_bytes": nbytes,
            "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)"}
    line = {"metric": "end-to-end tokens/s (B*L/time), Hyena-like model, greedy decoding", "value": round(B * L / (ms / 1e3), 1),
            "unit": "tokens/s", "ms_per_generation": round(ms, 1), "steps": steps, "dtype": "bf16 GEMMs / f32 mixer",
            "data": "synthetic: random-init weights, uniform random start tokens",
            "config": {"workload": "Hyena-like model, %d layers, B=%d, D=%d, L=%d, vocabulary %d" % (M, B, D, L, V),
                       **c},
            "mixer_share": {"mixer_us": round(mix_us, 1), "total_us": round(tot_us, 1),
                            "frac": round(mix_us / tot_us, 4) if tot_us else None,
                            "note": "traced generation: events around every block launch and the mixer steps of "
                                    "every 64th token (scaled)"},
            "host_issue_ms": round(host_ms, 1),
            "graphs_off": {"ms_per_generation": round(ms_eager, 1), "host_issue_ms": round(host_ms_eager, 1)},
            "roofline": roof,
            "oracle_check": {"tokens": T_s, "max_logit_err_over_rms": logit_err,
                             "bound": (3 * M + 1) * 2.0 ** -8,
                             "greedy_agree": int((tf == ref["next"]).sum()), "of": int(tf.size)},
            "cpu_baseline": {"value": round(B * T_s / sec, 3), "unit": "tokens/s", "kind": "oracle",
                             "cores": 1, "sample": "first %d tokens of the same generation (fp64 numpy)" % T_s},
            "clocks": clk, "setup_s": {"params": round(t_gen, 1)}}
    print(json.dumps(line), flush=True)
    return 0

DD_CONFIG = dict(G=18 * 864, L=1 << 17)


def dd_model_bytes(G, L):
    """Algorithmic bytes of one online pass of the data-dependent convolution: per
    channel, every block of size U moves 4U(3B+2) = 20U bytes at B = 1 (its U inputs,
    its taps' 2U values or their spectrum, U outputs read and written), two blocks at
    every step that is not a power of two; the red cell reads the running sum, x_0 and
    rho_0 and writes x_t, rho_t, y_t (24 bytes)."""
    total = 0
    for n in range(1, L):
        U = n & -n
        total += 20 * U * (1 if (n & (n - 1)) == 0 else 2)
    return G * (total + 24 * L)


def bench_dd(args):
    """The long convolution with a data-dependent filter (the pages' extension with
    two convolutions of the same size per step): one online pass of L steps over G
    channels, both sequences drawn on the device (synth.device_dd_inputs), every
    launch from the host, CUDA events around each pass.  Beside it the same shape with
    the filter fixed (rho of this draw as a precomputed filter) through Algorithm 1 on
    the per-token path with host launches: their ratio is the pages' factor of two.
    The oracle (fp64 causal convolution) on a bounded sample of channels and steps."""
    import torch
    import long_convolution_sequence_b200 as fi
    from long_convolution_sequence_b200 import synth
    G, L = DD_CONFIG["G"], DD_CONFIG["L"]
    x, rho = synth.device_dd_inputs(L, G, seed=0)
    y = torch.empty((L, G), device="cuda")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dd = fi.DataDependentConvolution(G, L)
    if args.dd_profile:
        # a profiling workload, not a measurement: one untimed pass (for ncu launch lists)
        dd.forward(x, rho, L, y)
        torch.cuda.synchronize()
        dd.close()
        print(json.dumps({"dd_profile_pass": True, "G": G, "L": L}), flush=True)
        return 0
    for _ in range(max(1, min(args.warmup, 1))):
        dd.reset()
        dd.forward(x, rho, L, y)
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 2))
    clocks = Clocks(0)
    clocks.start()
    ms = []
    for _ in range(steps):
        dd.reset()
        ev0.record()
        dd.forward(x, rho, L, y)
        ev1.record()
        torch.cuda.synchronize()
        ms.append(ev0.elapsed_time(ev1))
    clk = clocks.stop()
    t_dd = min(ms)
    # sampled parity of the timed pass: 4 channels over the first 4096 steps
    import oracle
    chans = [0, 1, G // 2, G - 1]
    Ts = 4096
    xs = x[:Ts, chans].cpu().numpy()
    rs = rho[:Ts, chans].cpu().numpy()
    ref = oracle.causal_conv_batch(np.ascontiguousarray(rs.T), np.ascontiguousarray(xs.T)).T
    got = y[:Ts, chans].cpu().numpy()
    err = float(np.abs(got - ref).max() / np.sqrt(np.mean(ref ** 2)))
    dd.close()
    del y
    torch.cuda.empty_cache()
    # the fixed filter of the same shape: one layer of G channels, filter = this rho
    h = rho.t().contiguous().view(1, G, L)
    ctx = fi.FlashInference(1, 1, G, L, h)
    del h
    torch.cuda.empty_cache()
    ctx.set_path(fi.FI_PATH_TOKEN)
    ctx.set_graphs(False)
    yy = torch.empty((L, 1, G), device="cuda")
    xv = x.view(L, 1, G)
    ctx.reset()
    ctx.forward(xv, L, yy)
    torch.cuda.synchronize()
    ctx.reset()
    ev0.record()
    ctx.forward(xv, L, yy)
    ev1.record()
    torch.cuda.synchronize()
    t_fixed = ev0.elapsed_time(ev1)
    ctx.close()
    # CPU oracle on a bounded sample: the lazy causal convolution of 16 channels over
    # the first T_s steps, scaled to G channels and L steps by the lazy cost T (T+1) / 2
    T_s = 1 << 14
    xc = x[:T_s, :16].cpu().numpy()
    rc = rho[:T_s, :16].cpu().numpy()
    t0 = time.perf_counter()
    oracle.causal_conv_batch(np.ascontiguousarray(rc.T), np.ascontiguousarray(xc.T))
    sec = time.perf_counter() - t0
    scale = (G / 16.0) * (L * (L + 1) / 2.0) / (T_s * (T_s + 1) / 2.0)
    hbm, src, _ = peaks()
    nbytes = dd_model_bytes(G, L)
    ach = nbytes / (t_dd / 1e3) / 1e9
    line = {"metric": "data-dependent filter: channel-steps/s (G*L/time), both sequences online",
            "value": round(G * L / (t_dd / 1e3), 1), "unit": "channel-steps/s", "ms_per_pass": round(t_dd, 2),
            "steps": steps, "higher_is_better": True, "dtype": "f32",
            "data": "synthetic: x ~ N(0,1), rho with the filters' law laid out by step (drawn on the device)",
            "config": {"workload": "data-dependent filter, %d channels (18 x 864), L=%d" % (G, L), "G": G, "L": L,
                       "launches": "host: each whole window of 128 steps one launch (its blocks below 128 folded "
                                   "in), then the blocks released at its end; the first window step by step"},
            "fixed_filter": {"ms_per_pass": round(t_fixed, 2), "path": "Algorithm 1, per-token path, host launches",
                             "ratio_dd_over_fixed": round(t_dd / t_fixed, 3),
                             "note": "not path for path: the data-dependent pass uses windows of given inputs"},
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": None, "kernel": "whole pass",
                         "model_bytes": nbytes, "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)"},
            "parity_sample": {"channels": chans, "steps": Ts, "max_err_over_rms": err},
            "cpu_baseline": {"value": round(G * L / (sec * scale), 3), "unit": "channel-steps/s", "kind": "oracle",
                             "cores": oracle.num_threads(),
                             "sample": "16 channels x first %d steps, lazy fp64, scaled by channels and T(T+1)/2" % T_s},
            "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def bench_prefill(args):
    """Prompt prefill (fi_prefill: one FFT convolution per layer) against the online
    teacher-forced path (fi_forward) over the same prompt, on the workload's stack; CUDA
    events, 2 warm-ups and 3 timed runs each; one JSON line per prompt length."""
    import torch
    import long_convolution_sequence_b200 as fi
    from long_convolution_sequence_b200 import synth
    M, B, D, L = WORKLOADS[args.workload]
    h = synth.filters(M, D, L, seed=0)
    ctx = fi.FlashInference(M, B, D, L, h)
    for p in [int(v) for v in args.prefill.split(",")]:
        x = torch.from_numpy(synth.inputs(p, B, D, seed=0)).cuda()
        y = torch.empty((p, B, D), device="cuda")

        def timed(fn, n=3):
            for _ in range(2):
                ctx.reset()
                fn()
            torch.cuda.synchronize()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            tot = 0.0
            for _ in range(n):
                ctx.reset()
                ev0.record()
                fn()
                ev1.record()
                torch.cuda.synchronize()
                tot += ev0.elapsed_time(ev1)
            return tot / n

        pre_ms = timed(lambda: ctx.prefill(x, p, y))
        y_pre = y.clone()
        on_ms = timed(lambda: ctx.forward(x, p, y))
        err = float((y_pre - y).abs().max() / y.pow(2).mean().sqrt())
        print(json.dumps({"metric": "prompt tokens/s", "prompt": p, "prefill_ms": round(pre_ms, 3),
                          "online_ms": round(on_ms, 3), "speedup": round(on_ms / pre_ms, 2),
                          "prefill_value": round(B * p / (pre_ms / 1e3), 1), "max_err_over_rms": err,
                          "config": {"workload": args.workload, "layers": M, "B": B, "D": D, "L": L}}), flush=True)
    ctx.close()
    return 0


def synth_start(B, D):
    from long_convolution_sequence_b200 import synth
    return synth.start_token(B, D, seed=0)


def bench_reference(args, M, B, D, L, synth):
    """The oracle as the reference arm: each step times a bounded sample of the same
    workload on the host cores and scales it to the metric's unit."""
    import oracle
    T_s = oracle_sample_size(M, L, budget_s=max(3.0, 60.0 / max(1, args.steps + args.warmup)))
    G_s = min(B * D, max(1, oracle.num_threads()))
    hs = np.ascontiguousarray(synth.filters(M, G_s, T_s, seed=0))
    x0 = synth.start_token(B, D, seed=0)
    for _ in range(args.warmup):
        time_oracle(hs, x0, min(T_s, 1024), G_s, M, B, D, L)
    vals, secs = [], []
    for _ in range(args.steps):
        v, s, desc = time_oracle(hs, x0, T_s, G_s, M, B, D, L)
        vals.append(v)
        secs.append(s)
    value = len(vals) / sum(1.0 / v for v in vals)
    ms = B * L / value * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded decaying-exponential random filters, N(0,1) start token",
        "config": {"workload": "closed-loop generation of %d tokens through %d long-convolution layers, "
                               "B=%d, D=%d, tanh block and sampler" % (L, M, B, D),
                   "layers": M, "B": B, "D": D, "L": L},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

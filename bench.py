#!/usr/bin/env python3
"""Throughput of the Mel-Band RoFormer core forward on B200 (audio-seconds per second).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the vocals model shape (dim 384, depth 6, 8 heads of 64, 60 mel bands over
n_fft 2048, mask MLP hidden 1536) on one static window of T = 1100 frames (11.0 s of
44.1 kHz stereo), B = 1, fp16 operands with fp32 accumulation, random-init weights
N(0, 0.02) rounded to fp16, stft_repr of seeded synthetic audio (tone stacks + pink
noise at -20 dBFS).  A step is one full core forward (band split, 6 x (time, band)
transformer, mask head, overlap average) through mrf_forward, inputs resident on the
device; the L2 is flushed (256 MiB write) before every timed step, outside its events.

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica on its own
windows (the forward has no exchange step): value = all ranks' audio / max rank time.

--impl reference times the float64 NumPy oracle on the host cores (rank 0 only), on a
bounded sample of the same model (a window of --ref-frames frames per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "audio-sec separated per sec (core fwd, fp16) at T=1100; attention TFLOP/s vs peak"
UNIT = "audio-s/s"
# "musetric/vocal-separation-roformer-onnx", section "What the row cap changed": the core
# forward at T = 1100 in 1.85 s per 11 s window (desktop NVIDIA, WebGPU, fp16): 11.0 / 1.85.
PAGES_AUDIO_S_PER_S = 11.0 / 1.85


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--frames", type=int, default=1100)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--ref-frames", type=int, default=32, help="window of one reference-arm step")
    ap.add_argument("--cpu-sample-frames", type=int, default=1100, help="window of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bf16", action="store_true", help="skip the bf16-mode timing beside the fp16 line")
    ap.add_argument("--chunk-sweep", type=str, default=None, metavar="SECONDS,...",
                    help="instead of the core forward: time mrf_separate_audio_chunked on a 60 s mix for each "
                         "chunk length (seconds), one JSON line each")
    ap.add_argument("--plain", action="store_true",
                    help="profiling run: warmup + steps eager forwards only, no timing or report")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


class RankGroup:
    """The ranks of a replicas run, one process per GPU: a barrier, the maximum of a number over
    the ranks (the slowest rank's device time) and the teardown.  No collective touches the data
    path.  Backend NCCL on GPUs; gloo for the CPU tests of this plumbing.  The group's timeout is
    short, so a rank that fails or leaves ends the others' next collective with an error."""

    def __init__(self, backend="nccl", timeout_s=120):
        self.rank, self.world, self.local = dist_env()
        self.backend = backend
        self._dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self._dist = dist

    def barrier(self):
        if self._dist is not None:
            self._dist.barrier()

    def max(self, value):
        if self._dist is None:
            return float(value)
        import torch
        t = torch.tensor([float(value)], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self._dist is not None:
            self._dist.barrier()
            self._dist.destroy_process_group()
            self._dist = None


def aggregate(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time (ms)."""
    return world * units_per_rank / (ms_max / 1e3)


def workload(cfg, B, T):
    return {"workload": f"vocals core forward, B={B}, T={T} ({B * T * cfg.hop / cfg.sample_rate:.2f} s audio)",
            "dim": cfg.dim, "depth": cfg.depth, "heads": cfg.heads, "dim_head": cfg.dim_head,
            "bands": cfg.num_bands, "n_fft": cfg.n_fft, "batch": B, "frames": T,
            "weights": "random-init N(0,0.02), fp16-rounded"}


def bench_config(cfg, B, T, world):
    """The `config` of both arms' JSON lines: the workload and how it is timed."""
    return dict(workload(cfg, B, T), l2="flushed by a 256 MiB write before every timed step",
                parallelism=f"replicas x{world}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 50 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"mrf_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        """Median SM clock over the samples taken under load (GPU utilisation >= 50 %; all
        samples when none is), the maximum clock, and every throttle reason seen active."""
        if not self.proc or not os.path.exists(self.path):
            return None
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clock_lines(lines)


def summarize_clock_lines(lines):
    """Summary of ClockSampler's CSV lines (index, sm, max sm, power, reasons, 4 throttle flags,
    utilisation)."""
    sm, busy, smax, reasons = [], [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            clk = float(parts[1])
            smax = max(smax, float(parts[2]))
        except ValueError:
            continue
        sm.append(clk)
        try:
            if len(parts) >= 10 and float(parts[9]) >= 50.0:
                busy.append(clk)
        except ValueError:
            pass
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    use = busy or sm
    return {"sm_mhz": statistics.median(use), "sm_max_mhz": smax, "reasons": sorted(reasons),
            "samples": len(sm), "samples_under_load": len(busy)}


def kernel_source_hash(files=None):
    """sha256 (16 hex digits) of the named files under csrc/ (all of csrc/ when None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "axial_band_split_b200", "csrc")
    for n in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu summary
    profiles/traffic.txt, if it was taken on the current sources of the profiled kernels; else
    None.  Format: '# comment' lines, 'sources <file> ...' (under csrc/), 'source_hash <hash>'
    of those files, then '<kernel> <bytes per launch>'."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    vals, files = {}, None
    with open(p) as f:
        for line in f:
            parts = line.split("#")[0].split()
            if parts and parts[0] == "sources":
                files = parts[1:]
            elif len(parts) == 2:
                vals[parts[0]] = parts[1]
    try:
        if vals.get("source_hash") != kernel_source_hash(files):
            return None
    except OSError:
        return None
    v = vals.get(kernel)
    return float(v) if v is not None else None


def frac_block(flops, ms, peaks):
    """Achieved TFLOP/s of `flops` done in `ms` per step, as fractions of the burst (the
    headline: these kernels run inside a forward of a few milliseconds) and sustained peaks."""
    if not ms:
        return {"tflops": None, "frac_of_peak": None, "frac_of_peak_sustained": None}
    tf = flops / (ms / 1e3) / 1e12
    return {"tflops": tf, "frac_of_peak": tf / peaks["bf16_tflops"],
            "frac_of_peak_sustained": tf / peaks["bf16_tflops_sustained"]}


def cpu_baseline(cfg, frames, rank):
    """The float64 oracle as it stands, timed on this host's cores on one forward of a
    `frames`-long window of the same model (a bounded sample of the workload)."""
    import numpy as np
    import synth
    from oracle import model as om
    from oracle import tables as ot
    widths = ot.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands)["widths"]
    W = synth.make_weights(cfg, widths, fp16=True)
    x = synth.make_stft_repr(cfg, 1, frames)
    t0 = time.perf_counter()
    om.forward(x, cfg, W)
    dt = time.perf_counter() - t0
    audio = frames * cfg.hop / cfg.sample_rate
    return {"value": audio / dt, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"one float64 forward of the vocals model on a B=1, T={frames} window "
                      f"({audio:.2f} s audio) in {dt:.1f} s on the host's cores (NumPy/OpenBLAS)"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    from oracle import model as om
    from oracle import tables as ot
    cfg = synth.VOCALS
    T = args.ref_frames
    widths = ot.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands)["widths"]
    W = synth.make_weights(cfg, widths, fp16=True)
    x = synth.make_stft_repr(cfg, 1, T)
    for _ in range(args.warmup):
        om.forward(x, cfg, W)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        om.forward(x, cfg, W)
    dt = time.perf_counter() - t0
    audio = args.steps * T * cfg.hop / cfg.sample_rate
    value = audio / dt
    sample = (f"float64 NumPy oracle, vocals model, one B=1 T={T} window ({T * cfg.hop / cfg.sample_rate:.2f} s "
              f"audio) per step, on the host's cores")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(cfg, args.batch, args.frames, world), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import numpy as np
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    ranks = RankGroup("nccl")
    from axial_band_split_b200 import accounting, build, mrf
    if rank == 0:
        build.build()
    ranks.barrier()
    import synth
    cfg = synth.VOCALS
    B, T = args.batch, args.frames
    widths = mrf.band_tables(cfg)["width"]
    W = {k: v.astype(np.float16) for k, v in synth.make_weights(cfg, widths, fp16=True).items()}
    model = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)
    x_host = synth.make_stft_repr(cfg, B, T, seed=1 + rank)
    x = torch.from_numpy(x_host).cuda()
    out = torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    def timed(fn, steps):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier()
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        barrier()
        ms = sum(a.elapsed_time(b) for a, b in ev)
        return ms

    fwd = lambda: model.forward(x, out)
    if args.plain:
        model.set_graph(False)
        for _ in range(args.warmup + args.steps):
            fwd()
        model.sync_status()
        torch.cuda.synchronize()
        print(f"plain run ok: {args.warmup + args.steps} forwards, {model.launches_per_forward(B, T)} launches each")
        ranks.close()
        model.close()
        return 0
    clk = ClockSampler(local).__enter__()  # sampled over warm-up, timed, per-kernel and e2e passes
    for _ in range(args.warmup):
        fwd()
    model.sync_status()
    ms = timed(fwd, args.steps)
    model.sync_status()
    ms_max = ranks.max(ms)
    launches = model.launches_per_forward(B, T)
    audio_per_rank = args.steps * accounting.audio_seconds(cfg, B, T)
    value = aggregate(audio_per_rank, world, ms_max)

    # end to end through the public host-buffer entry points, from and to pinned host memory.
    # Pipelined (mrf_forward_host_async + mrf_host_join): one event pair around all K calls and the
    # join, so the region holds every step's H2D copy, forward, D2H copy and L2 flush; the copies
    # of neighbouring steps run under each forward (a batch's first copy follows the start event).
    # Synchronous (mrf_forward_host, which waits for its own copies): an event pair around each
    # call, summed, as for `value`.
    # `region` times the same K device-buffer forwards under one event pair with the same flushes:
    # the pipelined figure's reference without copies.
    xin = torch.from_numpy(x_host).pin_memory()
    xouts = [model._out_like(xin, None) for _ in range(2)]

    def one_region(steps, host):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record(stream)
        for k in range(steps):
            flush.zero_()
            if host:
                model.forward_host_async(xin, xouts[k % 2], stream=stream)
            else:
                fwd()
        if host:
            model.host_join(stream)
        e1.record(stream)
        barrier()
        model.sync_status(stream)
        return e0.elapsed_time(e1)

    one_region(args.warmup, True)
    ms_e2e = ranks.max(one_region(args.steps, True))
    ms_region = ranks.max(one_region(args.steps, False))
    sync_fn = lambda: model.forward_host(xin, xouts[0], stream=stream)
    sync_fn()
    ms_e2e_sync = ranks.max(timed(sync_fn, args.steps))
    io_bytes = int(x_host.nbytes)
    out_bytes = int(xouts[0].numel() * 4)

    # per-kernel times: the same steps launched eagerly with an event pair around each kernel
    model.set_timing(True)
    ktimed = timed(fwd, args.steps)
    kt = model.kernel_times()
    model.set_timing(False)
    model.sync_status()

    # the same workload in the bf16 compute mode (weights rounded to bf16), device-timed like `value`
    bf_line = None
    if not args.no_bf16:
        Wb = {k: v for k, v in synth.make_weights(cfg, widths, bf16=True).items()}
        mb = mrf.Model(cfg, Wb, max_batch=B, max_frames=T, compute=mrf.MRF_BF16)
        outb = torch.empty_like(x)
        fwd_b = lambda: mb.forward(x, outb)
        for _ in range(args.warmup):
            fwd_b()
        mb.sync_status()
        ms_b = ranks.max(timed(fwd_b, args.steps))
        mb.sync_status()
        mb.close()
        bf_line = {"value": aggregate(audio_per_rank, world, ms_b), "unit": UNIT, "ms_per_step": ms_b / args.steps,
                   "dtype": "bf16", "note": "same workload, MRF_BF16 (bf16 operands, fp32 residual master copy)"}
    clk.__exit__()

    if rank != 0:
        ranks.close()
        model.close()
        return 0

    peaks, peak_src = load_peaks()
    work = accounting.kernel_work(cfg, widths, B, T)
    per_kernel = {}
    for name, (n, tot) in kt.items():
        kind, amount, nl = work.get(name, ("?", 0, n))
        per_launch = amount / max(nl, 1)
        avg = tot / max(n, 1)
        per_kernel[name] = {"launches_per_step": n / args.steps, "ms_per_step": tot / args.steps,
                            "share": tot / max(sum(v[1] for v in kt.values()), 1e-9),
                            "achieved": (per_launch / (avg / 1e3) / (1e12 if kind == "flop" else 1e9)) if avg > 0 else None,
                            "unit": "TFLOP/s" if kind == "flop" else "GB/s"}
    dom = max(kt.items(), key=lambda kv: kv[1][1])[0]
    kind, amount, nl = work[dom]
    avg_ms = kt[dom][1] / kt[dom][0]
    # The kernels are timed inside a forward of a few milliseconds, not a seconds-long loop, so
    # the tensor roofline is the burst GEMM peak; the sustained one is reported beside it.
    peak_sus = None
    if kind == "flop" and dom != "band_split":
        bound, unit = "tensor", "TFLOP/s"
        peak, peak_sus = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
        achieved = amount / nl / (avg_ms / 1e3) / 1e12
    elif kind == "flop":
        bound, unit = "alu", "TFLOP/s"
        peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        achieved = amount / nl / (avg_ms / 1e3) / 1e12
    else:
        bound, unit = "hbm", "GB/s"
        peak = peaks["hbm_gbs"]
        achieved = amount / nl / (avg_ms / 1e3) / 1e9
    attn_ms = sum(kt[k][1] for k in ("attn_time_tc", "attn_band_tc") if k in kt) / args.steps
    # dense projections: the GEMM launches this forward ran
    gemm_names = [k for k in kt if k.startswith("gemm_") and k in work]
    gemm_ms = sum(kt[k][1] for k in gemm_names) / args.steps
    attn_fl = accounting.attention_flops(cfg, widths, B, T)
    gemm_fl = sum(work[k][1] for k in gemm_names)
    total_fl = accounting.total_flops(cfg, widths, B, T)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": value / PAGES_AUDIO_S_PER_S, "dtype": "f16", "data": "synthetic",
        "config": bench_config(cfg, B, T, world),
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "peak_source": peak_src + (" burst" if bound == "tensor" else ""),
                     "peak_sustained": peak_sus, "frac_sustained": achieved / peak_sus if peak_sus else None,
                     "traffic": traffic_for(dom), "algorithmic_per_launch": amount / nl},
        "attention": frac_block(attn_fl, attn_ms, peaks),
        "gemm": frac_block(gemm_fl, gemm_ms, peaks),
        "forward": {"tflops": total_fl / (ms_max / args.steps / 1e3) / 1e12,
                    "frac_of_peak_burst": total_fl / (ms_max / args.steps / 1e3) / 1e12 / peaks["bf16_tflops"]},
        "kernels": per_kernel,
        "kernel_timing_ms_per_step": ktimed / args.steps,
        "e2e": {"value": aggregate(audio_per_rank, world, ms_e2e), "unit": UNIT,
                "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": out_bytes,
                "ms_per_step": ms_e2e / args.steps,
                "api": "mrf_forward_host_async x K + mrf_host_join, pinned host buffers, one event pair "
                       "around the K steps (copies, forwards and the per-step L2 flush inside)",
                "device_region_ms_per_step": ms_region / args.steps,
                "device_region_note": "the same K forwards from device buffers under one event pair with the same "
                                      "flushes: the pipelined figure without its copies",
                "sync_call": {"value": aggregate(audio_per_rank, world, ms_e2e_sync),
                              "ms_per_step": ms_e2e_sync / args.steps,
                              "api": "mrf_forward_host (waits for its copies), event pair per call"}},
        "bf16": bf_line,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_sample_frames, rank)
    print(json.dumps(line), flush=True)
    ranks.close()
    model.close()
    return 0


def run_chunk_sweep(args):
    """The chunk-length question the pages leave open: the full separation of one 60 s stereo mix
    (STFT, core forward with mask application, iSTFT, fades, overlap-add) per chunk length, up to 16
    chunks per forward, device-timed (CUDA events, L2 flushed before each timed call)."""
    import numpy as np
    import torch
    from axial_band_split_b200 import build, mrf
    import synth
    build.build()
    cfg = synth.VOCALS
    widths = mrf.band_tables(cfg)["width"]
    W = {k: v.astype(np.float16) for k, v in synth.make_weights(cfg, widths, fp16=True).items()}
    L = 60 * cfg.sample_rate
    mix = torch.from_numpy(synth.synth_audio(L, seed=7, clicks=True).astype(np.float32)).cuda()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for sec in [float(v) for v in args.chunk_sweep.split(",")]:
        chunk = int(round(sec * cfg.sample_rate))
        T = 1 + chunk // cfg.hop
        plan = mrf.chunk_plan(cfg.sample_rate, L, chunk)
        m = mrf.Model(cfg, W, max_batch=16, max_frames=T)
        out = torch.empty((1, 2, L), dtype=torch.float32, device="cuda")
        for _ in range(max(args.warmup, 1)):
            m.separate_audio(mix, cfg.hop, out, chunk_samples=chunk)
        m.sync_status()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record()
            m.separate_audio(mix, cfg.hop, out, chunk_samples=chunk)
            e1.record()
        torch.cuda.synchronize()
        m.sync_status()
        ms = sorted(a.elapsed_time(b) for a, b in ev)[len(ev) // 2]
        m.close()
        n = len(plan["off"])
        print(json.dumps({"chunk_s": sec, "chunk_samples": chunk, "frames_per_chunk": T, "chunks": n,
                          "forwards": -(-n // 16), "ms_per_60s": ms, "real_time_factor": ms / 1e3 / 60.0,
                          "audio_s_per_s": 60.0 / (ms / 1e3), "steps": args.steps,
                          "model": "vocals (dim 384, depth 6, 60 bands), fp16, random-init",
                          "mix": "60 s synthetic stereo (tones, pink noise, clicks)"}), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.chunk_sweep:
        return run_chunk_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

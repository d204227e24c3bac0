"""Throughput of the B200 audio-encoder forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload batch16_10to30s|single_30s|clip_10min|tiny_1s]

A step is one forward of the whole hot path (log-mel, conv stem, 32 layers,
head, adapter) over one batch: by default the 16 clips of 10-30 s (seeds
0-15), which is the batched 30 s throughput case.  Inputs are synthetic and
seeded; weights are random-init bf16.  Timing: CUDA events on the encoder's
stream around each step, with a 512 MB buffer written between steps (L2
flush, outside the events); barrier + synchronize on both sides of the K
steps; multi-GPU runs take the max over ranks, each rank encoding its own
batch (clips are independent: weak scaling, no collective on the data path).

At N = 1 the line also carries `other_configs`: the 1 s / 4-layer clip, the
single 30 s clip, the 10-min clip and the 60-min clip streamed in 64 s pieces
(with the encoder's device memory), each timed the same way, the batch and
the streamed clip again with 4-bit weights (`_w4`), and the batch with FP8
q/k/v and fc1 GEMMs (`_fp8`); and
`cpu_baseline` times the oracle on all host cores and on one core.

The reference arm (--impl reference) times the CPU oracle on the host cores
on one 800-frame window of the same batch per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from audio_encoder_b200 import synth  # noqa: E402

MFLOP_PER_TOKEN = 1737.5e6   # algorithmic work per valid token (stem + 32 layers + head + adapter)
L2_FLUSH_BYTES = 512 << 20


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def workload_clips(name):
    desc, make, n_layers = synth.WORKLOADS[name]
    return desc, make(), n_layers


def model_flops(tokens, n_layers, n_taps=0):
    # stem 353.6 + 39.83 per layer + head/adapter 109.2 MFLOP per token; each
    # layer tap runs one more head/adapter set
    return tokens * (353.6e6 + 39.83e6 * n_layers + 109.2e6 * (1 + n_taps))


class Clocks:
    """nvidia-smi sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "20"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.p:
            self.p.terminate()
            try:
                out, _ = self.p.communicate(timeout=5)
            except Exception:
                self.p.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except Exception:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * (mx or 1)] or sm
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_max(value, dist, device):
    """Max of a float over all ranks (the value itself on one process)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(world, units_per_rank, ms_per_step):
    """Whole-job throughput: every rank processes its own units each step,
    and the step takes as long as the slowest rank."""
    return world * units_per_rank / (ms_per_step / 1e3)


def dist_setup(n_gpus):
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import datetime

    import torch
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, world, dist


def oracle_sample(clips, n_layers, windows, blob=None, threads=None):
    """The oracle, as it stands, on the first `windows` 800-frame windows of
    clip 0 with all host threads (or `threads` of them)."""
    import oracle
    blob = synth.make_weights(n_layers) if blob is None else blob
    all_threads = oracle.max_threads()
    if threads:
        oracle.set_threads(threads)
    try:
        m = oracle.Model(blob, n_layers)
        pcm = clips[0]
        gmax = oracle.clip_log_max(pcm)
        t0 = time.perf_counter()
        toks = 0
        for c in range(windows):
            toks += m.encode_chunks(pcm, c, c + 1, gmax=gmax).shape[0]
        dt = time.perf_counter() - t0
        m.close()
        used = oracle.max_threads()
    finally:
        if threads:
            oracle.set_threads(all_threads)
    return dt, toks, used


def gemm_source_hash():
    h = hashlib.sha256()
    for f in ["gemm.cuh", "common.cuh"]:
        with open(os.path.join(ROOT, "audio_encoder_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if the
    GEMM sources are unchanged since the capture; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("captured_source_hash") != gemm_source_hash():
            return None
        return e["bytes_per_launch_full_size"]
    except Exception:
        return None


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    desc, clips, n_layers = workload_clips(args.workload)
    blob = synth.make_weights(n_layers)
    import oracle
    m = oracle.Model(blob, n_layers)
    pcm = clips[0]
    gmax = oracle.clip_log_max(pcm)
    nc = oracle.num_chunks(pcm.size)

    def step(i):
        c = i % nc
        return m.encode_chunks(pcm, c, c + 1, gmax=gmax).shape[0]

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    toks = 0
    for i in range(args.steps):
        toks += step(i)
    dt = time.perf_counter() - t0
    audio_s = toks / 12.5
    v = audio_s / dt
    line = {
        "impl": "reference", "metric": "audio-sec encoded/sec", "value": v, "unit": "audio-s/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "tokens_per_s": toks / dt,
        "config": {"workload": args.workload, "description": desc, "step": "one 800-frame window of clip 0",
                   "layers": n_layers},
        "cpu_baseline": {"value": v, "unit": "audio-s/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"{args.steps} windows of 100 tokens (8 s of audio each) of clip 0"},
        "e2e": {"value": v, "unit": "audio-s/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch

    from audio_encoder_b200 import binding

    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    desc, clips, n_layers = workload_clips(args.workload)
    blob = synth.make_weights(n_layers)
    total_samples = sum(c.size for c in clips)
    stream = torch.cuda.Stream()
    mel_samples = 9_600_000  # the 10-min clip, for the log-mel roofline
    enc = binding.Encoder(blob, n_layers, max_samples=max(total_samples + 4 * len(clips), mel_samples),
                          max_clips=len(clips), out_dtype=binding.OUT_BF16, stream=stream,
                          fp8=args.gemm_dtype == "fp8", nvfp4=args.gemm_dtype == "nvfp4")
    tap_layers = [int(v) for v in args.taps.split(",")] if args.taps else []
    with torch.cuda.stream(stream):
        xs = [torch.from_numpy(c).to(dev) for c in clips]
        tokens = sum(binding.num_tokens(c.size) for c in clips)
        out = torch.empty((tokens, 2048), dtype=torch.bfloat16, device=dev)
        tap_out = [torch.empty((tokens, 2048), dtype=torch.bfloat16, device=dev) for _ in tap_layers]
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    if tap_layers:
        enc.set_taps(tap_layers, synth.make_tap_weights(len(tap_layers)))
    audio_s = total_samples / 16000.0
    torch.cuda.synchronize()

    def step():
        if tap_layers:
            enc.forward_taps(xs, out=out, taps=tap_out)
        else:
            enc.forward(xs, out=out)

    warmup = args.warmup if args.ncu else max(args.warmup, 3)
    for _ in range(warmup):
        step()
    enc.synchronize()

    # ---- timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = enc.launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(dev.index) as clk:
        for i in range(args.steps):
            with torch.cuda.stream(stream):
                flush.fill_(float(i))
                ev[i][0].record(stream)
                step()
                ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches = enc.launch_count() - launches0
    if args.ncu:  # a capture run: no timing report
        print(json.dumps({"ncu_run": True, "steps": args.steps, "warmup": warmup, "gpu_launches": launches}))
        enc.close()
        return
    # Per-kernel breakdown: the same K steps again, launched one by one with
    # CUDA events around every launch (the timed steps above replay the
    # forward as one CUDA graph, which per-launch events would break up).
    enc.profile_enable(400 * (args.steps + 1))
    for i in range(args.steps):
        with torch.cuda.stream(stream):
            flush.fill_(float(i))
            step()
    stats = enc.profile_read()
    enc.profile_enable(0)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = reduce_max(float(sum(step_ms)), dist, dev)
    enc.synchronize()

    # ---- end to end through the host API: pinned PCM in, rows out to host
    # (the host API returns the final rows only, so a run with layer taps
    # reports no end-to-end figure)
    e2e_ms = [float("nan")]
    if not tap_layers:
        pinned = [torch.from_numpy(c).pin_memory() for c in clips]
        rows_host = torch.empty((tokens, 2048), dtype=torch.bfloat16).pin_memory()
        enc.forward_host(pinned, rows_host)
        e2e_ms = []
        for i in range(max(2, min(args.steps, 10))):
            flush.fill_(float(i))
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            enc.forward_host(pinned, rows_host)
            b.record(stream)
            b.synchronize()
            e2e_ms.append(a.elapsed_time(b))
    e2e_step = reduce_max(float(np.mean(e2e_ms)), dist, dev)

    if rank != 0:
        enc.close()
        if dist:
            dist.destroy_process_group()
        return

    # log-mel kernel alone on the 10-min clip (inputs resident, L2 flushed
    # between launches): algorithmic bytes = 4 B per sample read + 512 B per
    # frame written
    mel_roof = None
    if rank == 0:
        with torch.cuda.stream(stream):
            pcm10 = torch.from_numpy(synth.pcm_long(2, mel_samples)).to(dev)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            enc.logmel(pcm10)
        enc.profile_enable(400)
        for i in range(10):
            with torch.cuda.stream(stream):
                flush.fill_(float(i))
                enc.logmel(pcm10)
        mst = enc.profile_read()
        enc.profile_enable(0)
        if "logmel" in mst:
            m = mst["logmel"]
            gbs = m["bytes"] / (m["ms"] / 1e3) / 1e9
            hbm = peaks()["hbm"]
            mel_roof = {"kernel": "logmel", "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                        "frac": gbs / hbm, "ms_per_launch": m["ms"] / m["launches"],
                        "bytes_per_launch": m["bytes"] / m["launches"],
                        "workload": "one 10-min clip, 9.6M samples, 60000 frames"}
        del pcm10

    pk = peaks()
    ms_per_step = total_ms / args.steps
    value = weak_scaling_throughput(world, audio_s, ms_per_step)
    flops_step = model_flops(tokens, n_layers, len(tap_layers))
    tflops = flops_step / (ms_per_step / 1e3) / 1e12
    # dominant kernel: the category with the most device time
    dom_name, dom = max(stats.items(), key=lambda kv: kv[1]["ms"])
    per_launch_ms = dom["ms"] / dom["launches"]
    kernel_ms = sum(v["ms"] for v in stats.values())
    if dom["flops"] > 0 and dom_name.startswith("gemm"):
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16"], "frac_of_sustained": achieved / pk["bf16_sus"],
                "peak_note": f"{pk['src']} burst bf16 (the sustained figure, {pk['bf16_sus']}, gives "
                             f"frac_of_sustained)"}
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "peak_note": f"{pk['src']} HBM copy bandwidth"}
    roof.update({"kernel": dom_name, "launches_per_step": dom["launches"] / args.steps,
                 "ms_per_launch": per_launch_ms, "share_of_kernel_time": dom["ms"] / kernel_ms,
                 "traffic": profiled_traffic(dom_name),
                 "timing": "CUDA events around every launch, in a pass of the same steps launched one by one"})

    kernels = {k: {"ms_per_step": v["ms"] / args.steps, "launches_per_step": v["launches"] / args.steps,
                   "tflops": (v["flops"] / (v["ms"] / 1e3) / 1e12) if v["flops"] and v["ms"] else None,
                   "gbs": (v["bytes"] / (v["ms"] / 1e3) / 1e9) if v["bytes"] and v["ms"] else None}
               for k, v in sorted(stats.items(), key=lambda kv: -kv[1]["ms"])}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        dt, toks, cores = oracle_sample(clips, n_layers, windows=args.cpu_windows, blob=blob)
        cpu = {"value": (toks / 12.5) / dt, "unit": "audio-s/s", "cores": cores, "kind": "oracle",
               "sample": f"first {args.cpu_windows} 800-frame windows of clip 0 ({toks} tokens, "
                         f"{toks / 12.5:.0f} s of audio), all {n_layers} layers, {dt:.1f} s"}
        if not args.no_cpu_one_core:
            dt1, toks1, _ = oracle_sample(clips, n_layers, windows=1, blob=blob, threads=1)
            cpu["one_core"] = {"value": (toks1 / 12.5) / dt1, "unit": "audio-s/s", "cores": 1,
                               "sample": f"first 800-frame window of clip 0 ({toks1} tokens), {dt1:.1f} s"}

    line = {
        "metric": "audio-sec encoded/sec", "value": value, "unit": "audio-s/s", "n_gpus": world,
        "steps": args.steps, "warmup": warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if args.gemm_dtype == "bf16" else f"bf16 ({args.gemm_dtype} q/k/v and fc1 GEMMs)",
        "data": "synthetic (seeded PCM, random-init bf16 weights)",
        "tokens_per_s": weak_scaling_throughput(world, tokens, ms_per_step),
        "model_tflops": tflops,
        "tc_roofline_frac": tflops / pk["bf16"],
        "tc_roofline_frac_sustained": tflops / pk["bf16_sus"],
        "config": {"workload": args.workload, "description": desc, "clips_per_gpu": len(clips),
                   "audio_s_per_gpu": audio_s, "tokens_per_gpu": tokens, "layers": n_layers,
                   "out_dtype": "bf16", "l2": "512 MB buffer written between timed steps (outside the events)",
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   **({"gemm_dtype": args.gemm_dtype} if args.gemm_dtype != "bf16" else {}),
                   **({"tap_layers": tap_layers} if tap_layers else {})},
        "roofline": roof,
        "mel_roofline": mel_roof,
        "kernels": kernels,
        "kernel_ms_per_step_eager": kernel_ms / args.steps,
        "gpu_launches": launches,
        "e2e": None if tap_layers else {
            "value": weak_scaling_throughput(world, audio_s, e2e_step), "unit": "audio-s/s",
            "h2d_bytes_per_step": 4 * total_samples, "d2h_bytes_per_step": 2 * tokens * 2048,
            "ms_per_step": e2e_step},
        "cpu_baseline": cpu,
        "clocks": clk.summary(),
    }
    enc.close()
    if world == 1 and not args.no_other_configs and not tap_layers:
        line["other_configs"] = other_configs(args, dev)
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def measure_streamed(steps, warmup, dev, dist=None, world=1, weight_bits=16):
    """The 60-min clip encoded as a stream of 64 s pieces (1,024,000 samples,
    the last 256,000): a step is the whole-clip log-mel maximum (one pass)
    and the 57 piece forwards against it, each piece reading its 200-sample
    halo from the whole clip.  Returns the step time (max over ranks), the
    launch count, the clock record and the device memory the encoder holds
    (weights + workspace for one piece)."""
    import torch

    from audio_encoder_b200 import binding

    desc, clips, n_layers = workload_clips("clip_60min_streamed")
    pcm = clips[0]
    n = pcm.size
    piece = 1_024_000
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    stream = torch.cuda.Stream()
    enc = binding.Encoder(synth.make_weights(n_layers), n_layers, max_samples=piece, max_clips=1,
                          out_dtype=binding.OUT_BF16, stream=stream, weight_bits=weight_bits)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    tokens = binding.num_tokens(n)
    with torch.cuda.stream(stream):
        x = torch.from_numpy(pcm).to(dev)
        out = torch.empty((tokens, 2048), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    ranges = []
    r0 = 0
    for b in range(0, n, piece):
        e = min(b + piece, n)
        t = binding.range_tokens(n, b, e)
        ranges.append((b, e, r0, r0 + t))
        r0 += t
    assert r0 == tokens
    torch.cuda.synchronize()

    def step():
        with torch.cuda.stream(stream):
            lm = enc.log_max(x)
            for b, e, o0, o1 in ranges:
                enc.forward([(x, b, e, lm)], out=out[o0:o1])

    for _ in range(warmup):
        step()
    enc.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launches0 = enc.launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(dev.index) as clk:
        for i in range(steps):
            with torch.cuda.stream(stream):
                flush.fill_(float(i))
                ev[i][0].record(stream)
            step()
            with torch.cuda.stream(stream):
                ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches = enc.launch_count() - launches0
    total_ms = reduce_max(float(sum(a.elapsed_time(c) for a, c in ev)), dist, dev)
    enc.close()
    return dict(desc=desc, ms=total_ms / steps, audio_s=n / 16000.0, tokens=tokens, n_layers=n_layers,
                pieces=len(ranges), piece=piece, launches=launches, clocks=clk.summary(),
                encoder_device_bytes=int(free0 - free1), clip_and_rows_device_bytes=int(4 * n + 2 * tokens * 2048))


def run_streamed(args):
    """bench --workload clip_60min_streamed: sustained audio-seconds per
    second of the 60-min clip streamed in 64 s pieces, and the device memory
    the encoder holds.  Weak scaling: every rank streams its own clip."""
    import torch

    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    warmup = max(args.warmup, 3)
    r = measure_streamed(args.steps, warmup, dev, dist, world)
    ms = r["ms"]
    pk = peaks()
    tflops = model_flops(r["tokens"], r["n_layers"]) / (ms / 1e3) / 1e12
    if rank == 0:
        line = {
            "metric": "audio-sec encoded/sec", "value": weak_scaling_throughput(world, r["audio_s"], ms),
            "unit": "audio-s/s", "n_gpus": world, "steps": args.steps, "warmup": warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded PCM, random-init bf16 weights)",
            "tokens_per_s": weak_scaling_throughput(world, r["tokens"], ms),
            "model_tflops": tflops, "tc_roofline_frac": tflops / pk["bf16"],
            "tc_roofline_frac_sustained": tflops / pk["bf16_sus"],
            "config": {"workload": "clip_60min_streamed", "description": r["desc"], "pieces": r["pieces"],
                       "piece_samples": r["piece"], "audio_s_per_gpu": r["audio_s"], "tokens_per_gpu": r["tokens"],
                       "layers": r["n_layers"], "out_dtype": "bf16",
                       "encoder_device_bytes": r["encoder_device_bytes"],
                       "clip_and_rows_device_bytes": r["clip_and_rows_device_bytes"],
                       "l2": "512 MB buffer written between timed steps (outside the events)",
                       "parallelism": f"dp{world}" if world > 1 else "single"},
            "gpu_launches": r["launches"],
            "e2e": None,
            "clocks": r["clocks"],
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def measure_plain(workload, steps, warmup, dev, weight_bits=16, fp8=False, nvfp4=False):
    """One workload's forward timed as the headline is (device-resident PCM,
    CUDA events on the encoder's stream, L2 flushed between steps)."""
    import torch

    from audio_encoder_b200 import binding

    desc, clips, n_layers = workload_clips(workload)
    stream = torch.cuda.Stream()
    total = sum(c.size for c in clips)
    enc = binding.Encoder(synth.make_weights(n_layers), n_layers, max_samples=total, max_clips=len(clips),
                          out_dtype=binding.OUT_BF16, stream=stream, weight_bits=weight_bits, fp8=fp8, nvfp4=nvfp4)
    tokens = sum(binding.num_tokens(c.size) for c in clips)
    with torch.cuda.stream(stream):
        xs = [torch.from_numpy(c).to(dev) for c in clips]
        out = torch.empty((tokens, 2048), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    for _ in range(warmup):
        enc.forward(xs, out=out)
    enc.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with Clocks(dev.index) as clk:
        for i in range(steps):
            with torch.cuda.stream(stream):
                flush.fill_(float(i))
                ev[i][0].record(stream)
                enc.forward(xs, out=out)
                ev[i][1].record(stream)
        torch.cuda.synchronize()
    enc.synchronize()
    enc.close()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    return dict(desc=desc, ms=ms, audio_s=total / 16000.0, tokens=tokens, n_layers=n_layers, clocks=clk.summary())


def other_configs(args, dev):
    """Throughput of the other workloads at N = 1, each timed as the headline
    (the single 30 s clip, the 10-min clip, the 1 s / 4-layer clip, and the
    60-min clip streamed in 64 s pieces with the encoder's device memory)."""
    pk = peaks()
    res = {}
    steps = max(3, min(args.steps, 20))
    # then the 4-bit-weight encoder (round to nearest, groups of 128), the FP8
    # encoder (q/k/v and fc1 on e4m3 operands) and the NVFP4 encoder (q/k/v
    # and fc1 on NVFP4 operands; "bits" 44 below)
    for w, bits in (("tiny_1s", 16), ("single_30s", 16), ("clip_10min", 16), ("clip_60min_streamed", 16),
                    ("batch16_10to30s", 4), ("clip_60min_streamed", 4), ("batch16_10to30s", 8),
                    ("batch16_10to30s", 44)):
        if w == "clip_60min_streamed":
            r = measure_streamed(max(3, min(args.steps, 10)), 3, dev, weight_bits=bits)
        else:
            r = measure_plain(w, steps, 3, dev, weight_bits=4 if bits == 4 else 16, fp8=bits == 8,
                              nvfp4=bits == 44)
        tf = model_flops(r["tokens"], r["n_layers"]) / (r["ms"] / 1e3) / 1e12
        e = {"value": r["audio_s"] / (r["ms"] / 1e3), "unit": "audio-s/s", "ms_per_step": r["ms"],
             "tokens_per_s": r["tokens"] / (r["ms"] / 1e3), "tokens": r["tokens"], "layers": r["n_layers"],
             "model_tflops": tf, "tc_roofline_frac": tf / pk["bf16"], "tc_roofline_frac_sustained": tf / pk["bf16_sus"],
             "description": r["desc"], "clocks": r["clocks"]}
        if w == "clip_60min_streamed":
            e.update({"pieces": r["pieces"], "piece_samples": r["piece"],
                      "encoder_device_bytes": r["encoder_device_bytes"],
                      "clip_and_rows_device_bytes": r["clip_and_rows_device_bytes"]})
        e["weight_bits"] = 4 if bits == 4 else 16
        e["fp8_qkv_fc1"] = bits == 8
        e["nvfp4_qkv_fc1"] = bits == 44
        res[w if bits == 16 else w + {4: "_w4", 8: "_fp8", 44: "_nvfp4"}[bits]] = e
    return res


def run_sharded(args):
    """One long clip split over the ranks by whole 800-frame chunks
    (audio_encoder_b200.shard): a step is each rank's log-mel maximum over its
    range, one all-reduce(max) of that float over NCCL (the path's only
    exchange), and the rank's range encoded against the common maximum.
    Strong scaling: the same clip at every N; value = clip audio-seconds per
    step time (max over ranks)."""
    import torch

    from audio_encoder_b200 import binding, shard

    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    name = args.workload if args.workload in ("clip_10min", "clip_60min_streamed") else "clip_10min"
    desc, clips, n_layers = workload_clips(name)
    pcm = clips[0]
    n = pcm.size
    b, e = shard.chunk_ranges(n, world)[rank]
    stream = torch.cuda.Stream()
    enc = binding.Encoder(synth.make_weights(n_layers), n_layers, max_samples=max(e - b, 1), max_clips=1,
                          out_dtype=binding.OUT_BF16, stream=stream)
    with torch.cuda.stream(stream):
        x = torch.from_numpy(pcm).to(dev)
        rows_n = binding.range_tokens(n, b, e) if e > b else 0
        out = torch.empty((max(rows_n, 1), 2048), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    def max_reduce(t):
        if dist:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)

    def step():
        with torch.cuda.stream(stream):
            shard.encode_range(enc, x, rank, world, max_reduce, out=out[:rows_n] if rows_n else None)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(dev.index) as clk:
        for i in range(args.steps):
            with torch.cuda.stream(stream):
                flush.fill_(float(i))
                ev[i][0].record(stream)
            step()
            with torch.cuda.stream(stream):
                ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = reduce_max(float(sum(a.elapsed_time(c) for a, c in ev)), dist, dev)
    ms = total_ms / args.steps
    audio_s = n / 16000.0
    tokens = binding.num_tokens(n)
    if rank == 0:
        line = {
            "metric": "audio-sec encoded/sec", "value": audio_s / (ms / 1e3), "unit": "audio-s/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded PCM, random-init bf16 weights)",
            "tokens_per_s": tokens / (ms / 1e3),
            "model_tflops": model_flops(tokens, n_layers) / (ms / 1e3) / 1e12,
            "config": {"workload": name + "_sharded", "description": desc + ", chunk ranges split over ranks",
                       "audio_s": audio_s, "tokens": tokens, "layers": n_layers,
                       "l2": "512 MB buffer written between timed steps (outside the events)",
                       "parallelism": f"windows{world}" if world > 1 else "single"},
            "e2e": None,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    enc.close()
    if dist:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="batch16_10to30s", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-windows", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-one-core", action="store_true",
                    help="skip timing the oracle on one host core (one 800-frame window)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="report the default workload only (no per-config numbers for the other workloads)")
    ap.add_argument("--shard-clip", action="store_true",
                    help="one long clip (10 or 60 min) split over the ranks by chunk ranges (strong scaling)")
    ap.add_argument("--taps", default="",
                    help="comma-separated encoder layers (0-based) whose hidden states also go through a "
                         "head + adapter set of their own (layer taps); the step is forward_taps")
    ap.add_argument("--gemm-dtype", default="bf16", choices=["bf16", "fp8", "nvfp4"],
                    help="operands of every layer's q/k/v and fc1 GEMMs (the other GEMMs stay bf16); the "
                         "roofline stays the bf16 one")
    ap.add_argument("--ncu", action="store_true",
                    help="capture run for ncu: warm-up as given (may be 0), the timed steps only, no report")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.shard_clip:
        run_sharded(args)
    elif args.workload == "clip_60min_streamed":
        run_streamed(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

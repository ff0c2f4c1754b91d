"""Benchmark of the streaming KV hot path (one JSON line on rank 0).

One step = one streamed chunk through every DiT layer: for each layer,
sdv2_kv_append then sdv2_chunk_attention over the sink + window cache; then
sdv2_sink_refresh and sdv2_motion_noise_rate.  Default workload: the
Wan-1.3B-shaped stack at 512x512 (30 layers, 12 heads x 128, 32x32 tokens per
latent frame, chunk of 1 frame, 1 sink + 6 window frames, batch 1), with the
ring already wrapped (steady state), sink refresh on 1536-wide hidden states
and motion on 16x64x64 latents.  Inputs are seeded synthetic N(0,1) data.

On one GPU the default run also times, in the same process, the Wan-14B-shaped
stack at B = 1, 2, 4, 8 (the batch sweep) and the 1.3B shape at 480x832 with
four streams at staggered positions; each gets its own entry under
``workloads`` (value, ms_per_step, roofline, clocks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Under torchrun each rank runs an independent replica (the path has no
cross-GPU exchange); value = frames of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk-attn TFLOP/s + KV HBM GB/s vs roofline; latent frames/s (1.3B/14B shape)"
UNIT = "latent frames/s"

WORKLOADS = {
    # name: cache config + refresh/motion shapes (+ optional per-stream join steps)
    "wan1.3b-512x512": dict(batch=1, layers=30, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                            sink_frames=1, window_frames=6, embed_dim=1536, motion=(16, 64, 64)),
    # four independent streams at different positions: stream b joins the stream batch at
    # step join[b], so after the pre-roll the streams sit 0, 2, 6 and 12 frames apart (their
    # window slots differ: offsets 0, 2, 6, 4 modulo the 8-frame window)
    "wan1.3b-480x832-b4": dict(batch=4, layers=30, heads=12, head_dim=128, frame_h=30, frame_w=52, chunk_frames=2,
                               sink_frames=1, window_frames=8, embed_dim=1536, motion=(16, 60, 104),
                               join=(0, 1, 3, 6)),
}
for _b in (1, 2, 4, 8):   # the batch sweep of the 14B shape
    WORKLOADS[f"wan14b-512x512-b{_b}"] = dict(batch=_b, layers=40, heads=40, head_dim=128, frame_h=32, frame_w=32,
                                              chunk_frames=1, sink_frames=1, window_frames=6, embed_dim=5120,
                                              motion=(16, 64, 64))
# small-chunk, memory-bound regime: 128x128 video (8x8 latent tokens per frame),
# 16 independent streams
WORKLOADS["wan1.3b-128x128-b16"] = dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=8,
                                        chunk_frames=1, sink_frames=1, window_frames=6, embed_dim=1536,
                                        motion=(16, 16, 16))
# the same shapes with the fp8 (E4M3) block-scaled cache; 128x256 video (8x16 = 128 latent
# tokens per frame, whole 128-token blocks) for the memory-bound regime in both formats
WORKLOADS["wan1.3b-512x512-fp8"] = dict(WORKLOADS["wan1.3b-512x512"], kv_format="fp8")
WORKLOADS["wan14b-512x512-b8-fp8"] = dict(WORKLOADS["wan14b-512x512-b8"], kv_format="fp8")
WORKLOADS["wan1.3b-128x256-b16"] = dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=16,
                                        chunk_frames=1, sink_frames=1, window_frames=6, embed_dim=1536,
                                        motion=(16, 16, 32))
WORKLOADS["wan1.3b-128x256-b16-fp8"] = dict(WORKLOADS["wan1.3b-128x256-b16"], kv_format="fp8")
WORKLOADS["wan1.3b-128x128-b16-fp8"] = dict(WORKLOADS["wan1.3b-128x128-b16"], kv_format="fp8")
# the small-chunk shapes with the append fused into the attention (sdv2_append_attention)
WORKLOADS["wan1.3b-128x128-b16-fused"] = dict(WORKLOADS["wan1.3b-128x128-b16"], fused=True)
WORKLOADS["wan1.3b-128x256-b16-fused"] = dict(WORKLOADS["wan1.3b-128x256-b16"], fused=True)
WORKLOADS["tiny-stream"] = dict(batch=1, layers=1, heads=2, head_dim=64, frame_h=4, frame_w=4, chunk_frames=1,
                                sink_frames=1, window_frames=2, embed_dim=64, motion=(16, 4, 4))
DEFAULT_WORKLOAD = "wan1.3b-512x512"
# timed beside the default workload on one GPU, each under ``workloads``
EXTRA_WORKLOADS = ("wan14b-512x512-b1", "wan14b-512x512-b2", "wan14b-512x512-b4", "wan14b-512x512-b8",
                   "wan1.3b-480x832-b4", "wan1.3b-128x128-b16", "wan1.3b-128x128-b16-fused")
TAU = 0.9
# device-side wait (cycles, ~40 us at 1.9 GHz) queued ahead of every call that a timing
# pass brackets with events
LEAD_CYCLES = 80_000


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_digest(path):
    """sha256 prefix of a CUDA/C++ source with its // comments and blank lines removed:
    the same for two versions of the file that differ only in comments."""
    import hashlib
    lines = []
    for line in open(path, encoding="utf-8").read().splitlines():
        i = line.find("//")
        line = (line[:i] if i >= 0 else line).rstrip()
        if line:
            lines.append(line)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel code (else None)."""
    path = os.path.join(ROOT, "profiles", f"chunk_attention_{workload}.md")
    src = os.path.join(ROOT, "causal_dit_kv_b200", "csrc", "attention.cu")
    if not os.path.exists(path):
        return None
    digest = source_digest(src)
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":")[0].strip() in ("traffic_bytes_per_launch", "source_sha256_prefix"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("source_sha256_prefix") != digest:
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def workload_config(name, w, world):
    """The JSON config block of a workload (shared by both arms)."""
    n = w["frame_h"] * w["frame_w"]
    slots = w["sink_frames"] + w["window_frames"]
    cache_mb = 2.0 * w["layers"] * w["batch"] * slots * n * w["heads"] * w["head_dim"] * kv_elem(w) / 1e6
    cfg = {"workload": name, "batch": w["batch"], "layers": w["layers"], "heads": w["heads"],
           "head_dim": w["head_dim"], "tokens_per_frame": n, "chunk_frames": w["chunk_frames"],
           "sink_frames": w["sink_frames"], "window_frames": w["window_frames"], "keys_per_stream": slots * n,
           "queries_per_stream": w["chunk_frames"] * n, "refresh_embed_dim": w["embed_dim"],
           "motion_latent": list(w["motion"]),
           "l2": "inputs larger than L2 (per-step caches %.0f MB over %d layers)" % (cache_mb, w["layers"]),
           "kv_format": w.get("kv_format", "bf16"), "parallelism": f"replicas x{world}"}
    if "join" in w:
        cfg["stream_join_steps"] = list(w["join"])
    if w.get("fused"):
        cfg["append"] = "fused into the attention (sdv2_append_attention)"
    return cfg


def kv_elem(w):
    """Bytes per cached K or V element."""
    return 1 if w.get("kv_format", "bf16") == "fp8" else 2


def attn_flops(w, keys):
    lq = w["chunk_frames"] * w["frame_h"] * w["frame_w"]
    return sum(4.0 * w["heads"] * lq * k * w["head_dim"] for k in keys)


def attn_bytes(w, keys):
    """Bytes one attention kernel launch must move: K and V read once, the raw bf16
    queries read (the kernel rotates them on load), O (bf16) written.  The fp8 cache
    stores 1-byte codes and adds one K and one V scale per block of up to 128 tokens of a
    slot and head (frames of 64 tokens: one block per slot; their padding is not read).
    With the append fused in, the chunk's own K and V (part of the keys read once, from
    the caller's buffers) are also written to their ring slots."""
    n = w["frame_h"] * w["frame_w"]
    lq = w["chunk_frames"] * n
    hd = w["heads"] * w["head_dim"]
    e = kv_elem(w)
    total = 0.0
    for k in keys:
        total += 2.0 * e * k * hd + 2.0 * lq * hd + 2.0 * lq * hd
        if e == 1:
            total += 2 * 4.0 * w["heads"] * (k // n) * -(-n // 128)
        if w.get("fused"):
            total += 2.0 * 2.0 * lq * hd
    return total


def steady_keys(w):
    n = w["frame_h"] * w["frame_w"]
    return [(w["sink_frames"] + w["window_frames"]) * n] * w["batch"]


def attention_roofline(w, name, kern_us, peaks, peak_src):
    """Roofline entry of the attention kernel from its own event-timed duration.  The
    kernel is timed launch by launch in a pass of its own, so its tensor peak is the
    burst figure (bf16_tflops); the fraction against the sustained figure is reported
    beside it."""
    fp8 = w.get("kv_format", "bf16") == "fp8"
    keys = steady_keys(w)
    flops = attn_flops(w, keys)
    abytes = attn_bytes(w, keys)
    peak, peak_name = peaks["bf16_tflops"], "bf16_tflops (burst)"
    sustained = peaks.get("bf16_tflops_sustained", peak)
    if fp8:
        # E4M3 products: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25)
        peak, sustained, peak_name = 2.0 * peak, 2.0 * sustained, "bf16_tflops (burst) x 2 (nominal fp8/bf16 ratio)"
    hbm = peaks["hbm_gbs"]
    hbm_bound = abytes / (hbm * 1e9) > flops / (peak * 1e12)
    t = kern_us / 1e6
    achieved_tf = flops / t / 1e12
    achieved_gbs = abytes / t / 1e9
    r = {"kernel": "chunk_attention_kernel" + ("<fused append>" if w.get("fused") else ""),
         "bound": "hbm" if hbm_bound else "tensor",
         "achieved": round(achieved_gbs if hbm_bound else achieved_tf, 2), "peak": hbm if hbm_bound else peak,
         "unit": "GB/s" if hbm_bound else "TFLOP/s",
         "frac": round(achieved_gbs / hbm if hbm_bound else achieved_tf / peak, 4),
         "traffic": profiled_traffic(name),
         "peak_source": f"{peak_src} " + ("hbm_gbs" if hbm_bound else peak_name),
         "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": abytes,
         "avg_launch_us": round(kern_us, 3),
         "timing": "CUDA events recorded by the library right before and after the kernel's launch "
                   "(sdv2_cache_time_attention), in a pass of its own; each launch is preceded on the stream "
                   "by a short device-side wait so that the events time the kernel, not the host's launch latency"}
    if not hbm_bound:
        r["frac_vs_sustained_peak"] = round(achieved_tf / sustained, 4)
    return r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for name, val in zip(names, f[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if sm:
            out.update(sm_mhz=statistics.median(sm), sm_max_mhz=max(mx), reasons=sorted(reasons), samples=len(sm))
        return out


def max_over_ranks(values, dist, device):
    """Element-wise maximum of per-rank timings (every rank calls it once)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def stream_frames(w, step_index):
    """First frame of each stream's chunk at the given global step (-1: not yet joined)."""
    join = w.get("join", (0,) * w["batch"])
    tp = w["chunk_frames"]
    return [(step_index - j) * tp if step_index >= j else -1 for j in join]


def preroll_steps(w):
    """Steps after which every stream's ring has wrapped (every slot valid and reused)."""
    join = w.get("join", (0,) * w["batch"])
    slots = w["sink_frames"] + w["window_frames"]
    return max(join) + (slots + w["chunk_frames"] - 1) // w["chunk_frames"] + 1


# ----------------------------------------------------------------------------- our arm

class Runner:
    """One workload on one GPU: the cache, the input pool and the streamed step."""

    def __init__(self, w, dev, seed, n_inputs):
        import torch

        import synth
        from causal_dit_kv_b200 import KVCache, MotionState

        self.w = w
        self.dev = dev
        B, L, H, D = w["batch"], w["layers"], w["heads"], w["head_dim"]
        self.B, self.L = B, L
        N = w["frame_h"] * w["frame_w"]
        self.Tp = w["chunk_frames"]
        self.Lq = self.Tp * N
        E = w["embed_dim"]
        C, MH, MW = w["motion"]
        self.cache = KVCache(B, L, H, D, w["frame_h"], w["frame_w"], self.Tp, w["sink_frames"], w["window_frames"],
                             embed_dim=E, kv_format=w.get("kv_format", "bf16"))
        self.mot = MotionState(B, self.Tp, C, MH, MW, window=4, sigma=2.0, lam=0.9)
        self.scale = 1.0 / math.sqrt(D)
        # Input pool: two distinct steps' worth of Q/K/V for every layer, drawn on the
        # device.  Hidden states and latents form one continuous stream per step (a slowly
        # drifting chunk embedding with rare scene cuts, latents with segment-wise motion).
        self.n_inputs = n_inputs
        self.pool = []
        for p in range(2):
            qkv = [synth.chunk_qkv_on(dev, seed, B, self.Lq, H, D, p, l) for l in range(L)]
            self.pool.append(dict(q=[t[0] for t in qkv], k=[t[1] for t in qkv], v=[t[2] for t in qkv]))
        self.hid_seq = [h.to(dev) for h in synth.drifting_hidden(seed, B, self.Lq, E, n_inputs, drift=0.02,
                                                                 cut_prob=0.01)]
        self.lat_seq = [x.to(dev) for x in synth.motion_latents(seed, B, self.Tp, C, MH, MW, n_inputs)]
        self.out = torch.empty((B, self.Lq, H, D), dtype=torch.bfloat16, device=dev)
        self.out_slot = torch.empty(B, dtype=torch.int32, device=dev)
        self.rate = torch.empty(B, dtype=torch.float32, device=dev)
        self.n_step = 0
        self.stream = torch.cuda.current_stream(dev)

    def rec(self):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def lead(self):
        """Keep the GPU busy while the host submits the next timed call: a short device-side
        wait queued ahead of the start event, so the events time the GPU work of the call
        and not the host's launch latency (an idle GPU would timestamp the start event
        before the call's kernels have even been submitted)."""
        import torch
        torch.cuda._sleep(LEAD_CYCLES)

    def step(self, inp, ev=None, wait=None, kernel_ev=None):
        """One streamed chunk through every layer; ev (optional) collects event pairs per
        call; kernel_ev (optional) collects event pairs around each attention kernel alone;
        wait (optional) is called with the layer index (L for the refresh/motion inputs)
        before the calls that read that layer's inputs."""
        f0 = stream_frames(self.w, self.n_step)
        cache, rec = self.cache, self.rec
        fused = self.w.get("fused", False)
        for l in range(self.L):
            if wait is not None:
                wait(l)
            if ev is not None and not fused:
                self.lead()
                ev["append"].append([rec()])
            if not fused:
                cache.kv_append(l, inp["k"][l], inp["v"][l], f0)
            if ev is not None:
                if not fused:
                    ev["append"][-1].append(rec())
                self.lead()
                ev["attention"].append([rec()])
            if kernel_ev is not None:
                k0, k1 = rec(), rec()                    # recorded once so the CUDA events exist
                cache.time_attention(k0, k1)
                self.lead()
            if fused:
                cache.append_attention(l, inp["q"][l], inp["k"][l], inp["v"][l], self.out, f0, self.scale)
            else:
                cache.chunk_attention(l, inp["q"][l], self.out, f0, self.scale)
            if kernel_ev is not None:
                cache.time_attention()
                kernel_ev.append([k0, k1])
            if ev is not None:
                ev["attention"][-1].append(rec())
        if wait is not None:
            wait(self.L)
        if ev is not None:
            self.lead()
            ev["refresh"].append([rec()])
        i = self.n_step % self.n_inputs
        hid, lat = (inp["hid"], inp["lat"]) if "hid" in inp else (self.hid_seq[i], self.lat_seq[i])
        cache.sink_refresh(hid, TAU, f0, self.out_slot)
        if ev is not None:
            ev["refresh"][-1].append(rec())
            self.lead()
            ev["motion"].append([rec()])
        self.mot.noise_rate(lat, self.rate)
        if ev is not None:
            ev["motion"][-1].append(rec())
        self.n_step += 1

    def warm(self, warmup):
        import torch
        for i in range(preroll_steps(self.w) + warmup):
            self.step(self.pool[i % 2])
        torch.cuda.synchronize()

    def timed_steps(self, steps, pg=None):
        """Device time (ms) of `steps` whole steps, no events inside (they would break
        the overlap of dependent launches); returns (ms, launches, clocks)."""
        import torch

        from causal_dit_kv_b200 import binding
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches0 = binding.sdv2_launch_count()
        with ClockSampler(self.dev.index or 0) as clocks:
            if pg:
                pg.barrier()
            torch.cuda.synchronize()
            t0.record(self.stream)
            for i in range(steps):
                self.step(self.pool[i % 2])
            t1.record(self.stream)
            torch.cuda.synchronize()
            if pg:
                pg.barrier()
        return t0.elapsed_time(t1), binding.sdv2_launch_count() - launches0, clocks.summary()

    def kernel_us(self, steps):
        """Mean duration of the attention kernel alone (library-recorded events)."""
        import torch
        kev = []
        for i in range(steps):
            self.step(self.pool[i % 2], kernel_ev=kev)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in kev) * 1e3

    def call_us(self, steps):
        import torch
        ev = {k: [] for k in ("append", "attention", "refresh", "motion")}
        for i in range(steps):
            self.step(self.pool[i % 2], ev)
        torch.cuda.synchronize()
        return {k: (statistics.mean(a.elapsed_time(b) for a, b in pairs) * 1e3 if pairs else None)
                for k, pairs in ev.items()}

    def close(self):
        self.cache.close()
        self.mot.close()


def measure_extra(name, args, dev, peaks, peak_src):
    """Value, step time, attention roofline and clocks of one more workload (one GPU).
    Its hidden states and latents cycle through 8 consecutive chunks of the stream."""
    import torch
    w = WORKLOADS[name]
    run = Runner(w, dev, 2100, n_inputs=8)
    try:
        run.warm(args.warmup)
        ms, launches, clocks = run.timed_steps(args.steps)
        kern = run.kernel_us(args.steps)
        assert run.cache.check() == 0 and run.mot.check() == 0, "device status word set"
    finally:
        run.close()
        del run
        torch.cuda.empty_cache()
    frames = args.steps * w["batch"] * w["chunk_frames"]
    return {"value": round(frames / (ms / 1e3), 3), "unit": UNIT, "ms_per_step": round(ms / args.steps, 4),
            "steps": args.steps, "config": workload_config(name, w, 1),
            "roofline": attention_roofline(w, name, kern, peaks, peak_src), "gpu_launches": int(launches),
            "clocks": clocks}


def run_ours(args, w, name):
    import datetime

    import torch

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    dev = torch.device("cuda", local)
    B, L, H, D = w["batch"], w["layers"], w["heads"], w["head_dim"]
    Tp = w["chunk_frames"]
    C, MH, MW = w["motion"]
    run = Runner(w, dev, 2000 + rank, n_inputs=preroll_steps(w) + args.warmup + 5 * args.steps + 3)
    run.warm(args.warmup)

    ms, launches, clocks = run.timed_steps(args.steps, pg)
    call_us = run.call_us(args.steps)
    call_us["attn_kernel"] = run.kernel_us(args.steps)
    assert run.cache.check() == 0 and run.mot.check() == 0, "device status word set"

    # ---- end to end: pinned host inputs copied in, results copied out, every step.  The
    # copies run on their own stream, layer by layer, into one of two staging sets
    # (alternating by step), so step i+1's inputs arrive while step i computes; each
    # layer's calls wait only for that layer's inputs.
    stream = run.stream
    host_pool = []
    for i, p in enumerate(run.pool):
        host_pool.append(dict(q=[t.cpu().pin_memory() for t in p["q"]], k=[t.cpu().pin_memory() for t in p["k"]],
                              v=[t.cpu().pin_memory() for t in p["v"]], hid=run.hid_seq[i].cpu().pin_memory(),
                              lat=run.lat_seq[i].cpu().pin_memory()))
    stages = [dict(q=[torch.empty_like(t) for t in run.pool[0]["q"]], k=[torch.empty_like(t) for t in run.pool[0]["k"]],
                   v=[torch.empty_like(t) for t in run.pool[0]["v"]], hid=torch.empty_like(run.hid_seq[0]),
                   lat=torch.empty_like(run.lat_seq[0])) for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    landed = [[torch.cuda.Event() for _ in range(L + 1)] for _ in range(2)]   # per staging set: layer inputs in
    freed = [torch.cuda.Event() for _ in range(2)]                           # per staging set: last reader done
    res_out = torch.empty(tuple(run.out.shape), dtype=torch.bfloat16).pin_memory()
    res_rate = torch.empty(B, dtype=torch.float32).pin_memory()
    res_slot = torch.empty(B, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_pool[0]["q"] + host_pool[0]["k"] + host_pool[0]["v"])
    h2d += host_pool[0]["hid"].numel() * 2 + host_pool[0]["lat"].numel() * 4
    d2h = res_out.numel() * 2 + B * 8

    def e2e_step(i, hp):
        sg = stages[i % 2]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(freed[i % 2])
            for l in range(L):
                for key in ("q", "k", "v"):
                    sg[key][l].copy_(hp[key][l], non_blocking=True)
                landed[i % 2][l].record(copy_stream)
            sg["hid"].copy_(hp["hid"], non_blocking=True)
            sg["lat"].copy_(hp["lat"], non_blocking=True)
            landed[i % 2][L].record(copy_stream)
        run.step(sg, wait=lambda l: stream.wait_event(landed[i % 2][l]))
        freed[i % 2].record(stream)
        res_out.copy_(run.out, non_blocking=True)
        res_rate.copy_(run.rate, non_blocking=True)
        res_slot.copy_(run.out_slot, non_blocking=True)

    for i in range(2):
        freed[i].record(stream)
    e2e_step(0, host_pool[0])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    e0.record(stream)
    copy_stream.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i + 1, host_pool[i % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    # ---- the same step captured once as a CUDA graph and replayed: the library's host
    # work (ring bookkeeping, plans, launch set-up) leaves the timed region.  Every replay
    # repeats the captured step's slots and positions, so this is a timing of the
    # kernels as launched, reported beside the streamed value, not instead of it.
    graph_ms, graph_err, graph = 0.0, "", None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            run.step(run.pool[0])
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    except Exception as exc:                                   # reported, the streamed numbers stand
        graph_err = f"{type(exc).__name__}: {exc}"[:200]
    if pg:
        pg.barrier()                                           # every rank, whatever its capture did
    if not graph_err:
        try:
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            g1.record(stream)
            torch.cuda.synchronize()
            graph_ms = g0.elapsed_time(g1)
            assert run.cache.check() == 0 and run.mot.check() == 0, "device status word set"
        except Exception as exc:
            graph_err = f"{type(exc).__name__}: {exc}"[:200]
    del graph
    graph_fail = 1.0 if graph_err else 0.0

    if pg:
        ms, e2e_ms, graph_ms, graph_fail = max_over_ranks([ms, e2e_ms, graph_ms, graph_fail], pg, dev)
    frames = world * args.steps * B * Tp
    value = frames / (ms / 1e3)
    e2e_value = frames / (e2e_ms / 1e3)

    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    keys = steady_keys(w)
    flops = attn_flops(w, keys)
    abytes = attn_bytes(w, keys)
    attn_avg_s = call_us["attention"] / 1e6                  # whole call
    call_peak = peaks["bf16_tflops"] * (2.0 if kv_elem(w) == 1 else 1.0)
    achieved = flops / attn_avg_s / 1e12
    kv_gbs = abytes / attn_avg_s / 1e9
    Lq, N = run.Lq, w["frame_h"] * w["frame_w"]
    E = w["embed_dim"]
    kv_chunk = 2.0 * B * Lq * H * D * 2                      # K + V of the chunk, bf16
    append_bytes = kv_chunk + kv_chunk * kv_elem(w) / 2       # read (bf16) + written (bf16 or E4M3 codes)
    refresh_bytes = B * Lq * E * 2 + B * E * 8 * (w["sink_frames"] + 1)
    motion_bytes = B * (Tp + 2) * C * MH * MW * 4             # chunk + previous frame read, last frame written
    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3" if kv_elem(w) == 1 else "bf16",
        "data": "synthetic", "config": workload_config(name, w, world),
        "roofline": attention_roofline(w, name, call_us["attn_kernel"], peaks, peak_src),
        "rows": {
            "kv_append": ({"us": round(call_us["append"], 3), "bytes": append_bytes,
                           "gbs": round(append_bytes / call_us["append"] / 1e3, 1),
                           "frac_hbm": round(append_bytes / call_us["append"] / 1e3 / hbm, 4)}
                          if call_us["append"] is not None else
                          {"fused": "into the attention call (sdv2_append_attention)"}),
            "chunk_attention": {"us": round(call_us["attention"], 3), "tflops": round(achieved, 2),
                                "frac_tensor": round(achieved / call_peak, 4),
                                "kv_gbs": round(kv_gbs, 1), "frac_hbm": round(kv_gbs / hbm, 4),
                                "what": ("whole sdv2_append_attention call (append fused in): every kernel it "
                                         "launches" if w.get("fused") else
                                         "whole sdv2_chunk_attention call: every kernel it launches")},
            "sink_refresh": {"us": round(call_us["refresh"], 3), "bytes_without_copy": refresh_bytes,
                             "gbs": round(refresh_bytes / call_us["refresh"] / 1e3, 1)},
            "motion_noise_rate": {"us": round(call_us["motion"], 3), "bytes": motion_bytes,
                                  "gbs": round(motion_bytes / call_us["motion"] / 1e3, 1)},
            "note": "per-call times from a second pass with events around each call, each preceded by a "
                    "short device-side wait so the events time the GPU work, not the host's launch latency "
                    "(events serialise the dependent launches, so these are upper bounds of the in-step cost)"},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "cuda_graph": ({"value": round(frames / (graph_ms / 1e3), 3), "unit": UNIT,
                        "ms_per_step": round(graph_ms / args.steps, 4),
                        "what": "one captured step replayed (same slots and positions every replay)"}
                       if not graph_fail else {"unavailable": graph_err or "failed on another rank"}),
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    run.close()
    del run, stages, host_pool
    torch.cuda.empty_cache()
    if world == 1 and name == DEFAULT_WORKLOAD and not args.no_extra:
        result["workloads"] = {x: measure_extra(x, args, dev, peaks, peak_src) for x in EXTRA_WORKLOADS}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


# ----------------------------------------------------------------------------- oracle arms

def blas_threads():
    """Threads numpy's BLAS uses now (the oracle's matrix products run there)."""
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:                                   # pragma: no cover
        return None


def oracle_sample(w, threads=None):
    """Time the fp64 oracle on one layer of the workload's step (append + attention of
    every query of every stream) plus the refresh and motion of the step.  ``threads``
    limits numpy's BLAS threads (None: its default, every core).  Returns (time of the
    sample, time of the layer, time of refresh + motion) in seconds."""
    import contextlib

    import oracle as O
    import synth

    limit = contextlib.nullcontext()
    if threads is not None:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(limits=threads, user_api="blas")
    B, H, D = w["batch"], w["heads"], w["head_dim"]
    N = w["frame_h"] * w["frame_w"]
    Tp = w["chunk_frames"]
    Lq = Tp * N
    cfg = O.CacheConfig(batch=B, layers=1, heads=H, head_dim=D, frame_h=w["frame_h"], frame_w=w["frame_w"],
                        chunk_frames=Tp, sink_frames=w["sink_frames"], window_frames=w["window_frames"],
                        embed_dim=w["embed_dim"])
    if w.get("kv_format", "bf16") == "fp8":
        from oracle import sdv2_fp8 as F
        cache = F.OracleFp8Cache(cfg)
        append, attention, refresh = F.kv_append_fp8, F.chunk_attention_fp8, F.sink_refresh_fp8
    else:
        cache = O.OracleCache(cfg)
        append, attention, refresh = O.kv_append, O.chunk_attention, O.sink_refresh
    # fill to steady state (not timed)
    pre = (w["sink_frames"] + w["window_frames"] + Tp - 1) // Tp + 1
    for s in range(pre):
        _, k, v = synth.chunk_qkv(5, B, Lq, H, D, s, 0)
        append(cache, 0, synth.bf16_bits(k), synth.bf16_bits(v), [s * Tp] * B)
    mcfg = O.MotionConfig(batch=B, channels=w["motion"][0], height=w["motion"][1], width=w["motion"][2])
    mstate = O.MotionState(mcfg)
    lat = synth.motion_latents(5, B, Tp, *w["motion"], n_chunks=2)
    O.motion_noise_rate(mstate, next(lat).numpy())
    hid = next(synth.drifting_hidden(5, B, Lq, w["embed_dim"], 1))
    q, k, v = synth.chunk_qkv(5, B, Lq, H, D, pre, 0)
    f0 = [pre * Tp] * B
    x = next(lat).numpy()
    with limit:
        t0 = time.perf_counter()
        append(cache, 0, synth.bf16_bits(k), synth.bf16_bits(v), f0)
        attention(cache, 0, synth.bf16_bits(q), f0, 1.0 / math.sqrt(D))
        t1 = time.perf_counter()
        refresh(cache, synth.bf16_bits(hid), TAU, f0)
        O.motion_noise_rate(mstate, x)
        t2 = time.perf_counter()
    return t2 - t0, t1 - t0, t2 - t1


def _extrapolated_step(w, layer_s, rest_s):
    return layer_s * w["layers"] + rest_s


SAMPLE_TEXT = ("one sample = 1 of the {L} layers (append + attention of every query of every stream, fp64 "
               "numpy oracle) + the step's sink refresh and motion; full-step time extrapolated as "
               "{L} x layer + refresh + motion")


def cpu_baseline(w, samples=3):
    """The oracle on this host's cores: `samples` samples with numpy's default BLAS
    threading, and one with a single BLAS thread."""
    runs = [oracle_sample(w) for _ in range(samples)]
    layer_s = statistics.median(r[1] for r in runs)
    rest_s = statistics.median(r[2] for r in runs)
    one = oracle_sample(w, threads=1)
    frames = w["batch"] * w["chunk_frames"]
    step_s = _extrapolated_step(w, layer_s, rest_s)
    step1 = _extrapolated_step(w, one[1], one[2])
    return {"value": round(frames / step_s, 5), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "blas_threads": blas_threads(),
            "single_thread_value": round(frames / step1, 5),
            "sample": SAMPLE_TEXT.format(L=w["layers"]) + f"; median of {samples} samples with numpy's default "
                      f"BLAS threads (layer {layer_s:.2f} s), plus one with 1 BLAS thread (layer {one[1]:.2f} s)"}


def run_reference(args, w, name):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    layer, rest, sample = [], [], []
    for i in range(args.warmup + args.steps):
        s, l, r = oracle_sample(w)
        if i >= args.warmup:
            sample.append(s)
            layer.append(l)
            rest.append(r)
    step_s = _extrapolated_step(w, statistics.mean(layer), statistics.mean(rest))
    one = oracle_sample(w, threads=1)
    frames = w["batch"] * w["chunk_frames"]
    value = frames / step_s
    sample_text = SAMPLE_TEXT.format(L=w["layers"]) + (
        f"; each of the {args.steps} timed steps is one sample with numpy's default BLAS threads "
        f"({blas_threads()} threads on {os.cpu_count()} cores)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(statistics.mean(sample) * 1e3, 3),
        "step_is": "one sample (1 of the layers + refresh + motion); value is over the extrapolated full step",
        "ms_per_full_step_extrapolated": round(step_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(name, w, world), "gpu_launches": 0,
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                         "blas_threads": blas_threads(),
                         "single_thread_value": round(frames / _extrapolated_step(w, one[1], one[2]), 5),
                         "sample": sample_text},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the extra workloads timed beside the default one")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, args.workload)
    else:
        run_ours(args, w, args.workload)


if __name__ == "__main__":
    main()

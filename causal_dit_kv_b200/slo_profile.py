"""Measure L(T, B) of the streaming step on this GPU and fit the scheduler's model.

    python -m causal_dit_kv_b200.slo_profile [--workload wan1.3b-512x512] [--batches 1,2,4,8]
                                             [--target-fps 16] [--steps 1]

For each stream batch B, one step = every layer's sdv2_kv_append +
sdv2_chunk_attention, then sdv2_sink_refresh and sdv2_motion_noise_rate, on
seeded synthetic inputs already on the device, timed with CUDA events after
warm-up.  The (n*B*T, latency) points are fitted to L = alpha + beta*n*B*T
(causal_dit_kv_b200.scheduler) and the batch the SLO rule picks for the target
per-stream frame rate is printed as one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math


def measure_step_latency(shape: dict, batch: int, steps: int = 3, warmup: int = 3, seed: int = 7) -> float:
    """Mean device time of one streaming step (seconds) for `batch` streams."""
    import torch

    from causal_dit_kv_b200 import KVCache, MotionState

    L, H, D = shape["layers"], shape["heads"], shape["head_dim"]
    Tp, S, W = shape["chunk_frames"], shape["sink_frames"], shape["window_frames"]
    N = shape["frame_h"] * shape["frame_w"]
    Lq, E = Tp * N, shape["embed_dim"]
    C, MH, MW = shape["motion"]
    cache = KVCache(batch, L, H, D, shape["frame_h"], shape["frame_w"], Tp, S, W, embed_dim=E,
                    kv_format=shape.get("kv_format", "bf16"))
    mot = MotionState(batch, Tp, C, MH, MW)
    g = torch.Generator(device="cuda").manual_seed(seed)
    mk = lambda *s: torch.randn(s, generator=g, device="cuda").to(torch.bfloat16)
    q, k, v = mk(batch, Lq, H, D), mk(batch, Lq, H, D), mk(batch, Lq, H, D)
    hid = mk(batch, Lq, E)
    lat = torch.randn((batch, Tp, C, MH, MW), generator=g, device="cuda")
    out = torch.empty_like(q)
    slot = torch.empty(batch, dtype=torch.int32, device="cuda")
    rate = torch.empty(batch, dtype=torch.float32, device="cuda")
    frame = [0]

    def step():
        f0 = [frame[0]] * batch
        for layer in range(L):
            cache.kv_append(layer, k, v, f0)
            cache.chunk_attention(layer, q, out, f0, 1.0 / math.sqrt(D))
        cache.sink_refresh(hid, 0.9, f0, slot)
        mot.noise_rate(lat, rate)
        frame[0] += Tp

    for _ in range((S + W) // Tp + 1 + warmup):          # ring full, then warm
        step()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    assert cache.check() == 0 and mot.check() == 0
    cache.close()
    mot.close()
    return t0.elapsed_time(t1) / 1e3 / steps


def main():
    from causal_dit_kv_b200.profile_case import SHAPES as WORKLOADS
    from causal_dit_kv_b200.scheduler import choose_batch, fit_from_measurements, knee_batch

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="wan1.3b-512x512", choices=sorted(WORKLOADS))
    ap.add_argument("--batches", default="1,2,4,8")
    ap.add_argument("--target-fps", type=float, default=16.0)
    ap.add_argument("--denoise-steps", type=int, default=1)
    a = ap.parse_args()
    shape = WORKLOADS[a.workload]
    t = shape["chunk_frames"]
    pts = []
    for b in [int(x) for x in a.batches.split(",")]:
        lat = measure_step_latency(shape, b)
        pts.append((t, b, 1, lat))
    model = fit_from_measurements(pts)
    b_slo = choose_batch(model, t, a.target_fps, frames_available=64 * t, steps=a.denoise_steps)
    print(json.dumps({"workload": a.workload, "points": [{"B": b, "T": t, "latency_ms": round(l * 1e3, 4)}
                                                          for t, b, _, l in pts],
                      "alpha_ms": round(model.alpha * 1e3, 4), "beta_ms_per_frame": round(model.beta * 1e3, 5),
                      "target_fps_per_stream": a.target_fps, "denoise_steps": a.denoise_steps,
                      "chosen_batch": b_slo, "knee_batch": knee_batch(model, t, a.denoise_steps)}))


if __name__ == "__main__":
    main()

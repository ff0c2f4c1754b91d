"""Small, self-contained launches of one kernel of the path, for ncu captures.

    python -m causal_dit_kv_b200.profile_case --kernel attention [--workload wan1.3b-512x512]

Sets up one layer of the named workload's cache at steady state (ring full)
with a handful of appends, then runs the requested call once (append_attention:
the next chunk's append fused into its attention); the ncu capture selects the
kernel with -k.  Device memory stays well under 1 GB.
"""
from __future__ import annotations

import argparse
import math

SHAPES = {
    "wan1.3b-512x512": dict(batch=1, layers=30, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                            sink_frames=1, window_frames=6, embed_dim=1536, motion=(16, 64, 64)),
    "wan1.3b-480x832-b4": dict(batch=4, layers=30, heads=12, head_dim=128, frame_h=30, frame_w=52, chunk_frames=2,
                               sink_frames=1, window_frames=8, embed_dim=1536, motion=(16, 60, 104)),
    "wan1.3b-128x128-b16": dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=8, chunk_frames=1,
                                sink_frames=1, window_frames=6, embed_dim=1536, motion=(16, 16, 16)),
    "wan1.3b-512x512-fp8": dict(batch=1, layers=30, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                                sink_frames=1, window_frames=6, embed_dim=1536, motion=(16, 64, 64), kv_format="fp8"),
    "wan1.3b-128x256-b16": dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=16, chunk_frames=1,
                                sink_frames=1, window_frames=6, embed_dim=1536, motion=(16, 16, 32)),
    "wan1.3b-128x256-b16-fp8": dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=16,
                                    chunk_frames=1, sink_frames=1, window_frames=6, embed_dim=1536,
                                    motion=(16, 16, 32), kv_format="fp8"),
    "wan1.3b-128x128-b16-fp8": dict(batch=16, layers=30, heads=12, head_dim=128, frame_h=8, frame_w=8,
                                    chunk_frames=1, sink_frames=1, window_frames=6, embed_dim=1536,
                                    motion=(16, 16, 16), kv_format="fp8"),
    "wan14b-512x512-b1": dict(batch=1, layers=40, heads=40, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                              sink_frames=1, window_frames=6, embed_dim=5120, motion=(16, 64, 64)),
}


def main():
    import torch

    from causal_dit_kv_b200 import KVCache, MotionState

    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["attention", "append", "append_attention", "refresh", "motion"],
                    default="attention")
    ap.add_argument("--workload", choices=sorted(SHAPES), default="wan1.3b-512x512")
    ap.add_argument("--repeat", type=int, default=1)
    a = ap.parse_args()
    w = SHAPES[a.workload]
    B, H, D, Tp = w["batch"], w["heads"], w["head_dim"], w["chunk_frames"]
    N = w["frame_h"] * w["frame_w"]
    Lq = Tp * N
    cache = KVCache(B, 1, H, D, w["frame_h"], w["frame_w"], Tp, w["sink_frames"], w["window_frames"],
                    embed_dim=w["embed_dim"], kv_format=w.get("kv_format", "bf16"))
    g = torch.Generator(device="cuda").manual_seed(3)
    k = torch.randn((B, Lq, H, D), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Lq, H, D), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((B, Lq, H, D), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(q)
    n_pre = (w["sink_frames"] + w["window_frames"]) // Tp + 1
    frame = 0
    for _ in range(n_pre):
        cache.kv_append(0, k, v, [frame] * B)
        frame += Tp
    f0 = [frame - Tp] * B
    if a.kernel == "attention":
        for _ in range(a.repeat):
            cache.chunk_attention(0, q, out, f0, 1.0 / math.sqrt(D))
    elif a.kernel == "append_attention":
        for _ in range(a.repeat):
            cache.append_attention(0, q, k, v, out, [frame] * B, 1.0 / math.sqrt(D))
            frame += Tp
    elif a.kernel == "append":
        for _ in range(a.repeat):
            cache.kv_append(0, k, v, [frame] * B)
            frame += Tp
    elif a.kernel == "refresh":
        hid = torch.randn((B, Lq, w["embed_dim"]), generator=g, device="cuda").to(torch.bfloat16)
        slot = torch.empty(B, dtype=torch.int32, device="cuda")
        for _ in range(a.repeat):
            cache.sink_refresh(hid, 0.9, f0, slot)
    else:
        C, MH, MW = w["motion"]
        mot = MotionState(B, Tp, C, MH, MW)
        lat = torch.randn((B, Tp, C, MH, MW), generator=g, device="cuda")
        rate = torch.empty(B, dtype=torch.float32, device="cuda")
        for _ in range(a.repeat + 1):
            mot.noise_rate(lat, rate)
    torch.cuda.synchronize()
    assert cache.check() == 0
    print("profile case done:", a.kernel, a.workload)


if __name__ == "__main__":
    main()

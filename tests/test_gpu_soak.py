"""Long-stream soak on the Wan-1.3B 512x512 layer shape (B200).

2000 streamed chunks through one layer: RoPE phase reset every 256 frames,
cosine sink refresh (tau = 0.9) on seeded drifting chunk embeddings with scene
cuts, motion noise rate on 16x64x64 latents with a seeded piecewise-constant
motion schedule.  Every step's refresh decision, sink record and noise rate is
compared with the oracle; the cache bit for bit every 100 steps and around
every refresh; attention on sampled query rows at wraps, resets and refreshes.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from harness import ATTN_MAX_ABS, ATTN_MEAN_ABS, MOTION_REL, PairedStream, attn_errors, cache_bits_equal, f32

pytestmark = pytest.mark.gpu

N_CHUNKS = 2000


def test_soak_2000_chunks():
    from causal_dit_kv_b200 import MotionState as GpuMotion
    cfg = dict(batch=1, layers=1, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1, sink_frames=1,
               window_frames=6, rope_reset_period=256, embed_dim=1536)
    ps = PairedStream(seed=1005, **cfg)
    c = ps.cfg
    mcfg = O.MotionConfig(batch=1, channels=16, height=64, width=64, window=4, sigma=2.0, lam=0.9)
    ora_m = O.MotionState(mcfg)
    gpu_m = GpuMotion(1, 1, 16, 64, 64, window=4, sigma=2.0, lam=0.9)
    hid_gen = synth.drifting_hidden(5005, 1, c.chunk_tokens, c.embed_dim, N_CHUNKS, drift=0.05, cut_prob=0.01)
    lat_gen = synth.motion_latents(5005, 1, 1, 16, 64, 64, N_CHUNKS)
    out_slot = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    rate = torch.zeros(1, dtype=torch.float32, device="cuda")
    rows = np.arange(0, c.chunk_tokens, 61)
    refreshes = 0
    sampled = 0
    prev_fired = False
    for step in range(N_CHUNKS):
        ps.step_idx = step
        f0 = ps.advance()
        q, k, v = ps.inputs(0)
        ps.append(0, f0, k, v)
        f = f0[0]
        event = (f % 256 in (0, 1, 255)) or (f >= 7 and (f - 1) % 6 in (0, 5) and f < 40) or prev_fired \
            or step == N_CHUNKS - 1
        if event:
            out, want = ps.attention(0, f0, q, rows=rows)
            mx, mean = attn_errors(out, want, rows)
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (step, mx, mean)
            sampled += 1
        hid = next(hid_gen)
        ps.gpu.sink_refresh(hid.cuda(), 0.9, f0, out_slot)
        want_slot = O.sink_refresh(ps.ora, synth.bf16_bits(hid), f32(0.9), f0)
        x = next(lat_gen)
        gpu_m.noise_rate(x.cuda(), rate)
        want_rate, _ = O.motion_noise_rate(ora_m, x.numpy())
        got_slot = int(out_slot.item())
        assert got_slot == int(want_slot[0]), (step, got_slot, want_slot)
        got_rate = float(rate.item())
        assert abs(got_rate - want_rate[0]) <= MOTION_REL * abs(want_rate[0]), (step, got_rate, want_rate)
        prev_fired = got_slot >= 0
        refreshes += int(prev_fired)
        if step % 100 == 0 or prev_fired:
            k_ok, v_ok, _, _ = cache_bits_equal(ps, 0)
            assert k_ok and v_ok, step
            assert np.array_equal(ps.gpu.sink_frame().cpu().numpy(), ps.ora.sink_frame)
    assert 5 <= refreshes <= 200, refreshes
    assert sampled >= 20
    assert ps.gpu.check() == 0 and gpu_m.check() == 0

"""Sink refresh and motion/EMA kernels vs the oracle (B200).

Refresh decisions, sink records and cache contents bit for bit; chunk-mean
embeddings to fp64 rounding; motion values and noise rates within 1e-4
relative.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from harness import MOTION_REL, PairedStream, cache_bits_equal, f32

pytestmark = pytest.mark.gpu


def _run_refresh(cfg, n_chunks, tau, seed, drift, cut):
    ps = PairedStream(seed=seed, **cfg)
    c = ps.cfg
    hidden_gen = synth.drifting_hidden(seed, c.batch, c.chunk_tokens, c.embed_dim, n_chunks, drift=drift,
                                       cut_prob=cut)
    out_slot = torch.full((c.batch,), -7, dtype=torch.int32, device="cuda")
    fired = 0
    for step in range(n_chunks):
        ps.step_idx = step
        f0 = ps.advance()
        for layer in range(c.layers):
            _, k, v = ps.inputs(layer)
            ps.append(layer, f0, k, v)
        hid = next(hidden_gen)
        ps.gpu.sink_refresh(hid.cuda(), tau, f0, out_slot)
        want = O.sink_refresh(ps.ora, synth.bf16_bits(hid), f32(tau), f0)
        got = out_slot.cpu().numpy().astype(np.int64)
        assert np.array_equal(got, want), (step, got, want)
        fired += int((want >= 0).sum())
        assert np.array_equal(ps.gpu.sink_frame().cpu().numpy(), ps.ora.sink_frame), step
        emb = ps.gpu.sink_embed().cpu().numpy()
        np.testing.assert_allclose(emb, ps.ora.sink_embed, rtol=1e-12, atol=1e-14)
        if step % 5 == 0 or want.max() >= 0:
            for layer in range(c.layers):
                k_ok, v_ok, _, _ = cache_bits_equal(ps, layer)
                assert k_ok and v_ok, (step, layer)
    return fired


def test_refresh_small_many_events():
    cfg = dict(batch=2, layers=2, heads=2, head_dim=64, frame_h=4, frame_w=4, chunk_frames=1, sink_frames=3,
               window_frames=2, embed_dim=64)
    fired = _run_refresh(cfg, 40, 0.9, seed=2001, drift=2.0, cut=0.1)
    assert fired >= 5


def test_refresh_two_frame_chunks():
    cfg = dict(batch=3, layers=1, heads=2, head_dim=64, frame_h=4, frame_w=6, chunk_frames=2, sink_frames=1,
               window_frames=4, embed_dim=128, rope_reset_period=5)
    fired = _run_refresh(cfg, 25, 0.8, seed=2002, drift=3.0, cut=0.2)
    assert fired >= 3


def test_refresh_full_width_1536():
    cfg = dict(batch=1, layers=2, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1, sink_frames=1,
               window_frames=6, embed_dim=1536)
    _run_refresh(cfg, 10, 0.9, seed=2003, drift=1.0, cut=0.2)


def _run_motion(batch, chunk_frames, C, H, W, n_chunks, seed, **kw):
    from causal_dit_kv_b200 import MotionState as GpuMotion
    mcfg = O.MotionConfig(batch=batch, channels=C, height=H, width=W, **kw)
    ora = O.MotionState(mcfg)
    gpu = GpuMotion(batch, chunk_frames, C, H, W, window=mcfg.window, sigma=mcfg.sigma, lam=mcfg.lam,
                    s_min=mcfg.s_min, s_max=mcfg.s_max, s_init=mcfg.s_init)
    rate = torch.zeros(batch, dtype=torch.float32, device="cuda")
    d = torch.zeros((batch, chunk_frames), dtype=torch.float32, device="cuda")
    gen = synth.motion_latents(seed, batch, chunk_frames, C, H, W, n_chunks, sigma=mcfg.sigma)
    worst = 0.0
    for _ in range(n_chunks):
        x = next(gen)
        gpu.noise_rate(x.cuda(), rate, d)
        want_rate, want_d = O.motion_noise_rate(ora, x.numpy())
        g_rate = rate.cpu().numpy().astype(np.float64)
        g_d = d.cpu().numpy().astype(np.float64)
        rel_r = np.abs(g_rate - want_rate) / np.abs(want_rate)
        assert rel_r.max() <= MOTION_REL, rel_r
        first = want_d < 0
        assert np.array_equal(g_d[first], want_d[first])
        nz = ~first & (want_d > 0)
        rel_d = np.abs(g_d[nz] - want_d[nz]) / want_d[nz]
        assert rel_d.size == 0 or rel_d.max() <= MOTION_REL
        assert np.all(g_d[~first & (want_d == 0)] == 0)
        worst = max(worst, float(rel_r.max()))
    return worst


def test_motion_tiny_16ch_4x4():
    _run_motion(1, 1, 16, 4, 4, 30, seed=3001, window=4, sigma=2.0, lam=0.9)


def test_motion_64x64_multi_block_and_chunks():
    _run_motion(2, 2, 16, 64, 64, 40, seed=3002, window=4, sigma=2.0, lam=0.9)


def test_motion_odd_size():
    _run_motion(3, 3, 3, 17, 29, 10, seed=3003, window=2, sigma=1.0, lam=0.5)

"""The KV append fused into the chunk attention (sdv2_append_attention) vs the fp64
oracle's append followed by its attention, through the C ABI (B200).

The cache is compared bit for bit with the oracle after every fused call (the
fused kernel writes the chunk's rows itself, rotated by the append's rule), the
attention output within the same bounds as the plain attention.  The cases cover
the pair mode, KV splits with the assembled tile in one piece, chunk rows that
straddle two KV tiles, two query tiles, ring wrap with T' = 2, streams in several
phases in one launch, calls that
fall back to two launches, and fused and plain calls mixed on one cache.
"""
import numpy as np
import pytest

from harness import ATTN_MAX_ABS, ATTN_MEAN_ABS, PairedStream, attn_errors, cache_bits_equal

pytestmark = pytest.mark.gpu

SMS = 148


def _run(ps: PairedStream, n_steps: int, active_fn=None, check_every=1, plain_fn=None):
    """Step the paired stream; returns the fused-kernel mode of every call (0: two launches)."""
    from causal_dit_kv_b200 import binding as B
    modes = []
    for step in range(n_steps):
        ps.step_idx = step
        f0 = ps.advance(active_fn(step) if active_fn else None)
        for layer in range(ps.cfg.layers):
            q, k, v = ps.inputs(layer)
            if plain_fn is not None and plain_fn(step):
                ps.append(layer, f0, k, v)
                out, want = ps.attention(layer, f0, q)
                modes.append(None)
            else:
                modes.append(B.sdv2_append_attention_mode(ps.gpu.cfg, f0, SMS))
                out, want = ps.append_attention(layer, f0, q, k, v)
            mx, mean = attn_errors(out, want)
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (step, layer, mx, mean)
            if step % check_every == 0 or step == n_steps - 1:
                k_ok, v_ok, _, _ = cache_bits_equal(ps, layer)
                assert k_ok and v_ok, (step, layer, k_ok, v_ok)
    assert ps.gpu.check() == 0
    return modes


def test_fused_small_chunks_pair_mode():
    """The 128x128 small-chunk shape (64 tokens per frame, 12 heads x 128, 1 sink + 6 window
    frames, 16 streams, one joining late): one KV tile holds each stream's chunk, 192 units."""
    cfg = dict(batch=16, layers=1, heads=12, head_dim=128, frame_h=8, frame_w=8, chunk_frames=1, sink_frames=1,
               window_frames=6)
    ps = PairedStream(seed=2001, **cfg)
    modes = _run(ps, 9, check_every=2, active_fn=lambda s: set(range(15)) if s < 3 else set(range(16)))
    assert set(modes) == {2}


def test_fused_split_pieces_d64():
    """Four (stream, head) units on 148 SMs: every unit is split over the KV range, the
    chunk's tile lands in one piece (first in its order), the merge combines them."""
    from causal_dit_kv_b200 import binding as B
    cfg = dict(batch=1, layers=2, heads=4, head_dim=64, frame_h=8, frame_w=8, chunk_frames=1, sink_frames=1,
               window_frames=6)
    ps = PairedStream(seed=2002, **cfg)
    assert B.sdv2_attention_splits(ps.gpu.cfg, [448], SMS) > 1
    modes = _run(ps, 10)
    assert set(modes) == {1}


def test_fused_chunk_rows_straddle_two_tiles():
    """96 tokens per frame: a slot's rows cross a 128-key tile boundary at most positions,
    so two assembled tiles (both K stages) come first; d = 128, 2 sinks, ring wrap."""
    cfg = dict(batch=2, layers=1, heads=3, head_dim=128, frame_h=8, frame_w=12, chunk_frames=1, sink_frames=2,
               window_frames=4, rope_reset_period=5)
    ps = PairedStream(seed=2003, **cfg)
    modes = _run(ps, 11, active_fn=lambda s: {0, 1} if s >= 2 else {0})
    assert set(modes) == {1}


def test_fused_pair_mode_odd_heads_ragged_staggered():
    """Odd head count (the last head of a stream runs alone), d = 64, 60 tokens per frame
    (ragged tiles; a slot may straddle two tiles, which takes that launch out of the pair
    mode) and streams joining at different steps."""
    cfg = dict(batch=12, layers=2, heads=13, head_dim=64, frame_h=6, frame_w=10, chunk_frames=1, sink_frames=1,
               window_frames=3)
    ps = PairedStream(seed=2004, **cfg)
    modes = _run(ps, 8, check_every=3, active_fn=lambda s: {b for b in range(12) if s >= b % 2})
    assert 2 in modes and 1 in modes


def test_fused_two_frames_ring_wrap_reset():
    """T' = 2 (two new slots, not adjacent when the window wraps), temporal phase reset
    every 3 frames, three streams at staggered positions."""
    cfg = dict(batch=3, layers=1, heads=2, head_dim=128, frame_h=8, frame_w=8, chunk_frames=2, sink_frames=1,
               window_frames=3, rope_reset_period=3)
    ps = PairedStream(seed=2005, **cfg)
    modes = _run(ps, 9, active_fn=lambda s: {b for b in range(3) if s >= b})
    assert set(modes) == {1}


def test_fused_two_query_tiles_and_fallback():
    """96 tokens per frame and T' = 2: 192 queries (two query tiles in one CTA).  Where the
    chunk's two slots touch three tiles the call runs the append and the attention as two
    launches instead; both kinds of step occur."""
    cfg = dict(batch=2, layers=1, heads=2, head_dim=64, frame_h=8, frame_w=12, chunk_frames=2, sink_frames=1,
               window_frames=4)
    ps = PairedStream(seed=2006, **cfg)
    modes = _run(ps, 8, active_fn=lambda s: {0, 1} if s >= 1 else {0})
    assert 0 in modes and 1 in modes


def test_fused_many_phases_several_launches():
    """16 streams joining one step apart, no phase reset: 16 distinct temporal phases in one
    launch, each CTA copying its stream's rows of the cache's phase table."""
    cfg = dict(batch=16, layers=1, heads=2, head_dim=128, frame_h=4, frame_w=8, chunk_frames=1, sink_frames=1,
               window_frames=4)
    ps = PairedStream(seed=2007, **cfg)
    modes = _run(ps, 16, check_every=5, active_fn=lambda s: {b for b in range(16) if s >= b})
    assert set(modes) == {1}


def test_fused_and_plain_calls_mixed_and_large_chunk_fallback():
    """Fused and plain calls alternate on one cache (the frame bookkeeping is shared); a
    chunk of 512 queries never takes the fused kernel."""
    cfg = dict(batch=2, layers=2, heads=2, head_dim=64, frame_h=8, frame_w=8, chunk_frames=1, sink_frames=1,
               window_frames=4)
    ps = PairedStream(seed=2008, **cfg)
    _run(ps, 7, plain_fn=lambda s: s % 2 == 1)
    big = dict(batch=1, layers=1, heads=2, head_dim=64, frame_h=16, frame_w=16, chunk_frames=2, sink_frames=1,
               window_frames=2)
    ps2 = PairedStream(seed=2009, **big)
    assert set(_run(ps2, 4)) == {0}


def test_fused_skipped_streams_and_empty_call():
    import torch
    cfg = dict(batch=3, layers=1, heads=2, head_dim=64, frame_h=4, frame_w=4, chunk_frames=1, sink_frames=1,
               window_frames=2)
    ps = PairedStream(seed=2010, **cfg)
    q, k, v = ps.inputs(0)
    out = torch.full((3, 16, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    ps.gpu.append_attention(0, q.cuda(), k.cuda(), v.cuda(), out, [-1, -1, -1])
    assert torch.all(out == 7.0)
    modes = _run(ps, 5, active_fn=lambda s: {1} if s % 2 else {0, 2})
    assert set(modes) == {1}
    assert np.isfinite(out.float().cpu().numpy()).all()

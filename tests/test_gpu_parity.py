"""CUDA path vs the fp64 oracle, element by element, through the C ABI (B200).

Cache contents and ring indices are compared bit for bit; attention outputs
within 1.5e-2 max abs and 2e-3 mean abs error of the oracle evaluated on the
same bf16 inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from harness import ATTN_MAX_ABS, ATTN_MEAN_ABS, PairedStream, attn_errors, cache_bits_equal

pytestmark = pytest.mark.gpu

TINY = dict(batch=1, layers=1, heads=2, head_dim=64, frame_h=4, frame_w=4, chunk_frames=1, sink_frames=1,
            window_frames=2)


def _stream_and_check(ps: PairedStream, n_steps: int, check_every=1, attn_rows=None, active_fn=None):
    errs = []
    for step in range(n_steps):
        ps.step_idx = step
        active = active_fn(step) if active_fn else None
        f0 = ps.advance(active)
        for layer in range(ps.cfg.layers):
            q, k, v = ps.inputs(layer)
            ps.append(layer, f0, k, v)
            out, want = ps.attention(layer, f0, q, rows=attn_rows)
            mx, mean = attn_errors(out, want, attn_rows)
            errs.append((step, layer, mx, mean))
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (step, layer, mx, mean)
            if step % check_every == 0 or step == n_steps - 1:
                k_ok, v_ok, _, _ = cache_bits_equal(ps, layer)
                assert k_ok and v_ok, (step, layer, k_ok, v_ok)
    return errs


def test_tiny_stream_8_chunks():
    ps = PairedStream(seed=1001, **TINY)
    _stream_and_check(ps, 8)
    assert ps.gpu.check() == 0


def test_tiny_stream_d128_literal_split():
    cfg = dict(TINY, head_dim=128, rope_pairs=(22, 21, 21), rope_reset_period=3)
    ps = PairedStream(seed=1011, **cfg)
    _stream_and_check(ps, 8)


def test_ring_indices_match_oracle():
    ps = PairedStream(seed=1002, **dict(TINY, sink_frames=2, window_frames=3, chunk_frames=1, rope_reset_period=4))
    for step in range(11):
        ps.step_idx = step
        f0 = ps.advance()
        q, k, v = ps.inputs(0)
        ps.append(0, f0, k, v)
        frames, phases, valid = ps.gpu.query(0, 0)
        f_end = f0[0] + 1
        want = O.slot_frames(f_end, 2, 3)
        assert frames == want
        assert phases == [O.rope_phase(f, 4) if f >= 0 else -1 for f in want]
        assert valid == sum(O.valid_slot_counts(f_end, 2, 3))


def test_multi_tile_ragged_split_path():
    # Lq = 480 (one full and one ragged query-tile pair), Lk up to 960 (ragged
    # last KV tile), 3 streams with one joining late, phase reset every 3.
    from causal_dit_kv_b200 import binding as B
    cfg = dict(batch=3, layers=2, heads=2, head_dim=128, frame_h=12, frame_w=20, chunk_frames=2, sink_frames=1,
               window_frames=3, rope_reset_period=3)
    ps = PairedStream(seed=1003, **cfg)
    splits = B.sdv2_attention_splits(ps.gpu.cfg, [960, 960, 960], 148)
    assert splits > 1
    _stream_and_check(ps, 6, active_fn=lambda s: {0, 1} if s < 2 else {0, 1, 2})


@pytest.mark.parametrize("head_dim", [128, 64])
def test_single_tile_chunks_split_and_ragged(head_dim):
    # 80 queries (one query tile: the two accumulator sets take alternate KV tiles and
    # are merged in the CTA), 480 keys in 4 tiles with a ragged last one, split over the
    # KV range so that some splits hold a single tile (one accumulator set unused).
    from causal_dit_kv_b200 import binding as B
    cfg = dict(batch=2, layers=1, heads=3, head_dim=head_dim, frame_h=8, frame_w=10, chunk_frames=1, sink_frames=1,
               window_frames=5)
    ps = PairedStream(seed=1010 + head_dim, **cfg)
    assert B.sdv2_attention_splits(ps.gpu.cfg, [480, 480], 148) > 1
    _stream_and_check(ps, 8)


def test_small_chunk_many_streams():
    """The 128x128 small-chunk shape: 64 tokens per frame, 12 heads x 128, 1 sink + 6
    window frames, 16 independent streams, one of them starting late."""
    cfg = dict(batch=16, layers=1, heads=12, head_dim=128, frame_h=8, frame_w=8, chunk_frames=1, sink_frames=1,
               window_frames=6)
    ps = PairedStream(seed=1012, **cfg)
    from causal_dit_kv_b200 import binding as B
    assert B.sdv2_attention_pair_mode(ps.gpu.cfg, [448] * 16, 148) == 1     # 192 single-tile units: pair mode
    _stream_and_check(ps, 9, check_every=4, active_fn=lambda s: set(range(15)) if s < 3 else set(range(16)))


def test_pair_mode_odd_heads_staggered_streams():
    """Pair mode with an odd head count (the last head of every stream runs alone, both
    accumulator sets on its one query tile), d = 64, 60 tokens per frame (a ragged query
    tile and ragged key tiles) and streams joining at different steps, so their key
    counts differ while the two heads of a CTA always share one."""
    from causal_dit_kv_b200 import binding as B
    cfg = dict(batch=12, layers=2, heads=13, head_dim=64, frame_h=6, frame_w=10, chunk_frames=1, sink_frames=1,
               window_frames=3)
    ps = PairedStream(seed=1013, **cfg)
    assert B.sdv2_attention_pair_mode(ps.gpu.cfg, [240] * 12, 148) == 1     # 156 units
    _stream_and_check(ps, 8, active_fn=lambda s: {b for b in range(12) if s >= b % 4})


def test_many_heads_unsplit_path():
    # 37 heads x 4 query-tile pairs = 148 CTAs, one full wave: no KV split
    from causal_dit_kv_b200 import binding as B
    cfg = dict(batch=1, layers=1, heads=37, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1, sink_frames=1,
               window_frames=1)
    ps = PairedStream(seed=1004, **cfg)
    assert B.sdv2_attention_splits(ps.gpu.cfg, [2048], 148) == 1
    rows = np.sort(np.random.default_rng(4).choice(1024, 48, replace=False))
    _stream_and_check(ps, 4, attn_rows=rows)


def test_window_equals_chunk_and_reset_every_frame():
    cfg = dict(batch=2, layers=1, heads=3, head_dim=64, frame_h=8, frame_w=10, chunk_frames=2, sink_frames=2,
               window_frames=2, rope_reset_period=1)
    ps = PairedStream(seed=1005, **cfg)
    _stream_and_check(ps, 5)


def test_skipped_streams_and_empty_call():
    ps = PairedStream(seed=1006, **dict(TINY, batch=3))
    before = torch.zeros(1)
    f0 = [-1, -1, -1]
    q, k, v = ps.inputs(0)
    n0 = ps.gpu.layout.total_bytes
    ps.gpu.kv_append(0, k.cuda(), v.cuda(), f0)        # nothing to do
    out = torch.full((3, 16, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    ps.gpu.chunk_attention(0, q.cuda(), out, f0)
    assert torch.all(out == 7.0)                      # untouched
    assert n0 > 0 and before.numel() == 1
    _stream_and_check(ps, 4, active_fn=lambda s: {1} if s % 2 else {0, 2})


def test_state_errors():
    from causal_dit_kv_b200 import SDV2Error
    from causal_dit_kv_b200 import binding as B
    ps = PairedStream(seed=1007, **TINY)
    q, k, v = ps.inputs(0)
    with pytest.raises(SDV2Error) as e:
        ps.gpu.kv_append(0, k.cuda(), v.cuda(), [3])   # frame 3 before 0..2
    assert e.value.status == B.SDV2_E_STATE
    out = torch.empty((1, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(SDV2Error) as e:
        ps.gpu.chunk_attention(0, q.cuda(), out, [0])  # attention before append
    assert e.value.status == B.SDV2_E_STATE
    kk = k.cuda()
    with pytest.raises(SDV2Error) as e:
        B.sdv2_kv_append(ps.gpu.handle, 0, kk.data_ptr() + 2, v.cuda(), [0], 1)
    assert e.value.status == B.SDV2_E_ALIGN
    with pytest.raises(SDV2Error) as e:
        ps.gpu.kv_append(5, k.cuda(), v.cuda(), [0])
    assert e.value.status == B.SDV2_E_ARG


@pytest.mark.parametrize("steps", [9])
def test_full_size_1p3b_512_sampled(steps):
    """Wan-1.3B-shaped layer at 512x512 (12 heads x 128, 32x32 tokens, 1 sink + 6 window
    frames), streamed past the ring wrap; cache compared bit for bit, attention on
    sampled query rows (all heads) in the launch configuration the benchmark uses."""
    cfg = dict(batch=1, layers=1, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1, sink_frames=1,
               window_frames=6)
    ps = PairedStream(seed=1001, **cfg)
    rows = np.sort(np.random.default_rng(0).choice(1024, 96, replace=False))
    _stream_and_check(ps, steps, check_every=4, attn_rows=rows)


def test_full_size_1p3b_480p_sampled():
    """1.3B shape at 480x832: 30x52 = 1560 tokens per frame, T' = 2, 1 sink + 8 window,
    4 independent streams at different positions (frames 0, 4, 18 and 40)."""
    cfg = dict(batch=4, layers=1, heads=12, head_dim=128, frame_h=30, frame_w=52, chunk_frames=2, sink_frames=1,
               window_frames=8)
    ps = PairedStream(seed=1002, **cfg)
    starts = [0, 4, 18, 40]
    # warm-up: advance each stream alone to its start frame
    step = 0
    while any(ps.next[b] < starts[b] for b in range(4)):
        ps.step_idx = 1000 + step
        active = {b for b in range(4) if ps.next[b] < starts[b]}
        f0 = ps.advance(active)
        _, k, v = ps.inputs(0)
        ps.append(0, f0, k, v)
        step += 1
    rows = np.sort(np.random.default_rng(1).choice(3120, 64, replace=False))
    rows = np.concatenate([rows, [3119, 3072, 3071]])    # the ragged last query tile
    _stream_and_check(ps, 3, check_every=2, attn_rows=np.unique(rows))


def test_full_size_14b_sampled():
    """Wan-14B-shaped layer at 512x512: 40 heads x 128, 1024 tokens per frame, B = 2."""
    cfg = dict(batch=2, layers=1, heads=40, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1, sink_frames=1,
               window_frames=6)
    ps = PairedStream(seed=1003, **cfg)
    rows = np.sort(np.random.default_rng(2).choice(1024, 32, replace=False))
    _stream_and_check(ps, 8, check_every=7, attn_rows=rows)


@pytest.mark.parametrize("splits", ["split", "unsplit"])
def test_back_to_back_attention_calls(splits):
    """Several attention calls on the same appended chunk in a row (and on
    alternating layers) give the same, correct output: a call's split partials
    and its in-kernel query rotation never disturb what an earlier call, still
    running or being merged, reads."""
    if splits == "split":
        cfg = dict(batch=1, layers=2, heads=12, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                   sink_frames=1, window_frames=6)
    else:
        cfg = dict(batch=1, layers=2, heads=37, head_dim=128, frame_h=32, frame_w=32, chunk_frames=1,
                   sink_frames=1, window_frames=1)
    ps = PairedStream(seed=1301, **cfg)
    c = ps.cfg
    from causal_dit_kv_b200 import binding as B
    n_split = B.sdv2_attention_splits(ps.gpu.cfg, [(c.sink_frames + c.window_frames) * c.frame_h * c.frame_w], 148)
    assert (n_split > 1) == (splits == "split")
    for step in range(c.sink_frames + c.window_frames + 1):
        ps.step_idx = step
        f0 = ps.advance()
        for layer in range(c.layers):
            _, k, v = ps.inputs(layer)
            ps.append(layer, f0, k, v)
    rows = np.arange(0, c.chunk_tokens, 97)
    qs = [ps.inputs(layer)[0] for layer in range(c.layers)]
    wants = [O.chunk_attention(ps.ora, layer, synth.bf16_bits(qs[layer]), f0, 1.0 / math.sqrt(c.head_dim), rows=rows)
             for layer in range(c.layers)]
    outs = [torch.zeros((c.batch, c.chunk_tokens, c.heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
            for _ in range(6)]
    qd = [q.cuda() for q in qs]
    for i, out in enumerate(outs):                    # no synchronisation between the calls
        ps.gpu.chunk_attention(i % c.layers, qd[i % c.layers], out, f0)
    torch.cuda.synchronize()
    for i, out in enumerate(outs):
        mx, mean = attn_errors(out, wants[i % c.layers], rows)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (i, mx, mean)
        assert torch.equal(out, outs[i % c.layers])

"""Pins for the oracle's sink refresh and motion/EMA noise rate (CPU only).

Hand-built embeddings with known angles decide the refresh; the motion
pins are closed forms (zero motion, constant shift, clipping, the EMA's
geometric solution) and the k-frame maximum over a hand-made sequence.
"""
import math

import numpy as np

import synth
from oracle import (CacheConfig, MotionConfig, MotionState, OracleCache, bf16_encode, kv_append,
                    motion_noise_rate, sink_refresh, slot_of_frame)


def _cache(S=3, W=2, D=4, layers=2):
    cfg = CacheConfig(batch=1, layers=layers, heads=1, head_dim=64, frame_h=1, frame_w=2,
                      chunk_frames=1, sink_frames=S, window_frames=W, embed_dim=D)
    return cfg, OracleCache(cfg)


def _hidden(vec, tokens):
    # every token equal to vec (exact in bf16 for the small integers used here)
    return bf16_encode(np.tile(np.asarray(vec, dtype=np.float64), (1, tokens, 1)))


def _advance(cfg, cache, f):
    _, k, v = synth.chunk_qkv(f, 1, cfg.chunk_tokens, 1, 64, f, 0)
    for layer in range(cfg.layers):
        kv_append(cache, layer, synth.bf16_bits(k), synth.bf16_bits(v), [f])


def _fill_sinks(cfg, cache, vecs):
    for f, vec in enumerate(vecs):
        _advance(cfg, cache, f)
        out = sink_refresh(cache, _hidden(vec, cfg.chunk_tokens), 0.9, [f])
        assert out[0] == -1          # filling a sink only records its embedding


def test_identical_embedding_no_refresh():
    cfg, cache = _cache()
    _fill_sinks(cfg, cache, [[1, 0, 0, 0], [0, 1, 0, 0], [1, 1, 0, 0]])
    _advance(cfg, cache, 3)
    # the new chunk equals sink 0 -> but the min over sinks decides: sink 1 is orthogonal
    out = sink_refresh(cache, _hidden([1, 0, 0, 0], 2), 0.9, [3])
    assert out[0] == 1
    _advance(cfg, cache, 4)
    # now all sinks relate to e=[1,0,0,0] by cos {1, 1 (refreshed), 1/sqrt2}: min = 0.707 < 0.9
    out = sink_refresh(cache, _hidden([1, 0, 0, 0], 2), 0.9, [4])
    assert out[0] == 2
    _advance(cfg, cache, 5)
    out = sink_refresh(cache, _hidden([1, 0, 0, 0], 2), 0.9, [5])
    assert out[0] == -1              # every sink identical to the chunk: cos = 1 >= tau


def test_known_argmin_and_tie_break():
    cfg, cache = _cache()
    a = [math.cos(0.3), math.sin(0.3)]
    # sinks at angles 0.3, 1.2, 1.2 rad from the x axis; chunk on the x axis
    _fill_sinks(cfg, cache, [[a[0], a[1], 0, 0], [math.cos(1.2), math.sin(1.2), 0, 0],
                             [math.cos(1.2), math.sin(1.2), 0, 0]])
    _advance(cfg, cache, 3)
    h = _hidden([1, 0, 0, 0], 2)
    out = sink_refresh(cache, h, 0.99, [3])
    assert out[0] == 1               # sinks 1 and 2 tie (bf16-identical); lowest index wins


def test_threshold_single_sink():
    for tau, want in [(0.5, -1), (0.8, 0)]:
        cfg, cache = _cache(S=1, W=2)
        _fill_sinks(cfg, cache, [[1, 0, 0, 0]])
        _advance(cfg, cache, 1)
        # cos(chunk, sink) = 1/sqrt(2) + small: below 0.8, above 0.5
        out = sink_refresh(cache, _hidden([1, 1, 0, 0], 2), tau, [1])
        assert out[0] == want


def test_refresh_copies_last_frame_all_layers():
    cfg, cache = _cache(S=1, W=2, layers=3)
    _fill_sinks(cfg, cache, [[1, 0, 0, 0]])
    _advance(cfg, cache, 1)
    before = cache.k.copy()
    out = sink_refresh(cache, _hidden([0, 1, 0, 0], 2), 0.9, [1])
    assert out[0] == 0
    s_last = slot_of_frame(1, 1, 2)
    assert np.array_equal(cache.k[:, 0, 0], before[:, 0, s_last])
    assert np.array_equal(cache.v[:, 0, 0], cache.v[:, 0, s_last])
    assert cache.sink_frame[0, 0] == 1


def test_zero_norm_never_refreshes():
    cfg, cache = _cache(S=1)
    _fill_sinks(cfg, cache, [[1, 0, 0, 0]])
    _advance(cfg, cache, 1)
    assert sink_refresh(cache, _hidden([0, 0, 0, 0], 2), 0.9, [1])[0] == -1


def _mcfg(**kw):
    args = dict(batch=1, channels=2, height=3, width=4, window=3, sigma=2.0, lam=0.9,
                s_min=0.5, s_max=0.9, s_init=0.7)
    args.update(kw)
    return MotionConfig(**args)


def test_static_frames_drive_rate_to_smax_geometrically():
    cfg = _mcfg(lam=0.3)
    st = MotionState(cfg)
    x = np.random.default_rng(0).standard_normal((1, 1, 2, 3, 4))
    rate, d = motion_noise_rate(st, x)
    assert d[0, 0] == -1 and rate[0] == 0.7          # first frame: no predecessor
    for t in range(1, 8):
        rate, d = motion_noise_rate(st, x)
        assert d[0, 0] == 0.0
        want = 0.9 + (1 - 0.3) ** t * (0.7 - 0.9)       # s_t = T + (1-lam)^t (s0 - T)
        assert abs(rate[0] - want) < 1e-15


def test_constant_shift_gives_exact_motion():
    cfg = _mcfg(sigma=4.0, lam=1.0)
    st = MotionState(cfg)
    x = np.zeros((1, 1, 2, 3, 4))
    motion_noise_rate(st, x)
    rate, d = motion_noise_rate(st, x + 1.5)
    assert d[0, 0] == 1.5
    assert abs(rate[0] - (0.9 - 0.4 * (1.5 / 4.0))) < 1e-15   # lam = 1: rate = target
    rate, d = motion_noise_rate(st, x + 1.5 - 10.0)            # |shift| 10 >= sigma: clipped
    assert d[0, 0] == 10.0 and abs(rate[0] - 0.5) < 1e-15


def test_window_max_and_direction():
    cfg = _mcfg(window=3, sigma=8.0, lam=1.0)
    st = MotionState(cfg)
    shifts = [0, 4, 5, 6, 6.5, 6.5, 6.5, 6.5]     # frame-to-frame steps 4, 1, 1, .5, 0, 0, 0
    dbar_want = [None, 4, 4, 4, 1, 1, 0.5, 0]
    rates = []
    for s, want in zip(shifts, dbar_want):
        rate, _ = motion_noise_rate(st, np.full((1, 1, 2, 3, 4), s))
        if want is not None:
            assert abs(rate[0] - (0.9 - 0.4 * want / 8.0)) < 1e-15
            rates.append(rate[0])
    # more motion -> lower noise rate
    assert rates[0] < rates[-1]


def test_chunk_of_several_frames_equals_frame_by_frame():
    cfg = _mcfg(batch=2)
    gen = synth.motion_latents(3, 2, 4, 2, 3, 4, n_chunks=3)
    chunks = [c.numpy() for c in gen]
    a, b = MotionState(cfg), MotionState(_mcfg(batch=2))
    for c in chunks:
        ra, da = motion_noise_rate(a, c)
        for t in range(c.shape[1]):
            rb, db = motion_noise_rate(b, c[:, t:t + 1])
            assert np.array_equal(da[:, t], db[:, 0])
        assert np.array_equal(ra, rb)

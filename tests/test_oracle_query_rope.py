"""Pins of the oracle's query rotation (``chunk_queries_rotated``), CPU only.

The query side of the attention has to rotate every frame of a chunk at that
frame's own temporal phase, and that phase has to restart at the reset period
(qq8o.cn walkthrough, "Adaptive sink and RoPE refresh").  None of the checks
below reuse the function under test for their expected value:

  * measured angles: the angle a query pair turns by, read back with atan2 and
    divided by the pair's frequency, equals a hand-written phase list for a
    chunk that straddles a reset (e.g. [3, 0] for frames 3, 4 with period 4);
  * a plain-Python brute force of the 3D rotation on a tiny head, with the
    per-frame phases written out by hand;
  * zero offset: RoPE(q) . RoPE(k) equals the raw q . k when the key was
    rotated at the same frame and token (and differs at another frame);
  * the key path: a query vector appended as a key lands in the cache with the
    same bits as the bf16 rounding of its own rotation;
  * the period: shifting the chunk by the reset period leaves every rotated
    query unchanged; within a period, q . k depends only on the frame offset.

Each one fails if the function rotated every frame of the chunk at the first
frame's phase, or ignored the reset.
"""
import math

import numpy as np
import pytest

import synth
from oracle import (CacheConfig, OracleCache, bf16_decode, bf16_encode, chunk_queries_rotated, kv_append,
                    rope_phase, rope_rotate, rope_token_cos_sin, slot_of_frame)


def _cfg(**kw):
    args = dict(batch=1, layers=1, heads=2, head_dim=16, frame_h=2, frame_w=3, chunk_frames=2, sink_frames=1,
                window_frames=4, rope_pairs=(4, 2, 2), rope_reset_period=4, embed_dim=8)
    args.update(kw)
    return CacheConfig(**args)


def _bits(x):
    """fp64 values that are exact bf16 -> bf16 bit patterns."""
    b = bf16_encode(x)
    assert np.array_equal(bf16_decode(b), x)
    return b


def _random_q(cfg, seed):
    q, _, _ = synth.chunk_qkv(seed, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, 0, 0)
    return synth.bf16_bits(q)[0]                                   # [T'N][H][d]


@pytest.mark.parametrize("f0,reset,tp,phases", [
    (3, 4, 2, [3, 0]),            # straddles the reset
    (2, 4, 3, [2, 3, 0]),         # three frames, the last one after the reset
    (5, 4, 2, [1, 2]),            # second period
    (3, 0, 2, [3, 4]),            # no reset
    (7, 1, 2, [0, 0]),            # reset every frame: every frame at phase 0
])
def test_query_phase_of_every_frame_read_back_from_its_angle(f0, reset, tp, phases):
    cfg = _cfg(chunk_frames=tp, rope_reset_period=reset)
    N, d = cfg.tokens_per_frame, cfg.head_dim
    n_t = cfg.rope_pairs[0]
    # query (1, 0) in every pair: the rotated pair is (cos a, sin a), a = the pair's angle
    x = np.zeros((cfg.chunk_tokens, cfg.heads, d))
    x[..., 0::2] = 1.0
    qr = chunk_queries_rotated(cfg, _bits(x), f0)
    for i, ph in enumerate(phases):
        tok = i * N                                                 # token (row 0, col 0) of frame i
        # h and w pairs sit at position 0 for this token: untouched
        assert np.array_equal(qr[tok, :, 2 * n_t:], x[tok, :, 2 * n_t:])
        for j in range(n_t):
            a = math.atan2(qr[tok, 0, 2 * j + 1], qr[tok, 0, 2 * j])
            omega = 10000.0 ** (-j / n_t)                           # frequencies pinned elsewhere
            want = ph * omega
            diff = (a - want + math.pi) % (2 * math.pi) - math.pi   # equal modulo a full turn
            assert abs(diff) < 1e-12, (i, j, a, want)


def _brute_rotate(vec, t_pos, row, col, pairs, base=10000.0):
    """3D RoPE of one head vector in plain Python: pair j of an axis with n pairs turns
    by position * base^(-j / n); t pairs first, then h, then w; pair k = dims (2k, 2k+1)."""
    out = list(vec)
    k = 0
    for pos, n in ((t_pos, pairs[0]), (row, pairs[1]), (col, pairs[2])):
        for j in range(n):
            a = pos * base ** (-j / n)
            c, s = math.cos(a), math.sin(a)
            x0, x1 = vec[2 * k], vec[2 * k + 1]
            out[2 * k] = x0 * c - x1 * s
            out[2 * k + 1] = x0 * s + x1 * c
            k += 1
    return out


def test_query_rotation_brute_force_with_hand_phases():
    cfg = _cfg(chunk_frames=3, rope_reset_period=3)
    f0 = 2
    hand_phases = [2, 0, 1]                                         # frames 2, 3, 4 with period 3
    qb = _random_q(cfg, 11)
    qr = chunk_queries_rotated(cfg, qb, f0)
    q = bf16_decode(qb)
    N = cfg.tokens_per_frame
    for tok in range(cfg.chunk_tokens):
        i, n = divmod(tok, N)
        row, col = divmod(n, cfg.frame_w)
        for h in range(cfg.heads):
            want = _brute_rotate(list(q[tok, h]), hand_phases[i], row, col, cfg.rope_pairs)
            assert np.max(np.abs(qr[tok, h] - np.array(want))) < 1e-13, (tok, h)


def _key_rotated(cfg, k, frame):
    """A key of one frame [N][H][d] rotated as the cache's append rotates it (fp64, not
    rounded), from the key path's own per-frame phase."""
    c, s = rope_token_cos_sin([rope_phase(frame, cfg.rope_reset_period)], cfg.frame_h, cfg.frame_w,
                              cfg.rope_pairs, cfg.rope_base)
    return rope_rotate(k, c, s)


@pytest.mark.parametrize("f0", [0, 2, 3, 6, 7])
def test_zero_offset_keeps_the_raw_dot_product(f0):
    """A T'=2 chunk with period 4: f0 = 3 and 7 straddle the reset."""
    cfg = _cfg(head_dim=128, rope_pairs=(22, 21, 21), frame_h=2, frame_w=2, rope_reset_period=4)
    N = cfg.tokens_per_frame
    qb = _random_q(cfg, 12)
    _, kk, _ = synth.chunk_qkv(13, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, 0, 0)
    k = bf16_decode(synth.bf16_bits(kk)[0])
    q = bf16_decode(qb)
    qr = chunk_queries_rotated(cfg, qb, f0)
    for i in range(cfg.chunk_frames):
        kr = _key_rotated(cfg, k[i * N:(i + 1) * N], f0 + i)
        other = _key_rotated(cfg, k[i * N:(i + 1) * N], f0 + i + 1)
        for n in range(N):
            for h in range(cfg.heads):
                raw = float(q[i * N + n, h] @ k[i * N + n, h])
                assert abs(float(qr[i * N + n, h] @ kr[n, h]) - raw) < 1e-12
                # the key one frame later is at offset -1: the product changes
                assert abs(float(qr[i * N + n, h] @ other[n, h]) - raw) > 1e-6


@pytest.mark.parametrize("f0", [1, 3, 5, 6])
def test_query_rotation_matches_the_key_written_at_the_same_frame(f0):
    """Append the query vectors as keys: the cache rounds RoPE(k) to bf16 once, per frame
    at that frame's phase; the rotated queries, rounded the same way, carry the same bits."""
    cfg = _cfg(rope_reset_period=3, window_frames=8)
    qb = _random_q(cfg, 14)
    cache = OracleCache(cfg)
    for f in range(0, f0, cfg.chunk_frames) if f0 % cfg.chunk_frames == 0 else []:
        kv_append(cache, 0, qb[None], qb[None], [f])
    if f0 % cfg.chunk_frames:
        cache.next_frame[0, 0] = f0                                # start the stream at f0
    kv_append(cache, 0, qb[None], qb[None], [f0])
    qr = chunk_queries_rotated(cfg, qb, f0)
    N = cfg.tokens_per_frame
    for i in range(cfg.chunk_frames):
        s = slot_of_frame(f0 + i, cfg.sink_frames, cfg.window_frames)
        assert np.array_equal(cache.k[0, 0, s], bf16_encode(qr[i * N:(i + 1) * N])), i


def test_shift_by_the_period_changes_nothing_and_offsets_decide_within_a_period():
    cfg = _cfg(rope_reset_period=5)
    qb = _random_q(cfg, 15)
    base = chunk_queries_rotated(cfg, qb, 1)
    assert np.array_equal(chunk_queries_rotated(cfg, qb, 1 + 5), base)
    assert np.array_equal(chunk_queries_rotated(cfg, qb, 1 + 10), base)
    assert not np.array_equal(chunk_queries_rotated(cfg, qb, 2), base)
    # inside one period, q . k depends only on the frame offset between query and key
    N = cfg.tokens_per_frame
    _, kk, _ = synth.chunk_qkv(16, 1, N, cfg.heads, cfg.head_dim, 0, 0)
    k = bf16_decode(synth.bf16_bits(kk)[0])
    q_at = {f0: chunk_queries_rotated(cfg, qb, f0) for f0 in (0, 1, 2, 3)}
    # frame 1 of a chunk at f0 sits at f0 + 1; key at f0: offset 1 in every case
    dots = [float(q_at[f0][N + 4, 1] @ _key_rotated(cfg, k, f0)[4, 1]) for f0 in (0, 1, 2, 3)]
    assert max(dots) - min(dots) < 1e-12

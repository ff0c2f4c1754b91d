"""Pins for the oracle's RoPE, append and attention (CPU only).

Each check rests on something other than the oracle's own formulas:
closed forms of a plane rotation, the relative-position property of RoPE,
hand-derived frequencies, torch's fp64 scaled_dot_product_attention, brute
force in plain Python, and invariants (row sums, permutations, ring vs a
linear history).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import (CacheConfig, OracleCache, attention_reference, bf16_decode, bf16_encode,
                    chunk_attention, chunk_queries_rotated, kv_append, rope_axis_cos_sin,
                    rope_pair_split, rope_phase, rope_rotate, rope_token_cos_sin, slot_of_frame,
                    valid_keys)


def test_pair_split():
    assert rope_pair_split(128) == (22, 21, 21)
    assert rope_pair_split(64) == (12, 10, 10)
    assert sum(rope_pair_split(96)) == 48


def test_frequencies_hand_values():
    # base**(-j/n): j = 0 -> 1 rad/step; j = n/2 -> base**-0.5 = 0.01 for base 1e4.
    c, s = rope_axis_cos_sin([1], 22, 10000.0)
    assert c[0, 0] == math.cos(1.0) and s[0, 0] == math.sin(1.0)
    assert abs(math.atan2(s[0, 11], c[0, 11]) - 0.01) < 1e-15
    c, s = rope_axis_cos_sin([0, 3], 21, 10000.0)
    assert np.all(c[0] == 1.0) and np.all(s[0] == 0.0)       # position 0: identity


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_rotation_preserves_norm_and_single_pair_closed_form():
    rng = np.random.default_rng(1)
    for _ in range(50):
        a, b, tq, tk = rng.uniform(-7, 7, 4)
        nq, nk = rng.uniform(0.1, 3, 2)
        q = np.array([[nq * math.cos(a), nq * math.sin(a)]])
        k = np.array([[nk * math.cos(b), nk * math.sin(b)]])
        qr = rope_rotate(q, np.array([[math.cos(tq)]]), np.array([[math.sin(tq)]]))
        kr = rope_rotate(k, np.array([[math.cos(tk)]]), np.array([[math.sin(tk)]]))
        # a plane rotation by t turns the angle a into a + t
        assert abs(float(qr[0] @ kr[0]) - nq * nk * math.cos((a + tq) - (b + tk))) < 1e-12
        assert abs(np.linalg.norm(qr) - nq) < 1e-13


def test_axis_layout_and_token_grid():
    # t pairs first, then h, then w; token n sits at (n // fw, n % fw).
    fh, fw, pairs = 3, 5, (4, 2, 2)
    d = 2 * sum(pairs)
    x = _rand((fh * fw, d), 2)
    for phase, n, moved in [(3, 0, "t"), (0, fw, "h"), (0, 1, "w"), (0, 0, "")]:
        cos, sin = rope_token_cos_sin([phase], fh, fw, pairs, 10000.0)
        r = rope_rotate(x, cos, sin)
        bounds = {"t": (0, 2 * pairs[0]), "h": (2 * pairs[0], 2 * (pairs[0] + pairs[1])),
                  "w": (2 * (pairs[0] + pairs[1]), d)}
        for axis, (lo, hi) in bounds.items():
            same = np.array_equal(r[n, lo:hi], x[n, lo:hi])
            assert same == (axis != moved), (phase, n, axis)


def test_dot_depends_only_on_offset():
    # shifting both positions of a (q, k) pair by the same amount leaves q.k unchanged
    fh, fw = 4, 6
    pairs = rope_pair_split(64)
    q = _rand((64,), 3)
    k = _rand((64,), 4)

    def rot(v, phase, n):
        c, s = rope_token_cos_sin([phase], fh, fw, pairs, 10000.0)
        return rope_rotate(v[None, :], c[n:n + 1], s[n:n + 1])[0]

    base = rot(q, 5, 7) @ rot(k, 2, 1)
    # time shift
    assert abs(rot(q, 9, 7) @ rot(k, 6, 1) - base) < 1e-11
    # spatial shift by one row and one column (7 -> 14, 1 -> 8)
    assert abs(rot(q, 5, 7 + fw + 1) @ rot(k, 2, 1 + fw + 1) - base) < 1e-11
    # a different offset changes it
    assert abs(rot(q, 5, 7) @ rot(k, 3, 1) - base) > 1e-6


def _small_cfg(**kw):
    args = dict(batch=2, layers=2, heads=3, head_dim=64, frame_h=2, frame_w=3, chunk_frames=1,
                sink_frames=1, window_frames=2, rope_reset_period=0, embed_dim=16)
    args.update(kw)
    return CacheConfig(**args)


def _stream(cfg, n_steps, seed=11):
    cache = OracleCache(cfg)
    hist = []
    for step in range(n_steps):
        f0 = np.full(cfg.batch, step * cfg.chunk_frames)
        q, k, v = synth.chunk_qkv(seed, cfg.batch, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        for layer in range(cfg.layers):
            kv_append(cache, layer, synth.bf16_bits(k), synth.bf16_bits(v), f0)
        hist.append((f0, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)))
    return cache, hist


def test_append_rotates_k_once_and_copies_v():
    cfg = _small_cfg(chunk_frames=2, window_frames=3, rope_reset_period=0)
    cache, hist = _stream(cfg, 1)
    f0, _, kb, vb = hist[0]
    N = cfg.tokens_per_frame
    for b in range(cfg.batch):
        for i in range(cfg.chunk_frames):
            f = int(f0[b]) + i
            s = slot_of_frame(f, cfg.sink_frames, cfg.window_frames)
            assert np.array_equal(cache.v[0, b, s], vb[b, i * N:(i + 1) * N])
            c, sn = rope_token_cos_sin([f], cfg.frame_h, cfg.frame_w, cfg.rope_pairs, cfg.rope_base)
            want = bf16_encode(rope_rotate(bf16_decode(kb[b, i * N:(i + 1) * N]), c, sn))
            assert np.array_equal(cache.k[0, b, s], want)
    # frame 0 at phase 0 with row 0, col 0: the first token is not rotated at all
    assert np.array_equal(cache.k[0, 0, 0, 0], kb[0, 0])


def test_phase_reset_gives_bit_identical_keys():
    cfg = _small_cfg(rope_reset_period=3, window_frames=5)
    cache = OracleCache(cfg)
    _, k, v = synth.chunk_qkv(3, cfg.batch, cfg.chunk_tokens, cfg.heads, cfg.head_dim, 0, 0)
    kb, vb = synth.bf16_bits(k), synth.bf16_bits(v)
    for f in range(5):
        kv_append(cache, 0, kb, vb, np.full(cfg.batch, f))
    # frames 1 and 4 share phase 1 (4 mod 3); same input keys -> identical rotated keys
    s1, s4 = slot_of_frame(1, 1, 5), slot_of_frame(4, 1, 5)
    assert np.array_equal(cache.k[0, :, s1], cache.k[0, :, s4])
    assert not np.array_equal(cache.k[0, :, s1], cache.k[0, :, slot_of_frame(2, 1, 5)])


def test_attention_reference_matches_torch_sdpa():
    rng = np.random.default_rng(7)
    for lq, lk, d in [(5, 9, 8), (16, 48, 64), (33, 130, 128)]:
        q, k, v = rng.standard_normal((lq, d)), rng.standard_normal((lk, d)), rng.standard_normal((lk, d))
        scale = 1.0 / math.sqrt(d)
        out, p = attention_reference(q, k, v, scale)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], scale=scale)[0]
        assert np.max(np.abs(out - want.numpy())) < 1e-12
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-13


def test_attention_reference_brute_force_python():
    rng = np.random.default_rng(8)
    q, k, v = rng.standard_normal((3, 4)), rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    out, _ = attention_reference(q, k, v, 0.7)
    for i in range(3):
        s = [0.7 * sum(q[i, t] * k[j, t] for t in range(4)) for j in range(6)]
        e = [math.exp(x) for x in s]
        z = sum(e)
        for t in range(4):
            assert abs(out[i, t] - sum(e[j] * v[j, t] for j in range(6)) / z) < 1e-13


def test_attention_invariants():
    rng = np.random.default_rng(9)
    q, k, v = rng.standard_normal((7, 16)), rng.standard_normal((20, 16)), rng.standard_normal((20, 16))
    base, _ = attention_reference(q, k, v, 0.25)
    perm = rng.permutation(20)
    permuted, _ = attention_reference(q, k[perm], v[perm], 0.25)
    assert np.max(np.abs(base - permuted)) < 1e-13
    uniform = np.tile(rng.standard_normal((1, 16)), (20, 1))
    out_u, _ = attention_reference(q, k, uniform, 0.25)
    assert np.max(np.abs(out_u - uniform[:7])) < 1e-13
    out0, _ = attention_reference(q, k, v, 0.0)
    assert np.max(np.abs(out0 - v.mean(axis=0))) < 1e-13


def test_single_valid_key_returns_its_value():
    # one token per frame, first chunk: exactly one valid key per head
    cfg = _small_cfg(frame_h=1, frame_w=1, batch=1, layers=1)
    cache = OracleCache(cfg)
    q, k, v = synth.chunk_qkv(4, 1, 1, cfg.heads, cfg.head_dim, 0, 0)
    kv_append(cache, 0, synth.bf16_bits(k), synth.bf16_bits(v), [0])
    out = chunk_attention(cache, 0, synth.bf16_bits(q), [0], 0.125)
    assert np.array_equal(out[0, 0], bf16_decode(synth.bf16_bits(v))[0, 0])


@pytest.mark.parametrize("S,W,Tp,reset", [(1, 2, 1, 0), (2, 3, 1, 4), (1, 4, 2, 3)])
def test_ring_attention_equals_linear_history(S, W, Tp, reset):
    """Attention over the ring cache equals attention over the sink frames plus
    the last W frames kept as a plain time-ordered list."""
    cfg = _small_cfg(sink_frames=S, window_frames=W, chunk_frames=Tp, rope_reset_period=reset,
                     batch=1, layers=1)
    cache = OracleCache(cfg)
    N = cfg.tokens_per_frame
    frames = []   # (rotated k fp64 [N][H][d], v fp64) per frame, in time order
    for step in range(7):
        f0 = step * Tp
        q, k, v = synth.chunk_qkv(21, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
        kv_append(cache, 0, kb, vb, [f0])
        for i in range(Tp):
            c, s = rope_token_cos_sin([rope_phase(f0 + i, reset)], cfg.frame_h, cfg.frame_w,
                                      cfg.rope_pairs, cfg.rope_base)
            kr = bf16_decode(bf16_encode(rope_rotate(bf16_decode(kb[0, i * N:(i + 1) * N]), c, s)))
            frames.append((kr, bf16_decode(vb[0, i * N:(i + 1) * N])))
        kept = frames[:S] + frames[S:][-W:] if len(frames) > S else frames
        klin = np.concatenate([f[0] for f in kept])
        vlin = np.concatenate([f[1] for f in kept])
        out = chunk_attention(cache, 0, qb, [f0], 0.1)
        qr = chunk_queries_rotated(cfg, qb[0], f0)
        for h in range(cfg.heads):
            want, _ = attention_reference(qr[:, h], klin[:, h], vlin[:, h], 0.1)
            assert np.max(np.abs(out[0, :, h] - want)) < 1e-12
        kc, _ = valid_keys(cache, 0, 0)
        assert kc.shape[0] == klin.shape[0]

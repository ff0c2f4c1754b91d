"""Pins of the oracle's fp8 (E4M3) cache: the encoder against torch's own E4M3
conversion and the format's closed forms, the block quantiser against its
error bound, and the cache layouts against the bf16 cache they quantise."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from oracle.sdv2_fp8 import (BLOCK_TOKENS, E4M3_MAX, OracleFp8Cache, chunk_attention_fp8, e4m3_decode,
                             e4m3_encode, e4m3_round, kv_append_fp8, quantize_block, sink_refresh_fp8)


def _torch_e4m3_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_encoder_matches_torch_conversion_in_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0,                          # normal range
        rng.standard_normal(5000) * 2.0 ** -8,                      # subnormal range
        rng.uniform(-464.0, 464.0, 5000),                           # up to the rounding edge of 448
        [0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -11, 1.0625, 1.1875, 464.0, -464.0, 2.0 ** -6, 15.5, 0.5 * 2.0 ** -9],
    ]).astype(np.float32).astype(np.float64)
    ours = e4m3_encode(x)
    assert np.array_equal(ours, _torch_e4m3_bits(x))
    assert np.array_equal(e4m3_decode(ours), e4m3_round(x))


def test_ties_go_to_even_and_saturation():
    # 1 + 1/16 is halfway between 1.0 (mantissa 000) and 1.125 (001): even wins
    assert e4m3_encode(np.array([1.0625]))[0] == 0x38
    assert e4m3_encode(np.array([1.1875]))[0] == 0x3A            # halfway 1.125 / 1.25 -> 1.25 (010)
    assert e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00       # halfway 0 / 2^-9 -> 0
    big = np.array([448.0, 449.0, 480.0, 1e6, -1e30])
    assert list(e4m3_encode(big)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = e4m3_decode(codes)
    assert np.array_equal(e4m3_encode(vals), codes)
    assert vals.max() == E4M3_MAX and np.min(vals[vals > 0]) == 2.0 ** -9
    assert np.isnan(e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_block_quantiser_bound_and_extremes():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((128, 128)) * 3.0).astype(np.float32).astype(np.float64)
    codes, scale = quantize_block(x)
    amax = np.abs(x).max()
    assert scale == np.float32(np.float32(amax) / np.float32(448.0))
    deq = e4m3_decode(codes) * float(scale)
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert e4m3_decode(np.array([codes[i]]))[0] == np.copysign(448.0, x[i])
    # error bound: half a quantum of the element's binade (2^-4 relative in the normal range,
    # 2^-10 * scale absolute below it), plus the fp32 roundings of the scale and the product
    rel_ok = np.abs(deq - x) <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * float(scale)) * (1 + 1e-6) + 1e-12
    assert rel_ok.all()
    z_codes, z_scale = quantize_block(np.zeros((4, 128)))
    assert not z_codes.any() and z_scale == 0.0


def _cfg(**kw):
    base = dict(batch=2, layers=2, heads=2, head_dim=128, frame_h=10, frame_w=15, chunk_frames=1, sink_frames=1,
                window_frames=3, embed_dim=32, rope_reset_period=0)
    base.update(kw)
    return O.CacheConfig(**base)


def test_fp8_cache_layouts_track_the_bf16_cache():
    cfg = _cfg()
    c8 = OracleFp8Cache(cfg)
    N = cfg.tokens_per_frame                                  # 150 tokens: one full block and one ragged block
    assert c8.np_tokens == 256
    for step in range(6):                                     # wraps the window
        q, k, v = synth.chunk_qkv(31, cfg.batch, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        kv_append_fp8(c8, 0, k.view(torch.int16).numpy().view(np.uint16), v.view(torch.int16).numpy().view(np.uint16),
                      [step] * cfg.batch)
    for b in range(cfg.batch):
        kq, vq = c8.dequantized(0, b, cfg.slots)
        kb = O.bf16_decode(c8.base.k[0, b]).reshape(cfg.slots * N, cfg.heads, cfg.head_dim)
        vb = O.bf16_decode(c8.base.v[0, b]).reshape(cfg.slots * N, cfg.heads, cfg.head_dim)
        for got, want, sc in ((kq, kb, c8.k_scale), (vq, vb, c8.v_scale)):
            bound = np.maximum(2.0 ** -4 * np.abs(want), 2.0 ** -10 * float(sc[0, b].max())) * (1 + 1e-6) + 1e-12
            assert (np.abs(got - want) <= bound).all()
    assert not c8.k8[:, :, :, N:].any() and not c8.v8t[..., N:].any()   # padding tokens hold code 0
    assert c8.k_scale.shape[-1] == 256 // BLOCK_TOKENS


def test_fp8_attention_close_to_bf16_attention_and_refresh_copies_codes():
    cfg = _cfg(batch=1, window_frames=2)
    c8 = OracleFp8Cache(cfg)
    scale = 1.0 / np.sqrt(cfg.head_dim)
    for step in range(4):
        q, k, v = synth.chunk_qkv(41, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        as16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
        for layer in range(cfg.layers):
            kv_append_fp8(c8, layer, as16(k), as16(v), [step])
        got = chunk_attention_fp8(c8, 0, as16(q), [step], scale)
        want = O.chunk_attention(c8.base, 0, as16(q), [step], scale)
        err = np.abs(got - want)
        # K, V each within 2^-4 relative: logits move by < 0.1 here, outputs by a few 1e-2 at most
        assert err.max() < 6e-2 and err.mean() < 1e-2
    hid = np.zeros((1, cfg.chunk_tokens, cfg.embed_dim), np.uint16)
    hid[..., 0] = 0x3F80                                   # the chunk embedding e_0 = (1, 0, ...)
    c8.base.sink_embed[0, 0, 1] = 1.0                       # a sink embedding orthogonal to it
    slot = sink_refresh_fp8(c8, hid, 0.9, [3])
    assert slot[0] == 0
    s_last = O.slot_of_frame(3, cfg.sink_frames, cfg.window_frames)
    for arr in (c8.k8, c8.v8t, c8.k_scale, c8.v_scale):
        assert np.array_equal(arr[:, 0, 0], arr[:, 0, s_last])


def test_block_quantiser_tiny_block_clamps_the_inverse():
    # amax below 448 / FLT_MAX: 448 / amax overflows fp32 and the inverse is clamped to the
    # largest finite fp32 (not infinity), so zeros stay zero (no 0 * inf) and every code is
    # finite; the largest element then maps to amax * FLT_MAX (about 3.4 here), not to 448
    x = np.array([0.0, 1e-38, -5e-39, 2.0 ** -130], dtype=np.float32).astype(np.float64)
    codes, scale = quantize_block(x)
    assert scale == np.float32(np.float32(1e-38) / np.float32(448.0))
    assert codes[0] == 0x00 and codes[1] == 0x46 and codes[2] & 0x80          # 0x46 = 3.5
    with np.errstate(over="ignore"):
        inv = np.float32(np.finfo(np.float32).max)
        want = e4m3_encode((x.astype(np.float32) * inv).astype(np.float64))
    assert np.array_equal(codes, want)

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


def _quant_err(x, scales_per_elem):
    """Largest error the block quantiser may make on x (see the quantiser bound test):
    half a quantum of x's binade, 2^-4 |x| in the normal range, 2^-10 * scale below it,
    with room for the fp32 roundings of the scale and the product."""
    return np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scales_per_elem) * (1 + 1e-6) + 1e-12


def _block_scales(sc, n_tokens):
    """Per-token scales [slots * N][H] from per-(slot, head, block) scales [slots][H][n_blk]."""
    blk = np.arange(n_tokens) // BLOCK_TOKENS
    per_tok = sc[:, :, blk].astype(np.float64)                     # [slots][H][N]
    return per_tok.transpose(0, 2, 1).reshape(-1, sc.shape[1])


def test_fp8_cache_tracks_the_bf16_cache():
    cfg = _cfg()
    c8 = OracleFp8Cache(cfg)
    N = cfg.tokens_per_frame                                  # 150 tokens: one full block and one of 22 tokens
    assert c8.n_blk == 2
    for step in range(6):                                     # wraps the window
        q, k, v = synth.chunk_qkv(31, cfg.batch, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        kv_append_fp8(c8, 0, k.view(torch.int16).numpy().view(np.uint16), v.view(torch.int16).numpy().view(np.uint16),
                      [step] * cfg.batch)
    for b in range(cfg.batch):
        kq, vq = c8.dequantized(0, b, cfg.slots)
        kb = O.bf16_decode(c8.base.k[0, b]).reshape(cfg.slots * N, cfg.heads, cfg.head_dim)
        vb = O.bf16_decode(c8.base.v[0, b]).reshape(cfg.slots * N, cfg.heads, cfg.head_dim)
        for got, want, sc in ((kq, kb, c8.k_scale[0, b]), (vq, vb, c8.v_scale[0, b])):
            # element by element, each against the scale of its own (slot, head, block): a
            # transposed or misplaced block, or a scale taken over the wrong tokens, fails here
            assert (np.abs(got - want) <= _quant_err(want, _block_scales(sc, N)[..., None])).all()
            # every block's largest element is coded as +-448 exactly
            for s in range(cfg.slots):
                for h in range(cfg.heads):
                    for j in range(c8.n_blk):
                        t0, t1 = s * N + j * BLOCK_TOKENS, s * N + min(N, (j + 1) * BLOCK_TOKENS)
                        amax = np.abs(want[t0:t1, h]).max()
                        assert sc[s, h, j] == np.float32(np.float32(amax) / np.float32(448.0))


def _fp8_attention_sigma(qr, kb, vb, ks, vs, scale):
    """Per-element RMS of |fp8 attention - bf16 attention| implied by the quantiser's
    per-element error bound e (uniform rounding error in [-e, e], RMS e / sqrt(3),
    independent between elements).  qr [rows][d]; kb, vb [Lk][d] the bf16 values; ks, vs
    [Lk] the scale of each key's block.  To first order, with p the bf16 probabilities
    and o the bf16 output,
        do_c = sum_j p_j dv_jc + sum_j p_j (ds_j - mean_p ds)(v_jc - o_c),
        ds_j = scale * sum_c q_c dk_jc,
    so sigma_c^2 = sum_j p_j^2 (ev_jc^2 / 3 + var(ds_j) (v_jc - o_c)^2) with
    var(ds_j) = scale^2 sum_c q_c^2 ek_jc^2 / 3 (the mean term is dropped: p is spread
    over thousands of keys)."""
    o, p = O.attention_reference(qr, kb, vb, scale)
    ek = _quant_err(kb, ks[:, None])
    ev = _quant_err(vb, vs[:, None])
    var_s = scale ** 2 * ((qr ** 2) @ (ek ** 2).T) / 3.0                     # [rows][Lk]
    p2 = p ** 2
    dv = vb[None, :, :] - o[:, None, :]                                       # [rows][Lk][d]
    var = p2 @ (ev ** 2 / 3.0) + np.einsum("rj,rjc->rc", p2 * var_s, dv ** 2)
    return np.sqrt(var), o


def test_fp8_attention_within_the_quantisation_bound_and_refresh_copies_codes():
    cfg = _cfg(batch=1, window_frames=2)
    c8 = OracleFp8Cache(cfg)
    N = cfg.tokens_per_frame
    scale = 1.0 / np.sqrt(cfg.head_dim)
    as16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    for step in range(4):
        q, k, v = synth.chunk_qkv(41, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        for layer in range(cfg.layers):
            kv_append_fp8(c8, layer, as16(k), as16(v), [step])
        got = chunk_attention_fp8(c8, 0, as16(q), [step], scale)
        want = O.chunk_attention(c8.base, 0, as16(q), [step], scale)
        sv, wv = O.valid_slot_counts(step + 1, cfg.sink_frames, cfg.window_frames)
        kb, vb = O.valid_keys(c8.base, 0, 0)
        qr = O.chunk_queries_rotated(cfg, as16(q)[0], step)
        ks = _block_scales(c8.k_scale[0, 0, :sv + wv], N)
        vs = _block_scales(c8.v_scale[0, 0, :sv + wv], N)
        ratios = []
        for h in range(cfg.heads):
            sigma, o = _fp8_attention_sigma(qr[:, h], kb[:, h], vb[:, h], ks[:, h], vs[:, h], scale)
            assert np.allclose(o, want[0, :, h], rtol=0, atol=1e-12)
            err = np.abs(got[0, :, h] - want[0, :, h])
            assert (err <= 6.0 * sigma).all(), (step, h, float((err / sigma).max()))
            ratios.append(err / sigma)
        # |N(0, 1)| has mean 0.80; the uniform-error RMS over-estimates E4M3's rounding error
        assert float(np.concatenate(ratios).mean()) < 1.0
    hid = np.zeros((1, cfg.chunk_tokens, cfg.embed_dim), np.uint16)
    hid[..., 0] = 0x3F80                                   # the chunk embedding e_0 = (1, 0, ...)
    c8.base.sink_embed[0, 0, 1] = 1.0                       # a sink embedding orthogonal to it
    slot = sink_refresh_fp8(c8, hid, 0.9, [3])
    assert slot[0] == 0
    s_last = O.slot_of_frame(3, cfg.sink_frames, cfg.window_frames)
    for arr in (c8.k8, c8.v8, c8.k_scale, c8.v_scale):
        assert np.array_equal(arr[:, 0, 0], arr[:, 0, s_last])


def test_fp8_attention_bound_catches_a_planted_scale_error():
    """The tolerance of the test above has power: with one block's V scale doubled in the
    oracle's copy (a plausible indexing slip), the fp8 attention leaves it."""
    cfg = _cfg(batch=1, window_frames=2, heads=1)
    c8 = OracleFp8Cache(cfg)
    N = cfg.tokens_per_frame
    scale = 1.0 / np.sqrt(cfg.head_dim)
    as16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    for step in range(3):
        q, k, v = synth.chunk_qkv(43, 1, cfg.chunk_tokens, cfg.heads, cfg.head_dim, step, 0)
        for layer in range(cfg.layers):
            kv_append_fp8(c8, layer, as16(k), as16(v), [step])
    c8.v_scale[0, 0, 1, 0, 0] *= 2.0
    got = chunk_attention_fp8(c8, 0, as16(q), [2], scale)
    kb, vb = O.valid_keys(c8.base, 0, 0)
    qr = O.chunk_queries_rotated(cfg, as16(q)[0], 2)
    c8.v_scale[0, 0, 1, 0, 0] /= 2.0
    ks = _block_scales(c8.k_scale[0, 0, :3], N)
    vs = _block_scales(c8.v_scale[0, 0, :3], N)
    sigma, o = _fp8_attention_sigma(qr[:, 0], kb[:, 0], vb[:, 0], ks[:, 0], vs[:, 0], scale)
    assert (np.abs(got[0, :, 0] - o) > 6.0 * sigma).any()


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

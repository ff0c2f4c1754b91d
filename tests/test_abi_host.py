"""C ABI and host-side logic, no GPU needed: the library loads, exports every
function include/sdv2.h declares, and its pure host helpers (ring slots,
phases, valid prefix, buffer layout, split plan) agree with the oracle."""
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from causal_dit_kv_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        from causal_dit_kv_b200 import build
        build.build()
    binding.lib()
    return binding


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sdv2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdv2_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(B):
    declared = _declared_functions()
    assert len(declared) >= 20
    lib = B.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(B.EXPORTED) == declared


def test_version_and_error_string(B):
    assert "sm_100a" in B.sdv2_version()
    assert isinstance(B.sdv2_last_error(), str)


@pytest.mark.parametrize("S,W", [(1, 2), (2, 3), (1, 6), (1, 8), (3, 1)])
def test_slots_phases_valid_match_oracle(B, S, W):
    for f in range(0, 200):
        assert B.sdv2_slot_of_frame(f, S, W) == O.slot_of_frame(f, S, W)
        assert B.sdv2_valid_slots(f + 1, S, W) == O.valid_slot_counts(f + 1, S, W)
    for T in (0, 1, 3, 256):
        for f in (0, 1, 255, 256, 257, 1999):
            assert B.sdv2_rope_phase(f, T) == O.rope_phase(f, T)
    assert B.sdv2_slot_of_frame(-1, S, W) == -1


def test_config_validation(B):
    ok = B.make_cache_config(1, 30, 12, 128, 32, 32, 1, 1, 6, embed_dim=1536)
    assert B.sdv2_cache_bytes(ok) > 0
    bad = [B.make_cache_config(1, 1, 1, 96, 4, 4, 1, 1, 2),          # head_dim
           B.make_cache_config(1, 1, 1, 64, 4, 4, 3, 1, 2),          # window < chunk
           B.make_cache_config(65, 1, 1, 64, 4, 4, 1, 1, 2),         # batch limit
           B.make_cache_config(1, 1, 1, 64, 4, 4, 1, 1, 2, rope_pairs=(10, 10, 10)),  # pairs sum
           B.make_cache_config(1, 1, 1, 64, 4, 4, 1, 1, 2, embed_dim=3)]             # odd embed
    for cfg in bad:
        with pytest.raises(B.SDV2Error):
            B.sdv2_cache_bytes(cfg)


def test_layout_regions_are_disjoint_and_aligned(B):
    cfg = B.make_cache_config(4, 30, 12, 128, 30, 52, 2, 1, 8, embed_dim=1536)
    lay = B.sdv2_cache_layout_of(cfg)
    kv_bytes = 4 * 9 * 1560 * 12 * 128 * 2
    assert lay.layer_stride == kv_bytes
    assert lay.v_offset >= lay.k_offset + 30 * kv_bytes
    offs = [lay.k_offset, lay.v_offset, lay.sink_embed_offset, lay.sink_frame_offset, lay.status_offset,
            lay.scratch_offset]
    assert offs == sorted(offs)
    assert all(o % 256 == 0 for o in offs)
    assert lay.scratch_offset + lay.scratch_bytes == lay.total_bytes == B.sdv2_cache_bytes(cfg)


def test_fp8_layout_and_validation(B):
    # 480x832 latent (N = 1560): slots padded to 13 blocks of 128 tokens
    cfg = B.make_cache_config(4, 30, 12, 128, 30, 52, 2, 1, 8, embed_dim=1536, kv_format="fp8")
    lay = B.sdv2_cache_layout_of(cfg)
    assert lay.tokens_padded == 1664
    assert lay.layer_stride == 4 * 9 * 1664 * 12 * 128                 # one byte per code
    assert lay.scale_slot_stride == 12 * 13 == 156
    assert lay.scale_layer_stride == 4 * 9 * 156 * 4
    offs = [lay.k_offset, lay.v_offset, lay.k_scale_offset, lay.v_scale_offset, lay.sink_embed_offset,
            lay.scratch_offset]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay.v_offset >= lay.k_offset + 30 * lay.layer_stride
    assert lay.v_scale_offset >= lay.k_scale_offset + 30 * lay.scale_layer_stride
    bf16 = B.sdv2_cache_layout_of(B.make_cache_config(4, 30, 12, 128, 30, 52, 2, 1, 8, embed_dim=1536))
    assert bf16.k_scale_offset == 0 and bf16.tokens_padded == 0
    assert lay.total_bytes < bf16.total_bytes                          # half the K/V bytes plus scales
    odd = B.make_cache_config(1, 1, 3, 128, 4, 4, 1, 1, 2, kv_format="fp8")
    assert B.sdv2_cache_layout_of(odd).scale_slot_stride == 4        # 3 heads x 1 block, padded to 4 floats
    for bad in (B.make_cache_config(1, 1, 1, 64, 4, 4, 1, 1, 2, kv_format="fp8"),   # head_dim 64
                B.make_cache_config(1, 1, 1, 128, 4, 4, 1, 1, 2, kv_format=7)):     # unknown format
        with pytest.raises(B.SDV2Error):
            B.sdv2_cache_bytes(bad)


def test_split_plan(B):
    c2 = B.make_cache_config(1, 30, 12, 128, 32, 32, 1, 1, 6)
    # 48 units (12 heads x 4 query-tile pairs) on 148 SMs: every unit split over the KV range
    whole, pieces = B.sdv2_attention_plan(c2, [7168], 148)
    assert whole == 0 and 2 <= pieces <= 16 and 48 * pieces <= 148
    assert B.sdv2_attention_splits(c2, [7168], 148) == pieces
    # 37 heads x 4 pairs = 148 units fill the GPU exactly once: nothing split
    full = B.make_cache_config(1, 1, 37, 128, 32, 32, 1, 1, 6)
    assert B.sdv2_attention_plan(full, [7168], 148) == (148, 1)
    # 624 units are 4 full waves + 32: the 32 of the last wave are split, the rest run whole
    c3 = B.make_cache_config(4, 30, 12, 128, 30, 52, 2, 1, 8)
    whole, pieces = B.sdv2_attention_plan(c3, [14040] * 4, 148)
    assert whole == 4 * 148 and pieces > 1 and (624 - whole) * pieces <= 148
    # 160 units: one full wave whole, the 12 left split finely enough to fill one more wave
    c4 = B.make_cache_config(1, 40, 40, 128, 32, 32, 1, 1, 6)
    whole, pieces = B.sdv2_attention_plan(c4, [7168], 148)
    assert whole == 148 and pieces > 4 and 12 * pieces <= 148
    # pair mode: chunks of one query tile with more (stream, head) units than SMs
    small = B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6)
    assert B.sdv2_attention_pair_mode(small, [448] * 16, 148) == 1
    assert B.sdv2_attention_plan(small, [448] * 16, 148) == (192, 1)
    assert B.sdv2_attention_pair_mode(small, [448] * 12 + [0] * 4, 148) == 0          # 144 units fit one wave
    assert B.sdv2_attention_pair_mode(B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6, kv_format="fp8"),
                                      [448] * 16, 148) == 1                           # both cache formats
    assert B.sdv2_attention_pair_mode(c2, [7168], 148) == 0                           # 1024 queries
    tiny = B.make_cache_config(1, 1, 2, 64, 4, 4, 1, 1, 2)
    assert B.sdv2_attention_plan(tiny, [48], 148) == (2, 1)     # 2 heads, a single KV tile: nothing to split
    assert B.sdv2_attention_plan(c2, [0], 148) == (0, 1)        # no active stream


def _fuse_mode_model(cfg, f0s, sms):
    """The fused append + attention rule restated: bf16 cache, at most 256 queries, at most 4
    chunk frames whose temporal pairs fit 48 entries and whose phases are below 4096 (the cache's
    fp64 phase table), fp64 row and column tables within 256 head_dim - 1024 bytes, the chunk's rows of every
    stream within at
    most two 128-key tiles of its slot-major prefix; pair mode when every stream has one such
    tile, chunks of at most 128 queries, at least two heads and more (stream, head) units than SMs."""
    n = cfg.frame_h * cfg.frame_w
    c2 = cfg.head_dim // 2
    tp, nt = cfg.chunk_frames, (cfg.rope_pairs[0] if any(cfg.rope_pairs) else c2 - 2 * (c2 // 3))
    nh = cfg.rope_pairs[1] if any(cfg.rope_pairs) else c2 // 3
    nw = cfg.rope_pairs[2] if any(cfg.rope_pairs) else c2 // 3
    if cfg.kv_format != 0 or tp * n > 256 or tp > 4 or tp * nt > 48 or 16 * (cfg.frame_h * nh + cfg.frame_w * nw) > 256 * cfg.head_dim - 1024:
        return 0
    reset = cfg.rope_reset_period
    n_phase = min(reset if reset > 0 else 4096, 4096)     # the cache's precomputed temporal phases
    one, active = True, 0
    for f0 in f0s:
        if f0 < 0:
            continue
        active += 1
        if any(O.rope_phase(f0 + i, reset) >= n_phase for i in range(tp)):
            return 0
        tiles = set()
        for i in range(tp):
            s = O.slot_of_frame(f0 + i, cfg.sink_frames, cfg.window_frames)
            tiles |= set(range(s * n // 128, (s * n + n - 1) // 128 + 1))
        if len(tiles) > 2:
            return 0
        one = one and len(tiles) == 1
    pair = one and tp * n <= 128 and cfg.heads >= 2 and active * cfg.heads > sms
    return 2 if pair else 1


def test_append_attention_mode(B):
    small = B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6)
    assert B.sdv2_append_attention_mode(small, [5] * 16, 148) == 2          # 192 units, one tile each
    assert B.sdv2_append_attention_mode(small, [5] * 12 + [-1] * 4, 148) == 1
    assert B.sdv2_append_attention_mode(B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6, kv_format="fp8"),
                                        [5] * 16, 148) == 0
    assert B.sdv2_append_attention_mode(B.make_cache_config(1, 1, 12, 128, 32, 32, 1, 1, 6), [3], 148) == 0
    straddle = B.make_cache_config(16, 1, 12, 128, 8, 12, 1, 2, 4)         # 96 tokens per frame
    assert B.sdv2_append_attention_mode(straddle, [1] * 16, 148) == 1       # rows 96..191: two tiles
    assert B.sdv2_append_attention_mode(straddle, [0] * 16, 148) == 2       # rows 0..95: one tile, pair mode
    two = B.make_cache_config(1, 1, 2, 64, 8, 12, 2, 1, 4)                  # T' = 2, 192 queries
    assert B.sdv2_append_attention_mode(two, [0], 148) == 1
    assert B.sdv2_append_attention_mode(two, [4], 148) == 0                 # slots 4 and 1: three tiles
    assert B.sdv2_append_attention_mode(B.make_cache_config(1, 1, 2, 128, 8, 8, 3, 1, 6), [0], 148) == 0  # 3 x 22 pairs
    assert B.sdv2_append_attention_mode(B.make_cache_config(1, 1, 2, 128, 4, 4, 3, 1, 6, rope_pairs=(10, 27, 27)),
                                        [0], 148) == 1
    assert B.sdv2_append_attention_mode(B.make_cache_config(1, 1, 2, 128, 1, 128, 1, 1, 6), [0], 148) == 0  # 128 x 21 x 16 B
    assert B.sdv2_append_attention_mode(small, [4095] * 16, 148) == 2                 # no reset: phase table 0 .. 4095
    assert B.sdv2_append_attention_mode(small, [4096] + [5] * 15, 148) == 0
    assert B.sdv2_append_attention_mode(B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6, rope_reset_period=9000),
                                        [8999] * 16, 148) == 0                         # phase 8999 > 4095
    assert B.sdv2_append_attention_mode(B.make_cache_config(16, 1, 12, 128, 8, 8, 1, 1, 6, rope_reset_period=300),
                                        [10 ** 6] * 16, 148) == 2
    import random
    rng = random.Random(5)
    for _ in range(400):
        b, h, d = rng.randint(1, 24), rng.choice([1, 2, 7, 12, 13]), rng.choice([64, 128])
        fh, fw, tp = rng.randint(1, 12), rng.choice([rng.randint(1, 16), rng.randint(60, 200)]), rng.randint(1, 5)
        s_, w = rng.randint(1, 3), rng.randint(tp, 8)
        cfg = B.make_cache_config(b, 1, h, d, fh, fw, tp, s_, w, rope_reset_period=rng.choice([0, 0, 7, 5000]))
        if B.lib().sdv2_cache_bytes(cfg) == 0:
            continue                                                        # (a config the library rejects)
        f0s = [rng.choice([-1, rng.randint(0, 40), rng.randint(4000, 4200)]) for _ in range(b)]
        sms = rng.choice([16, 148])
        assert B.sdv2_append_attention_mode(cfg, f0s, sms) == _fuse_mode_model(cfg, f0s, sms), (b, h, d, fh, fw, tp)


def test_null_handles_are_rejected_without_a_device(B):
    import ctypes
    lib = B.lib()
    assert lib.sdv2_cache_time_attention(None, None, None) == B.SDV2_E_ARG
    assert lib.sdv2_cache_check(None) == B.SDV2_E_ARG
    assert lib.sdv2_cache_selftest_wait(None, ctypes.c_uint64(1000), None) == B.SDV2_E_ARG
    assert lib.sdv2_kv_append(None, 0, None, None, None, None) == B.SDV2_E_ARG
    assert "NULL" in lib.sdv2_last_error().decode() or "null" in lib.sdv2_last_error().decode()


def test_plan_properties_over_random_shapes(B):
    import random
    rng = random.Random(11)
    for _ in range(300):
        b, h = rng.randint(1, 16), rng.choice([1, 2, 8, 12, 24, 40])
        fh, fw, tp = rng.randint(1, 40), rng.randint(1, 60), rng.randint(1, 3)
        s_, w = rng.randint(1, 3), rng.randint(3, 10)
        cfg = B.make_cache_config(b, 1, h, 128, fh, fw, tp, s_, max(w, tp))
        n = fh * fw
        keys = [rng.choice([0, (s_ + max(w, tp)) * n, rng.randint(1, (s_ + max(w, tp)) * n)]) for _ in range(b)]
        sms = rng.choice([132, 148, 160])
        whole, pieces = B.sdv2_attention_plan(cfg, keys, sms)
        units = sum(1 for k in keys if k > 0) * h * ((tp * n + 255) // 256)
        assert 1 <= pieces <= 16 and pieces <= max(1, max(-(-k // 128) for k in keys))
        assert 0 <= whole <= units
        if pieces == 1:
            assert whole == units                     # nothing split
        else:
            assert whole == 0 or whole % sms == 0    # whole units fill complete waves
            assert whole < units


def test_fp8_plan_counts_whole_blocks_per_slot(B):
    # N = 1560 tokens per frame: 13 blocks of 128 per slot (the last one holds 24 tokens)
    bf = B.make_cache_config(1, 1, 12, 128, 30, 52, 2, 1, 8)
    f8 = B.make_cache_config(1, 1, 12, 128, 30, 52, 2, 1, 8, kv_format="fp8")
    keys = [9 * 1560]
    tiles_bf, tiles_f8 = -(-9 * 1560 // 128), 9 * 13
    assert tiles_bf == 110 and tiles_f8 == 117
    for cfg in (bf, f8):
        whole, pieces = B.sdv2_attention_plan(cfg, keys, 148)
        assert 1 <= pieces <= 16 and 0 <= whole <= 12 * 13


def test_fp8_plan_packs_64_token_slots_two_to_a_tile(B):
    # 8 x 8 = 64 tokens per frame: the fp8 kernel packs slots 2g and 2g + 1 into KV tile g,
    # so its plan counts ceil(slots / 2) tiles, as the bf16 plan counts ceil(64 slots / 128)
    import random
    rng = random.Random(5)
    for _ in range(200):
        b, h = rng.randint(1, 4), rng.choice([1, 2, 3, 12])
        s_, w = rng.randint(1, 3), rng.randint(1, 9)
        bf = B.make_cache_config(b, 1, h, 128, 8, 8, 1, s_, w)
        f8 = B.make_cache_config(b, 1, h, 128, 8, 8, 1, s_, w, kv_format="fp8")
        keys = [rng.choice([0, 64 * rng.randint(1, s_ + w)]) for _ in range(b)]
        if not any(keys):
            continue
        sms = rng.choice([16, 148])
        assert B.sdv2_attention_plan(f8, keys, sms) == B.sdv2_attention_plan(bf, keys, sms), (b, h, s_, w, keys)
        whole, pieces = B.sdv2_attention_plan(f8, keys, sms)
        assert pieces <= max(1, (max(keys) // 64 + 1) // 2)
    # one stream, two heads, five slots: three tiles, three pieces (five without the packing)
    f8 = B.make_cache_config(1, 1, 2, 128, 8, 8, 1, 1, 4, kv_format="fp8")
    assert B.sdv2_attention_plan(f8, [5 * 64], 148) == (0, 3)
    # 96-token slots are not packed: one padded block per slot, five tiles
    f8 = B.make_cache_config(1, 1, 2, 128, 8, 12, 1, 1, 4, kv_format="fp8")
    assert B.sdv2_attention_plan(f8, [5 * 96], 148)[1] == 5

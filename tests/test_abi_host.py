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


def test_split_plan(B):
    c2 = B.make_cache_config(1, 30, 12, 128, 32, 32, 1, 1, 6)
    s = B.sdv2_attention_splits(c2, [7168], 148)
    # 48 CTAs unsplit on 148 SMs: the plan splits the KV range to fill the GPU
    assert 2 <= s <= 4 and 48 * s <= 148
    c3 = B.make_cache_config(4, 30, 12, 128, 30, 52, 2, 1, 8)
    assert B.sdv2_attention_splits(c3, [14040] * 4, 148) == 1
    tiny = B.make_cache_config(1, 1, 2, 64, 4, 4, 1, 1, 2)
    assert B.sdv2_attention_splits(tiny, [48], 148) == 1
    assert B.sdv2_attention_splits(c2, [0], 148) == 1


def test_null_handles_are_rejected_without_a_device(B):
    import ctypes
    lib = B.lib()
    assert lib.sdv2_cache_time_attention(None, None, None) == B.SDV2_E_ARG
    assert lib.sdv2_cache_check(None) == B.SDV2_E_ARG
    assert lib.sdv2_cache_selftest_wait(None, ctypes.c_uint64(1000), None) == B.SDV2_E_ARG
    assert lib.sdv2_kv_append(None, 0, None, None, None, None) == B.SDV2_E_ARG
    assert "NULL" in lib.sdv2_last_error().decode() or "null" in lib.sdv2_last_error().decode()

"""Stream batch over denoising steps: entry bookkeeping (CPU) and parity through the
CUDA path against the oracle for the same staggered frame positions (GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from harness import ATTN_MAX_ABS, ATTN_MEAN_ABS, attn_errors


def _frames(streams, steps, micro_step, t=1):
    return [((micro_step - k) * t if micro_step - k >= 0 else -1) for s in range(streams) for k in range(steps)]


def test_staggered_positions_and_finished_entries():
    from causal_dit_kv_b200.stream_batch import StreamBatchCache
    sb = StreamBatchCache.__new__(StreamBatchCache)          # bookkeeping only, no device buffer
    sb.streams, sb.steps, sb.chunk_frames, sb.micro_step = 2, 3, 2, 0
    assert sb.chunk_first_frames() == [0, -1, -1, 0, -1, -1]
    assert sb.finished_entries() == []
    sb.micro_step = 4
    assert sb.chunk_first_frames() == [8, 6, 4, 8, 6, 4]
    assert sb.finished_entries() == [2, 5]
    assert sb.entry(1, 2) == 5


@pytest.mark.gpu
def test_stream_batch_parity():
    from causal_dit_kv_b200.stream_batch import StreamBatchCache
    S, n = 2, 3
    cfg = dict(layers=1, heads=2, head_dim=64, frame_h=4, frame_w=6, chunk_frames=1, sink_frames=1, window_frames=3)
    sb = StreamBatchCache(S, n, **cfg)
    ocfg = O.CacheConfig(batch=S * n, **cfg)
    ora = O.OracleCache(ocfg)
    scale = 1.0 / math.sqrt(cfg["head_dim"])
    for m in range(8):
        f0 = sb.chunk_first_frames()
        assert f0 == _frames(S, n, m)
        q, k, v = synth.chunk_qkv(77, S * n, ocfg.chunk_tokens, cfg["heads"], cfg["head_dim"], m, 0)
        sb.append(0, k.cuda(), v.cuda())
        O.kv_append(ora, 0, synth.bf16_bits(k), synth.bf16_bits(v), f0)
        out = torch.zeros((S * n, ocfg.chunk_tokens, cfg["heads"], cfg["head_dim"]), dtype=torch.bfloat16, device="cuda")
        sb.attention(0, q.cuda(), out, scale)
        want = O.chunk_attention(ora, 0, synth.bf16_bits(q), f0, np.float32(scale))
        mx, mean = attn_errors(out, want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (m, mx, mean)
        kg = sb.cache.k_cache(0).cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(kg, ora.k[0])
        sb.advance()
    sb.close()

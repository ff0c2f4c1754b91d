"""The streaming step captured as a CUDA graph: the captured kernels, replayed,
produce the same cache and output bits as the same calls made eagerly, and
every replay of a step reproduces them (B200)."""
import math

import pytest
import torch

import synth
from causal_dit_kv_b200 import KVCache

pytestmark = pytest.mark.gpu

# two query-tile pairs (one ragged) and a 3-way KV split: kernel and merge both captured
CFG = dict(batch=2, layers=2, heads=3, head_dim=128, frame_h=12, frame_w=15, chunk_frames=2, sink_frames=1,
           window_frames=4)


def _step(cache, qkv, out, f0):
    for layer in range(CFG["layers"]):
        q, k, v = qkv[layer]
        cache.kv_append(layer, k, v, f0)
        cache.chunk_attention(layer, q, out[layer], f0, 1.0 / math.sqrt(CFG["head_dim"]))


def test_captured_step_matches_eager_calls():
    B, L, H, D = CFG["batch"], CFG["layers"], CFG["heads"], CFG["head_dim"]
    Lq = CFG["chunk_frames"] * CFG["frame_h"] * CFG["frame_w"]
    steps = [[tuple(t.cuda() for t in synth.chunk_qkv(77, B, Lq, H, D, s, l)) for l in range(L)] for s in range(5)]
    eager, graphed = KVCache(**CFG), KVCache(**CFG)
    out_e = [torch.empty((B, Lq, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    out_g = [torch.empty_like(o) for o in out_e]
    Tp = CFG["chunk_frames"]
    for s in range(4):                                   # ring wrapped before the captured step
        _step(eager, steps[s], out_e, [s * Tp] * B)
        _step(graphed, steps[s], out_g, [s * Tp] * B)
    _step(eager, steps[4], out_e, [4 * Tp] * B)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _step(graphed, steps[4], out_g, [4 * Tp] * B)
    for _ in range(2):                                   # the first replay runs the step; the second repeats it
        graph.replay()
        torch.cuda.synchronize()
        for layer in range(L):
            assert torch.equal(out_g[layer], out_e[layer]), layer
            for get in (KVCache.k_cache, KVCache.v_cache):
                assert torch.equal(get(eager, layer).view(torch.int16), get(graphed, layer).view(torch.int16)), layer
    assert eager.check() == 0 and graphed.check() == 0
    del graph
    eager.close()
    graphed.close()

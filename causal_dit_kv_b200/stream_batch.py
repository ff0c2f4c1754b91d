"""Stream batch over denoising steps: n noise levels x S streams as one cache.

Source: qq8o.cn walkthrough of StreamDiffusionV2, "Multi-pipeline
orchestration extension" (each micro-step emits one fully denoised chunk;
the n denoising steps act as a batch multiplier) and Figure 7 there (depth =
noise level).  Reading: at micro-step m, the chunk that entered the pipeline
at micro-step m - k is at denoising step k, so the n chunks of a stream in
flight are staggered by one chunk each; every (stream, step) pair keeps its
own sink + window cache, and one append and one attention call per layer
serve all n*S entries, each at its own frame position.  Entry (s, k) starts
k micro-steps after entry (s, 0) (pipeline fill) and is skipped until then.

This is bookkeeping over the cache's batch dimension: the kernels already
take a frame position per stream.
"""
from __future__ import annotations

from typing import List

from .stream import KVCache


class StreamBatchCache:
    def __init__(self, streams: int, steps: int, layers: int, heads: int, head_dim: int, frame_h: int, frame_w: int,
                 chunk_frames: int, sink_frames: int, window_frames: int, **kw):
        if streams < 1 or steps < 1:
            raise ValueError("streams and steps must be >= 1")
        self.streams, self.steps, self.chunk_frames = streams, steps, chunk_frames
        self.cache = KVCache(streams * steps, layers, heads, head_dim, frame_h, frame_w, chunk_frames, sink_frames,
                             window_frames, **kw)
        self.micro_step = 0

    def entry(self, stream: int, step: int) -> int:
        """Batch index of (stream, denoising step)."""
        return stream * self.steps + step

    def chunk_first_frames(self) -> List[int]:
        """First frame of each entry's chunk at the current micro-step (-1: not started)."""
        out = []
        for s in range(self.streams):
            for k in range(self.steps):
                c = self.micro_step - k
                out.append(c * self.chunk_frames if c >= 0 else -1)
        return out

    def finished_entries(self) -> List[int]:
        """Entries whose chunk is at the last denoising step this micro-step (their
        attention output completes a chunk)."""
        if self.micro_step - (self.steps - 1) < 0:
            return []
        return [self.entry(s, self.steps - 1) for s in range(self.streams)]

    def append(self, layer: int, k, v, stream=None) -> None:
        self.cache.kv_append(layer, k, v, self.chunk_first_frames(), stream)

    def attention(self, layer: int, q, out, softmax_scale=None, stream=None) -> None:
        self.cache.chunk_attention(layer, q, out, self.chunk_first_frames(), softmax_scale, stream)

    def advance(self) -> None:
        self.micro_step += 1

    def close(self) -> None:
        self.cache.close()

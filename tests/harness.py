"""Drives the CUDA path and the oracle side by side on the same seeded inputs.

Test infrastructure: imports both ``oracle`` and ``causal_dit_kv_b200`` (the
two never import each other) and feeds them the same bytes from ``synth``.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
import synth

ATTN_MAX_ABS = 1.5e-2     # bf16 attention output vs the fp64 oracle, max abs error
ATTN_MEAN_ABS = 2e-3      # ... mean abs error
MOTION_REL = 1e-4         # fp32 motion / EMA outputs, relative error


def f32(x: float) -> float:
    """The value a float argument takes after crossing the C ABI as fp32."""
    return float(np.float32(x))


class PairedStream:
    """One cache config run through the CUDA library and the oracle."""

    def __init__(self, seed=1000, **cfg):
        from causal_dit_kv_b200 import KVCache
        self.seed = seed
        self.cfg = O.CacheConfig(**cfg)
        self.gpu = KVCache(**cfg)
        self.ora = O.OracleCache(self.cfg)
        self.next = [0] * self.cfg.batch
        self.step_idx = 0

    def inputs(self, layer):
        c = self.cfg
        return synth.chunk_qkv(self.seed, c.batch, c.chunk_tokens, c.heads, c.head_dim, self.step_idx, layer)

    def append(self, layer, f0, k, v):
        self.gpu.kv_append(layer, k.cuda(), v.cuda(), f0)
        O.kv_append(self.ora, layer, synth.bf16_bits(k), synth.bf16_bits(v), f0)

    def attention(self, layer, f0, q, rows=None):
        c = self.cfg
        out = torch.zeros((c.batch, c.chunk_tokens, c.heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
        scale = 1.0 / math.sqrt(c.head_dim)
        self.gpu.chunk_attention(layer, q.cuda(), out, f0, scale)
        want = O.chunk_attention(self.ora, layer, synth.bf16_bits(q), f0, f32(scale), rows=rows)
        return out, want

    def append_attention(self, layer, f0, q, k, v, rows=None):
        """The fused call on the GPU; the oracle's append, then its attention."""
        c = self.cfg
        out = torch.zeros((c.batch, c.chunk_tokens, c.heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
        scale = 1.0 / math.sqrt(c.head_dim)
        self.gpu.append_attention(layer, q.cuda(), k.cuda(), v.cuda(), out, f0, scale)
        O.kv_append(self.ora, layer, synth.bf16_bits(k), synth.bf16_bits(v), f0)
        want = O.chunk_attention(self.ora, layer, synth.bf16_bits(q), f0, f32(scale), rows=rows)
        return out, want

    def advance(self, active=None):
        """Next chunk's first frames (negative for streams not in ``active``)."""
        c = self.cfg
        f0 = []
        for b in range(c.batch):
            if active is None or b in active:
                f0.append(self.next[b])
                self.next[b] += c.chunk_frames
            else:
                f0.append(-1)
        return f0


def cache_bits_equal(ps: PairedStream, layer: int):
    k = ps.gpu.k_cache(layer).cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    v = ps.gpu.v_cache(layer).cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.array_equal(k, ps.ora.k[layer]), np.array_equal(v, ps.ora.v[layer]), k, v


def attn_errors(gpu_out: torch.Tensor, want: np.ndarray, rows=None):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g = g[:, rows]
        want = want[:, rows]
    mask = ~np.isnan(want)
    err = np.abs(g[mask] - want[mask])
    return float(err.max()), float(err.mean())

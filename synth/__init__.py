"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no RoPE, no attention, no cosine, no motion measure).
Every generator returns CPU torch tensors (callers move them to the GPU or
view their bits for the oracle), except ``chunk_qkv_on``, which draws the same
distribution directly on a device for benchmark inputs too large to draw on
the host (its values differ from ``chunk_qkv``'s; no oracle comparison uses it).  The recipes mirror the shapes and value
distributions of the streamed workloads: Q/K/V ~ N(0, 1) rounded to bf16,
chunk hidden states around a slowly drifting direction with seeded scene
cuts, and latent frames whose inter-frame steps follow a seeded piecewise-
constant magnitude schedule.
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_bf16(seed: int, shape) -> torch.Tensor:
    """N(0, 1) fp32 draws rounded to bf16 (torch's round-to-nearest-even)."""
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (a view, no rounding)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def chunk_qkv(seed: int, batch: int, chunk_tokens: int, heads: int, head_dim: int, step: int, layer: int):
    """Q, K, V [B][T'*N][H][d] bf16 for one streamed chunk of one layer."""
    base = (int(seed) * 1_000_003 + int(step) * 7919 + int(layer) * 104_729) & 0x7FFFFFFF
    shape = (batch, chunk_tokens, heads, head_dim)
    return (randn_bf16(base + 1, shape), randn_bf16(base + 2, shape), randn_bf16(base + 3, shape))


def chunk_qkv_on(device, seed: int, batch: int, chunk_tokens: int, heads: int, head_dim: int, step: int,
                 layer: int):
    """Q, K, V [B][T'*N][H][d] bf16 ~ N(0, 1) drawn on ``device`` with a seeded generator
    of that device (benchmark inputs only)."""
    import torch as _t
    base = (int(seed) * 1_000_003 + int(step) * 7919 + int(layer) * 104_729) & 0x7FFFFFFF
    g = _t.Generator(device=device)
    g.manual_seed(base)
    shape = (3, batch, chunk_tokens, heads, head_dim)
    x = _t.randn(shape, generator=g, dtype=_t.float32, device=device).to(_t.bfloat16)
    return x[0], x[1], x[2]


def drifting_hidden(seed: int, batch: int, chunk_tokens: int, dim: int, n_chunks: int,
                    drift: float = 0.08, amplitude: float = 0.5, cut_prob: float = 0.01):
    """Generator of hidden states [B][T'*N][D] bf16, one chunk per ``next()``.

    Each stream has a unit direction u that takes a Gaussian step of size
    ``drift`` per chunk and jumps to a fresh random direction with
    probability ``cut_prob`` (a scene cut).  Tokens are
    amplitude*sqrt(D)*u + N(0, 1).
    """
    g = _gen(seed)
    u = torch.randn((batch, dim), generator=g, dtype=torch.float64)
    u = u / u.norm(dim=1, keepdim=True)
    for _ in range(n_chunks):
        step = torch.randn((batch, dim), generator=g, dtype=torch.float64)
        u = u + drift * step / np.sqrt(dim)
        cut = torch.rand((batch,), generator=g, dtype=torch.float64) < cut_prob
        if bool(cut.any()):
            fresh = torch.randn((batch, dim), generator=g, dtype=torch.float64)
            u = torch.where(cut[:, None], fresh, u)
        u = u / u.norm(dim=1, keepdim=True)
        noise = torch.randn((batch, chunk_tokens, dim), generator=g, dtype=torch.float32)
        tok = amplitude * np.sqrt(dim) * u[:, None, :].to(torch.float32) + noise
        yield tok.to(torch.bfloat16)


def motion_latents(seed: int, batch: int, chunk_frames: int, channels: int, height: int, width: int,
                   n_chunks: int, sigma: float = 2.0, seg_min: int = 32, seg_max: int = 256):
    """Generator of latent chunks [B][T'][C][H][W] fp32, one per ``next()``.

    x_t = x_{t-1} + m * xi_t with xi ~ N(0, 1); the step magnitude m is
    constant over seeded segments of seg_min..seg_max frames and drawn from
    {0, sigma/4, sigma/2, sigma, 2*sigma}.
    """
    g = _gen(seed)
    levels = [0.0, 0.25 * sigma, 0.5 * sigma, sigma, 2.0 * sigma]
    x = torch.randn((batch, channels, height, width), generator=g, dtype=torch.float32)
    seg_left = [0] * batch
    mag = [0.0] * batch
    for _ in range(n_chunks):
        frames = []
        for _t in range(chunk_frames):
            steps = torch.randn((batch, channels, height, width), generator=g, dtype=torch.float32)
            m = torch.empty(batch, dtype=torch.float32)
            for b in range(batch):
                if seg_left[b] <= 0:
                    seg_left[b] = int(torch.randint(seg_min, seg_max + 1, (1,), generator=g))
                    mag[b] = levels[int(torch.randint(0, len(levels), (1,), generator=g))]
                seg_left[b] -= 1
                m[b] = mag[b]
            x = x + m[:, None, None, None] * steps
            frames.append(x.clone())
        yield torch.stack(frames, dim=1)

"""Handles that own their device buffers through torch and call libsdv2.

torch allocates the cache / motion-state buffers and names the stream; every
step of the path runs in the library's kernels.
"""
from __future__ import annotations

import math

from . import binding as B


class KVCache:
    """Sink + rolling-window K/V cache of ``layers`` DiT layers for ``batch`` streams."""

    def __init__(self, batch, layers, heads, head_dim, frame_h, frame_w, chunk_frames, sink_frames, window_frames,
                 rope_pairs=(0, 0, 0), rope_reset_period=0, embed_dim=0, rope_base=10000.0, device="cuda",
                 kv_format="bf16"):
        import torch
        self.cfg = B.make_cache_config(batch, layers, heads, head_dim, frame_h, frame_w, chunk_frames, sink_frames,
                                       window_frames, rope_pairs, rope_reset_period, embed_dim, rope_base, kv_format)
        self.kv_format = kv_format
        self.nbytes = B.sdv2_cache_bytes(self.cfg)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.handle = B.sdv2_cache_create(self.cfg, self.buffer, self.nbytes)
        self.layout = B.sdv2_cache_layout_get(self.handle)
        self.batch, self.layers, self.heads, self.head_dim = batch, layers, heads, head_dim
        self.frame_h, self.frame_w, self.chunk_frames = frame_h, frame_w, chunk_frames
        self.sink_frames, self.window_frames, self.embed_dim = sink_frames, window_frames, embed_dim
        self.tokens_per_frame = frame_h * frame_w
        self.chunk_tokens = chunk_frames * self.tokens_per_frame
        self.slots = sink_frames + window_frames

    def close(self):
        if self.handle:
            B.sdv2_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the path
    def kv_append(self, layer, k, v, chunk_first_frame, stream=None):
        B.sdv2_kv_append(self.handle, layer, k, v, chunk_first_frame, self.batch, stream)

    def chunk_attention(self, layer, q, out, chunk_first_frame, softmax_scale=None, stream=None):
        scale = 1.0 / math.sqrt(self.head_dim) if softmax_scale is None else softmax_scale
        B.sdv2_chunk_attention(self.handle, layer, q, out, chunk_first_frame, scale, self.batch, stream)

    def append_attention(self, layer, q, k, v, out, chunk_first_frame, softmax_scale=None, stream=None):
        """kv_append then chunk_attention of the same chunk, fused into one launch where it applies."""
        scale = 1.0 / math.sqrt(self.head_dim) if softmax_scale is None else softmax_scale
        B.sdv2_append_attention(self.handle, layer, q, k, v, out, chunk_first_frame, scale, self.batch, stream)

    def append_attention_mode(self, chunk_first_frame, sm_count):
        return B.sdv2_append_attention_mode(self.cfg, chunk_first_frame, sm_count)

    def time_attention(self, start=None, stop=None):
        """Record torch.cuda.Event start/stop (enable_timing=True, already recorded once so
        that they exist) around the attention kernel of the following chunk_attention
        calls; time_attention() switches it off."""
        B.sdv2_cache_time_attention(self.handle, start, stop)

    def sink_refresh(self, hidden, tau, chunk_first_frame, out_slot, stream=None):
        B.sdv2_sink_refresh(self.handle, hidden, tau, chunk_first_frame, out_slot, self.batch, stream)

    # -- views of the caller-owned buffer (for inspection and tests)
    def _region(self, offset, nbytes, dtype, shape):
        import torch
        return self.buffer[offset:offset + nbytes].view(dtype).view(*shape)

    def k_cache(self, layer):
        import torch
        if self.kv_format != "bf16":
            raise ValueError("an fp8 cache holds codes: use k_codes / v_codes / k_scales / v_scales")
        shape = (self.batch, self.slots, self.tokens_per_frame, self.heads, self.head_dim)
        off = self.layout.k_offset + layer * self.layout.layer_stride
        return self._region(off, self.layout.layer_stride, torch.bfloat16, shape)

    def v_cache(self, layer):
        import torch
        if self.kv_format != "bf16":
            raise ValueError("an fp8 cache holds codes: use k_codes / v_codes / k_scales / v_scales")
        shape = (self.batch, self.slots, self.tokens_per_frame, self.heads, self.head_dim)
        off = self.layout.v_offset + layer * self.layout.layer_stride
        return self._region(off, self.layout.layer_stride, torch.bfloat16, shape)

    # fp8 cache: E4M3 codes (uint8) and their per-block scales
    def k_codes(self, layer):
        """uint8 [B][S+W][Np][H][d]."""
        import torch
        shape = (self.batch, self.slots, self.layout.tokens_padded, self.heads, self.head_dim)
        return self._region(self.layout.k_offset + layer * self.layout.layer_stride, self.layout.layer_stride,
                            torch.uint8, shape)

    def v_codes(self, layer):
        """uint8 [B][S+W][H][d][Np] (token index innermost)."""
        import torch
        shape = (self.batch, self.slots, self.heads, self.head_dim, self.layout.tokens_padded)
        return self._region(self.layout.v_offset + layer * self.layout.layer_stride, self.layout.layer_stride,
                            torch.uint8, shape)

    def _scales(self, offset, layer):
        import torch
        nb = self.layout.tokens_padded // 128
        full = self._region(offset + layer * self.layout.scale_layer_stride, self.layout.scale_layer_stride,
                            torch.float32, (self.batch, self.slots, self.layout.scale_slot_stride))
        return full[:, :, :self.heads * nb].reshape(self.batch, self.slots, self.heads, nb)

    def k_scales(self, layer):
        """fp32 [B][S+W][H][Np/128]."""
        return self._scales(self.layout.k_scale_offset, layer)

    def v_scales(self, layer):
        return self._scales(self.layout.v_scale_offset, layer)

    def sink_embed(self):
        import torch
        d = max(self.embed_dim, 1)
        return self._region(self.layout.sink_embed_offset, 8 * self.batch * self.sink_frames * d, torch.float64,
                            (self.batch, self.sink_frames, d))

    def sink_frame(self):
        import torch
        return self._region(self.layout.sink_frame_offset, 8 * self.batch * self.sink_frames, torch.int64,
                            (self.batch, self.sink_frames))

    def status_word(self):
        import torch
        return self._region(self.layout.status_offset, 4, torch.int32, (1,))

    def query(self, b, layer):
        return B.sdv2_cache_query(self.handle, b, layer, self.slots)

    def check(self):
        return B.sdv2_cache_check(self.handle)


class MotionState:
    """Motion-aware noise-rate state of ``batch`` streams."""

    def __init__(self, batch, chunk_frames, channels, height, width, window=4, sigma=2.0, lam=0.9, s_min=0.5,
                 s_max=0.9, s_init=0.7, device="cuda"):
        import torch
        self.cfg = B.make_motion_config(batch, chunk_frames, channels, height, width, window, sigma, lam, s_min,
                                        s_max, s_init)
        self.nbytes = B.sdv2_motion_bytes(self.cfg)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.handle = B.sdv2_motion_create(self.cfg, self.buffer, self.nbytes)
        self.batch, self.chunk_frames = batch, chunk_frames

    def close(self):
        if self.handle:
            B.sdv2_motion_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def noise_rate(self, latents, out_rate, out_d=None, stream=None):
        B.sdv2_motion_noise_rate(self.handle, latents, out_rate, out_d, stream)

    def check(self):
        return B.sdv2_motion_check(self.handle)

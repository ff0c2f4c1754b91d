"""ctypes binding of libsdv2 (include/sdv2.h): argument marshalling only.

Every function keeps the C name and forwards device pointers, sizes and the
CUDA stream; all work runs in the library's kernels.  torch is used only to
own device memory and to name the current stream.  The library must be
built (``python -m causal_dit_kv_b200.build``); nothing here falls back to
another implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_uint32, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsdv2.so")

SDV2_OK, SDV2_E_ARG, SDV2_E_SHAPE, SDV2_E_ALIGN, SDV2_E_STATE, SDV2_E_CUDA, SDV2_E_DEVICE = 0, -1, -2, -3, -4, -5, -6
STATUS_NAMES = {0: "SDV2_OK", -1: "SDV2_E_ARG", -2: "SDV2_E_SHAPE", -3: "SDV2_E_ALIGN", -4: "SDV2_E_STATE",
                -5: "SDV2_E_CUDA", -6: "SDV2_E_DEVICE"}


class sdv2_cache_config(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("layers", c_int32), ("heads", c_int32), ("head_dim", c_int32),
                ("frame_h", c_int32), ("frame_w", c_int32), ("chunk_frames", c_int32), ("sink_frames", c_int32),
                ("window_frames", c_int32), ("rope_pairs", c_int32 * 3), ("rope_reset_period", c_int32),
                ("embed_dim", c_int32), ("rope_base", c_double), ("kv_format", c_int32)]


KV_BF16, KV_FP8_E4M3 = 0, 1
KV_FORMATS = {"bf16": KV_BF16, "fp8": KV_FP8_E4M3}


class sdv2_cache_layout(ctypes.Structure):
    _fields_ = [("k_offset", c_uint64), ("v_offset", c_uint64), ("layer_stride", c_uint64),
                ("sink_embed_offset", c_uint64), ("sink_frame_offset", c_uint64), ("status_offset", c_uint64),
                ("scratch_offset", c_uint64), ("scratch_bytes", c_uint64), ("total_bytes", c_uint64),
                ("k_scale_offset", c_uint64), ("v_scale_offset", c_uint64), ("scale_layer_stride", c_uint64),
                ("scale_slot_stride", c_uint32), ("tokens_padded", c_uint32)]


class sdv2_motion_config(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("chunk_frames", c_int32), ("channels", c_int32), ("height", c_int32),
                ("width", c_int32), ("window", c_int32), ("sigma", c_double), ("lambda_", c_double),
                ("s_min", c_double), ("s_max", c_double), ("s_init", c_double)]


class SDV2Error(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None

# (name, restype, argtypes) of every exported symbol.
_SIGNATURES = [
    ("sdv2_cache_bytes", c_size_t, [POINTER(sdv2_cache_config)]),
    ("sdv2_cache_layout_of", c_int32, [POINTER(sdv2_cache_config), POINTER(sdv2_cache_layout)]),
    ("sdv2_cache_create", c_int32, [POINTER(sdv2_cache_config), c_void_p, c_size_t, POINTER(c_void_p)]),
    ("sdv2_cache_destroy", c_int32, [c_void_p]),
    ("sdv2_kv_append", c_int32, [c_void_p, c_int32, c_void_p, c_void_p, POINTER(c_int64), c_void_p]),
    ("sdv2_chunk_attention", c_int32, [c_void_p, c_int32, c_void_p, c_void_p, POINTER(c_int64), c_float, c_void_p]),
    ("sdv2_append_attention", c_int32,
     [c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, POINTER(c_int64), c_float, c_void_p]),
    ("sdv2_sink_refresh", c_int32, [c_void_p, c_void_p, c_float, POINTER(c_int64), c_void_p, c_void_p]),
    ("sdv2_cache_query", c_int32, [c_void_p, c_int32, c_int32, POINTER(c_int64), POINTER(c_int32), POINTER(c_int32)]),
    ("sdv2_cache_layout_get", c_int32, [c_void_p, POINTER(sdv2_cache_layout)]),
    ("sdv2_cache_check", c_int32, [c_void_p]),
    ("sdv2_cache_selftest_wait", c_int32, [c_void_p, c_uint64, c_void_p]),
    ("sdv2_cache_time_attention", c_int32, [c_void_p, c_void_p, c_void_p]),
    ("sdv2_motion_bytes", c_size_t, [POINTER(sdv2_motion_config)]),
    ("sdv2_motion_create", c_int32, [POINTER(sdv2_motion_config), c_void_p, c_size_t, POINTER(c_void_p)]),
    ("sdv2_motion_destroy", c_int32, [c_void_p]),
    ("sdv2_motion_noise_rate", c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    ("sdv2_motion_check", c_int32, [c_void_p]),
    ("sdv2_motion_noise_rate_noalloc", c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    ("sdv2_slot_of_frame", c_int32, [c_int64, c_int32, c_int32]),
    ("sdv2_rope_phase", c_int64, [c_int64, c_int32]),
    ("sdv2_valid_slots", None, [c_int64, c_int32, c_int32, POINTER(c_int32), POINTER(c_int32)]),
    ("sdv2_attention_splits", c_int32, [POINTER(sdv2_cache_config), POINTER(c_int64), c_int32]),
    ("sdv2_attention_plan", c_int32, [POINTER(sdv2_cache_config), POINTER(c_int64), c_int32, POINTER(c_int32),
                                      POINTER(c_int32)]),
    ("sdv2_attention_pair_mode", c_int32, [POINTER(sdv2_cache_config), POINTER(c_int64), c_int32]),
    ("sdv2_append_attention_mode", c_int32, [POINTER(sdv2_cache_config), POINTER(c_int64), c_int32]),
    ("sdv2_launch_count", c_uint64, []),
    ("sdv2_last_error", c_char_p, []),
    ("sdv2_version", c_char_p, []),
]
EXPORTED = [name for name, _, _ in _SIGNATURES]


def lib():
    """The loaded libsdv2 (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m causal_dit_kv_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, restype, argtypes in _SIGNATURES:
            fn = getattr(handle, name)
            fn.restype = restype
            fn.argtypes = argtypes
        _lib = handle
    return _lib


def _check(status: int, where: str):
    if status != SDV2_OK:
        raise SDV2Error(status, where, lib().sdv2_last_error().decode())


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if not x.is_cuda:
            raise ValueError("expected a device tensor")
        if not x.is_contiguous():
            raise ValueError("expected a contiguous tensor")
        return x.data_ptr()
    raise TypeError(f"cannot pass {type(x)} as a device pointer")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _frames(chunk_first_frame, batch: int):
    arr = (c_int64 * batch)(*[int(x) for x in chunk_first_frame])
    return arr


def make_cache_config(batch, layers, heads, head_dim, frame_h, frame_w, chunk_frames, sink_frames, window_frames,
                      rope_pairs=(0, 0, 0), rope_reset_period=0, embed_dim=0, rope_base=10000.0,
                      kv_format="bf16") -> sdv2_cache_config:
    cfg = sdv2_cache_config()
    cfg.batch, cfg.layers, cfg.heads, cfg.head_dim = batch, layers, heads, head_dim
    cfg.frame_h, cfg.frame_w, cfg.chunk_frames = frame_h, frame_w, chunk_frames
    cfg.sink_frames, cfg.window_frames = sink_frames, window_frames
    cfg.rope_pairs = (c_int32 * 3)(*rope_pairs)
    cfg.rope_reset_period, cfg.embed_dim, cfg.rope_base = rope_reset_period, embed_dim, rope_base
    cfg.kv_format = KV_FORMATS[kv_format] if isinstance(kv_format, str) else int(kv_format)
    return cfg


def make_motion_config(batch, chunk_frames, channels, height, width, window=4, sigma=2.0, lam=0.9, s_min=0.5,
                       s_max=0.9, s_init=0.7) -> sdv2_motion_config:
    cfg = sdv2_motion_config()
    cfg.batch, cfg.chunk_frames, cfg.channels, cfg.height, cfg.width = batch, chunk_frames, channels, height, width
    cfg.window, cfg.sigma, cfg.lambda_, cfg.s_min, cfg.s_max, cfg.s_init = window, sigma, lam, s_min, s_max, s_init
    return cfg


# ---------------------------------------------------------------- C-named calls

def sdv2_cache_bytes(cfg: sdv2_cache_config) -> int:
    n = lib().sdv2_cache_bytes(ctypes.byref(cfg))
    if n == 0:
        raise SDV2Error(SDV2_E_SHAPE, "sdv2_cache_bytes", lib().sdv2_last_error().decode())
    return int(n)


def sdv2_cache_layout_of(cfg: sdv2_cache_config) -> sdv2_cache_layout:
    out = sdv2_cache_layout()
    _check(lib().sdv2_cache_layout_of(ctypes.byref(cfg), ctypes.byref(out)), "sdv2_cache_layout_of")
    return out


def sdv2_cache_create(cfg: sdv2_cache_config, dev_buf, nbytes: int) -> int:
    h = c_void_p()
    _check(lib().sdv2_cache_create(ctypes.byref(cfg), _ptr(dev_buf), nbytes, ctypes.byref(h)), "sdv2_cache_create")
    return h.value


def sdv2_cache_destroy(cache: int) -> None:
    _check(lib().sdv2_cache_destroy(cache), "sdv2_cache_destroy")


def sdv2_kv_append(cache: int, layer: int, k, v, chunk_first_frame, batch: int, stream=None) -> None:
    _check(lib().sdv2_kv_append(cache, layer, _ptr(k), _ptr(v), _frames(chunk_first_frame, batch), _stream(stream)),
           "sdv2_kv_append")


def sdv2_chunk_attention(cache: int, layer: int, q, out, chunk_first_frame, softmax_scale: float, batch: int,
                         stream=None) -> None:
    _check(lib().sdv2_chunk_attention(cache, layer, _ptr(q), _ptr(out), _frames(chunk_first_frame, batch),
                                      float(softmax_scale), _stream(stream)), "sdv2_chunk_attention")


def sdv2_append_attention(cache: int, layer: int, q, k, v, out, chunk_first_frame, softmax_scale: float, batch: int,
                          stream=None) -> None:
    _check(lib().sdv2_append_attention(cache, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                       _frames(chunk_first_frame, batch), float(softmax_scale), _stream(stream)),
           "sdv2_append_attention")


def sdv2_sink_refresh(cache: int, hidden, tau: float, chunk_first_frame, out_slot, batch: int, stream=None) -> None:
    _check(lib().sdv2_sink_refresh(cache, _ptr(hidden), float(tau), _frames(chunk_first_frame, batch), _ptr(out_slot),
                                   _stream(stream)), "sdv2_sink_refresh")


def sdv2_cache_query(cache: int, b: int, layer: int, slots: int):
    frames = (c_int64 * slots)()
    phases = (c_int32 * slots)()
    valid = c_int32()
    _check(lib().sdv2_cache_query(cache, b, layer, frames, phases, ctypes.byref(valid)), "sdv2_cache_query")
    return list(frames), list(phases), valid.value


def sdv2_cache_layout_get(cache: int) -> sdv2_cache_layout:
    out = sdv2_cache_layout()
    _check(lib().sdv2_cache_layout_get(cache, ctypes.byref(out)), "sdv2_cache_layout_get")
    return out


def sdv2_cache_check(cache: int) -> int:
    return int(lib().sdv2_cache_check(cache))


def sdv2_cache_selftest_wait(cache: int, limit_ns: int, stream=None) -> None:
    _check(lib().sdv2_cache_selftest_wait(cache, int(limit_ns), _stream(stream)), "sdv2_cache_selftest_wait")


def sdv2_cache_time_attention(cache: int, start=None, stop=None) -> None:
    """Record torch.cuda.Event `start`/`stop` around the attention kernel of every
    following sdv2_chunk_attention call (None, None switches it off)."""
    s = ctypes.c_void_p(start.cuda_event) if start is not None else None
    t = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
    _check(lib().sdv2_cache_time_attention(cache, s, t), "sdv2_cache_time_attention")


def sdv2_motion_bytes(cfg: sdv2_motion_config) -> int:
    n = lib().sdv2_motion_bytes(ctypes.byref(cfg))
    if n == 0:
        raise SDV2Error(SDV2_E_SHAPE, "sdv2_motion_bytes", lib().sdv2_last_error().decode())
    return int(n)


def sdv2_motion_create(cfg: sdv2_motion_config, dev_buf, nbytes: int) -> int:
    h = c_void_p()
    _check(lib().sdv2_motion_create(ctypes.byref(cfg), _ptr(dev_buf), nbytes, ctypes.byref(h)), "sdv2_motion_create")
    return h.value


def sdv2_motion_destroy(motion: int) -> None:
    _check(lib().sdv2_motion_destroy(motion), "sdv2_motion_destroy")


def sdv2_motion_noise_rate(motion: int, latents, out_rate, out_d=None, stream=None) -> None:
    _check(lib().sdv2_motion_noise_rate(motion, _ptr(latents), _ptr(out_rate), _ptr(out_d), _stream(stream)),
           "sdv2_motion_noise_rate")


def sdv2_motion_noise_rate_noalloc(motion: int, latents, out_rate, out_d=None, stream=None) -> None:
    """Same as sdv2_motion_noise_rate with the library's fixed scratch (no caller scratch)."""
    _check(lib().sdv2_motion_noise_rate_noalloc(motion, _ptr(latents), _ptr(out_rate), _ptr(out_d),
                                                _stream(stream)), "sdv2_motion_noise_rate_noalloc")


def sdv2_motion_check(motion: int) -> int:
    return int(lib().sdv2_motion_check(motion))


def sdv2_slot_of_frame(f: int, sink_frames: int, window_frames: int) -> int:
    return int(lib().sdv2_slot_of_frame(f, sink_frames, window_frames))


def sdv2_rope_phase(f: int, rope_reset_period: int) -> int:
    return int(lib().sdv2_rope_phase(f, rope_reset_period))


def sdv2_valid_slots(frame_end: int, sink_frames: int, window_frames: int):
    sv, wv = c_int32(), c_int32()
    lib().sdv2_valid_slots(frame_end, sink_frames, window_frames, ctypes.byref(sv), ctypes.byref(wv))
    return sv.value, wv.value


def sdv2_attention_splits(cfg: sdv2_cache_config, keys, sm_count: int) -> int:
    arr = (c_int64 * cfg.batch)(*[int(k) for k in keys])
    return int(lib().sdv2_attention_splits(ctypes.byref(cfg), arr, sm_count))


def sdv2_attention_pair_mode(cfg: sdv2_cache_config, keys, sm_count: int) -> int:
    arr = (c_int64 * cfg.batch)(*[int(k) for k in keys])
    return int(lib().sdv2_attention_pair_mode(ctypes.byref(cfg), arr, sm_count))


def sdv2_append_attention_mode(cfg: sdv2_cache_config, chunk_first_frame, sm_count: int) -> int:
    """0: two launches, 1: fused kernel, 2: fused kernel in the pair mode (-1: bad argument)."""
    arr = (c_int64 * cfg.batch)(*[int(f) for f in chunk_first_frame])
    return int(lib().sdv2_append_attention_mode(ctypes.byref(cfg), arr, sm_count))


def sdv2_attention_plan(cfg: sdv2_cache_config, keys, sm_count: int):
    """(whole_units, pieces): units [0, whole_units) run whole, the rest in `pieces` KV pieces."""
    arr = (c_int64 * cfg.batch)(*[int(k) for k in keys])
    whole, pieces = c_int32(0), c_int32(0)
    _check(lib().sdv2_attention_plan(ctypes.byref(cfg), arr, sm_count, ctypes.byref(whole), ctypes.byref(pieces)),
           "sdv2_attention_plan")
    return int(whole.value), int(pieces.value)


def sdv2_launch_count() -> int:
    return int(lib().sdv2_launch_count())


def sdv2_last_error() -> str:
    return lib().sdv2_last_error().decode()


def sdv2_version() -> str:
    return lib().sdv2_version().decode()

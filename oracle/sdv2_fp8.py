"""fp8 (E4M3) KV cache of the oracle: block-scaled storage of the cached keys and values.

TEST INFRASTRUCTURE ONLY (same rules as ``sdv2_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import it; it
shares no code with the CUDA path).

Source: agentlens project page "chenfengxu714/StreamDiffusionV2", roadmap
(FP8 support listed as planned work).  The page names the format only; the
readings taken here:

  * Format: OCP FP8 E4M3 (the "e4m3fn" variant): 1 sign bit, 4 exponent bits
    with bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN; largest
    finite magnitude 448 (1.75 * 2^8); subnormals are m * 2^-9, m = 1..7.
  * What is stored: the same values the bf16 cache holds (keys rotated by
    3D RoPE and rounded to bf16 once, values as given), quantised in blocks.
    A slot's N tokens are cut into blocks of 128 consecutive tokens (the
    last block may be shorter); every (layer, stream, slot, head, block) has
    one fp32 scale for K and one for V.
  * Quantisation of a block, all in fp32 with round-to-nearest-even:
        amax  = max |x| over the block's tokens and the head's d channels
        scale = amax / 448                    (the stored scale)
        inv   = 448 / amax, or 0 when amax == 0; +inf is replaced by the
                largest finite fp32 value (amax below 448 / FLT_MAX)
        code  = E4M3_RNE(x * inv), saturating to +-448
    The dequantised value is decode(code) * scale.
  * What the format is, independent of any storage order: for every
    (layer, stream, slot, token, head) the d codes of K and the d codes of V,
    and for every (layer, stream, slot, head, block of 128 tokens) one K
    scale and one V scale.  The arrays below index exactly that:
    K8, V8 [L][B][S+W][N][H][d], scales [L][B][S+W][H][ceil(N / 128)].
    The last block of a slot whose N is not a multiple of 128 holds fewer
    tokens; its scale is taken over those tokens only.
  * Attention: softmax(scale * RoPE(q) K^T) V evaluated in fp64 on the
    dequantised K and V of the valid slots, with q unquantised.  The CUDA
    path also rounds q (per row) and the probabilities to E4M3 before its
    tensor-core products; the tests' tolerance for this format covers those
    two roundings (each at most 2^-4 relative).
"""
from __future__ import annotations

import numpy as np

from .sdv2_oracle import (CacheConfig, OracleCache, bf16_decode, chunk_queries_rotated, kv_append,
                          attention_reference, sink_refresh, slot_of_frame, valid_slot_counts)

E4M3_MAX = 448.0
BLOCK_TOKENS = 128
_FLT_MAX = float(np.finfo(np.float32).max)


# --------------------------------------------------------------------------
# E4M3 encoding
# --------------------------------------------------------------------------

def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even, saturating at +-448.

    Normal values 2^-6 <= |x| have 4 significant bits: for 2^e <= |x| <
    2^(e+1) the spacing is 2^(e-3).  Below 2^-6 the spacing is the subnormal
    quantum 2^-9.  |x| / spacing is exact in fp64 (a power-of-two scale),
    ``np.rint`` rounds it half-to-even and the product back is exact.  A
    result above 448 becomes 448 (saturation, the rule of the conversion the
    cache uses).  Signs, including that of zero, are kept.  NaN is rejected.
    """
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no place in the cache")
    a = np.abs(x)
    _, e = np.frexp(np.where(a > 0, a, 1.0))          # a = m * 2^e, 0.5 <= m < 1, so 2^(e-1) <= a < 2^e
    q_exp = np.maximum(e.astype(np.int64) - 1 - 3, -9)
    q = np.ldexp(1.0, q_exp)
    r = np.rint(a / q) * q
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp64 -> E4M3 bit patterns (uint8), rounding with :func:`e4m3_round`."""
    r = e4m3_round(x)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << np.uint8(7)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    e = e.astype(np.int64) - 1                          # a = 1.m * 2^e for normal a
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, np.ldexp(a, -e) - 1.0, np.ldexp(a, 9)) * np.where(normal, 8.0, 1.0)
    mant_i = mant.astype(np.int64)
    assert np.all(mant_i == mant) and np.all((mant_i >= 0) & (mant_i < 8))
    return (sign | ((exp_field.astype(np.uint8) & 0xF) << 3) | mant_i.astype(np.uint8)).astype(np.uint8)


def e4m3_decode(bits: np.ndarray) -> np.ndarray:
    """E4M3 bit patterns (uint8) -> exact fp64 values (NaN for S.1111.111)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    ef = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(ef == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp(1.0 + m / 8.0, (ef - 7).astype(np.int64)))
    val = np.where((ef == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def quantize_block(x: np.ndarray):
    """Quantise one block (any shape, fp64 values that are fp32-exact).

    Returns (codes uint8 of x's shape, scale as an fp32 value).  The three
    fp32 operations (the scale, the inverse, the product) are each rounded
    once to nearest-even, as numpy's float32 arithmetic does.
    """
    x32 = np.asarray(x, dtype=np.float32)
    assert np.array_equal(x32.astype(np.float64), np.asarray(x, dtype=np.float64)), "inputs must be fp32 values"
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
    scale = np.float32(amax / np.float32(E4M3_MAX))
    if amax == 0:
        inv = np.float32(0.0)
    else:
        with np.errstate(over="ignore"):
            inv = np.float32(np.float32(E4M3_MAX) / amax)
        if not np.isfinite(inv):
            inv = np.float32(_FLT_MAX)
    prod = (x32 * inv).astype(np.float32)
    return e4m3_encode(prod.astype(np.float64)), scale


# --------------------------------------------------------------------------
# Cache
# --------------------------------------------------------------------------

def blocks_per_slot(tokens_per_frame: int) -> int:
    """Blocks of 128 tokens (the last one possibly shorter) that cover one slot."""
    return -(-tokens_per_frame // BLOCK_TOKENS)


class OracleFp8Cache:
    """The bf16 oracle cache (ring state, sinks, rotated keys) plus its E4M3 copy."""

    def __init__(self, cfg: CacheConfig):
        if cfg.head_dim != 128:
            raise ValueError("the fp8 cache is defined for head_dim 128")
        self.cfg = cfg
        self.base = OracleCache(cfg)
        c = cfg
        self.n_blk = blocks_per_slot(c.tokens_per_frame)
        shape = (c.layers, c.batch, c.slots, c.tokens_per_frame, c.heads, c.head_dim)
        self.k8 = np.zeros(shape, np.uint8)
        self.v8 = np.zeros(shape, np.uint8)
        self.k_scale = np.zeros((c.layers, c.batch, c.slots, c.heads, self.n_blk), np.float32)
        self.v_scale = np.zeros((c.layers, c.batch, c.slots, c.heads, self.n_blk), np.float32)

    def quantize_slot(self, layer: int, b: int, s: int) -> None:
        """Re-derive slot s's E4M3 codes and scales from the bf16 values it holds."""
        c = self.cfg
        N = c.tokens_per_frame
        k = bf16_decode(self.base.k[layer, b, s])             # [N][H][d]
        v = bf16_decode(self.base.v[layer, b, s])
        for blk in range(self.n_blk):
            t0, t1 = blk * BLOCK_TOKENS, min(N, (blk + 1) * BLOCK_TOKENS)
            for h in range(c.heads):
                kc, ks = quantize_block(k[t0:t1, h])
                vc, vs = quantize_block(v[t0:t1, h])
                self.k8[layer, b, s, t0:t1, h] = kc
                self.v8[layer, b, s, t0:t1, h] = vc
                self.k_scale[layer, b, s, h, blk] = ks
                self.v_scale[layer, b, s, h, blk] = vs

    def dequantized(self, layer: int, b: int, n_slots: int):
        """K, V of the first n_slots slots, fp64 [n_slots * N][H][d]: token n of a slot
        takes the scale of its head and of block n // 128."""
        c = self.cfg
        N, H, d = c.tokens_per_frame, c.heads, c.head_dim
        blk = np.arange(N) // BLOCK_TOKENS
        ks = self.k_scale[layer, b, :n_slots][:, :, blk].astype(np.float64)   # [s][H][N]
        vs = self.v_scale[layer, b, :n_slots][:, :, blk].astype(np.float64)
        k = e4m3_decode(self.k8[layer, b, :n_slots]) * ks.transpose(0, 2, 1)[..., None]   # [s][N][H][d]
        v = e4m3_decode(self.v8[layer, b, :n_slots]) * vs.transpose(0, 2, 1)[..., None]
        return k.reshape(n_slots * N, H, d), v.reshape(n_slots * N, H, d)


def kv_append_fp8(cache: OracleFp8Cache, layer: int, k_bits: np.ndarray, v_bits: np.ndarray,
                  chunk_first_frame) -> None:
    """a2 in the fp8 format: the bf16 append, then the written slots quantised."""
    c = cache.cfg
    kv_append(cache.base, layer, k_bits, v_bits, chunk_first_frame)
    for b in range(c.batch):
        f0 = int(chunk_first_frame[b])
        if f0 < 0:
            continue
        for i in range(c.chunk_frames):
            cache.quantize_slot(layer, b, slot_of_frame(f0 + i, c.sink_frames, c.window_frames))


def chunk_attention_fp8(cache: OracleFp8Cache, layer: int, q_bits: np.ndarray, chunk_first_frame,
                        scale: float, rows=None) -> np.ndarray:
    """a3 over the dequantised fp8 cache: fp64 [B][Lq][H][d] (NaN for skipped streams)."""
    c = cache.cfg
    Lq = c.chunk_tokens
    out = np.full((c.batch, Lq, c.heads, c.head_dim), np.nan)
    for b in range(c.batch):
        f0 = int(chunk_first_frame[b])
        if f0 < 0:
            continue
        if cache.base.next_frame[b, layer] != f0 + c.chunk_frames:
            raise ValueError("attention must follow the append of the same chunk")
        s_valid, w_valid = valid_slot_counts(f0 + c.chunk_frames, c.sink_frames, c.window_frames)
        k, v = cache.dequantized(layer, b, s_valid + w_valid)
        qr = chunk_queries_rotated(c, q_bits[b], f0)
        sel = np.arange(Lq) if rows is None else np.asarray(rows)
        for h in range(c.heads):
            o, _ = attention_reference(qr[sel, h], k[:, h], v[:, h], scale)
            out[b, sel, h] = o
    return out


def sink_refresh_fp8(cache: OracleFp8Cache, hidden_bits: np.ndarray, tau: float, chunk_first_frame):
    """a4 in the fp8 format: the refreshed sink takes the last frame's codes and scales."""
    c = cache.cfg
    out = sink_refresh(cache.base, hidden_bits, tau, chunk_first_frame)
    for b in range(c.batch):
        j = int(out[b])
        if j < 0:
            continue
        f_last = int(chunk_first_frame[b]) + c.chunk_frames - 1
        s_last = slot_of_frame(f_last, c.sink_frames, c.window_frames)
        for arr in (cache.k8, cache.v8, cache.k_scale, cache.v_scale):
            arr[:, b, j] = arr[:, b, s_last]
    return out

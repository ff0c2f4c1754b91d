"""Plain fp64 CPU oracle for the streaming causal-DiT KV path (StreamDiffusionV2).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code
with the CUDA path (``causal_dit_kv_b200``) and imports nothing from it.

What it computes, step by step and in the pages' order:

  a1  frame -> ring slot and temporal RoPE phase (sink frames + rolling
      window, periodic phase reset),
  a2  append of a chunk's K (rotated by 3D RoPE) and V into the cache,
  a3  attention of the chunk's queries over the valid sink+window keys,
  a4  adaptive sink refresh by cosine similarity of the chunk embedding,
  a5  motion estimate (frame-difference RMS) and EMA noise rate.

Sources (page title, section):
  * admirer.cn article on StreamDiffusionV2, "方法：算法與系統層面的聯合優化"
    item 1 (sink tokens + rolling KV cache) and item 2 (motion-aware noise).
  * qq8o.cn walkthrough "直播革命來了！StreamDiffusionV2…", sections
    "Adaptive sink and RoPE refresh" and "Motion-aware noise scheduler".
  * agentlens project page "chenfengxu714/StreamDiffusionV2", component
    table (KV cache = ring buffer with sliding-window attention) and the
    Python example (noise scale carried from chunk to chunk).

The formula bodies are blank on all pages.  Where a step is left open the
plainest reading is taken; each reading is stated at the function that
takes it.  Parity against "the authors' exact formulas" is therefore
UNPINNED; what is pinned is that this code computes the stated readings
(tests/test_oracle_*.py pin it against brute force, closed forms,
invariants and library special cases).

Precision: every floating-point step runs in fp64.  bf16 inputs are decoded
exactly; the only roundings back to bf16 are the ones the method's storage
format imposes (the cached, rotated K), done by round-to-nearest-even from
fp64 directly (no intermediate fp32).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------
# bf16 encoding (storage format of Q/K/V/O)
# --------------------------------------------------------------------------

_BF16_OVERFLOW = 2.0 ** 128  # smallest magnitude that no longer fits a finite bf16


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 to the nearest bf16 value, ties to even (IEEE RNE).

    bf16 keeps 8 significant bits and the fp32 exponent range.  For a finite
    x with 2**(e-1) <= |x| < 2**e the spacing of bf16 values is 2**(e-8); below
    the smallest normal (2**-126) the spacing is the subnormal quantum 2**-133.
    x / spacing is exact in fp64 (a power-of-two scale), ``np.rint`` rounds it
    half-to-even, and the product back is exact.  A result of 2**128 or more
    overflows to infinity.  Returns fp64 arrays holding bf16 values.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    finite = np.isfinite(x) & (x != 0.0)
    xf = x[finite]
    _, e = np.frexp(xf)                      # xf = m * 2**e, 0.5 <= |m| < 1
    q_exp = np.maximum(e.astype(np.int64) - 8, -133)
    q = np.ldexp(1.0, q_exp)
    r = np.rint(xf / q) * q
    r = np.where(np.abs(r) >= _BF16_OVERFLOW, np.copysign(np.inf, r), r)
    out[finite] = r
    return out


def bf16_encode(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), rounding with :func:`bf16_round`."""
    r = bf16_round(x)
    f32 = r.astype(np.float32)               # exact: every bf16 value is an fp32 value
    bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(r)
    if np.any(nan):
        bits = np.where(nan, np.uint16(0x7FC0), bits)
    return bits


# --------------------------------------------------------------------------
# a1: ring slots and RoPE phase
# --------------------------------------------------------------------------

def slot_of_frame(f: int, sink_frames: int, window_frames: int) -> int:
    """Ring slot that frame ``f`` is written to.

    Sink tokens + rolling KV cache (admirer.cn article, method item 1; the
    agentlens component table calls the cache a ring buffer for sliding-
    window attention): the first ``S`` frames stay in sink slots 0..S-1, every
    later frame overwrites the oldest window frame, window slot S + (f-S) mod W.
    """
    if f < 0:
        raise ValueError("negative frame index")
    if f < sink_frames:
        return f
    return sink_frames + (f - sink_frames) % window_frames


def rope_phase(f: int, reset_period: int) -> int:
    """Temporal RoPE phase of frame ``f``.

    qq8o.cn walkthrough, "Adaptive sink and RoPE refresh": the RoPE phase is
    reset once the frame index passes a threshold (formula blank on the page).
    Reading: phase = f mod T_reset, so frames f and f + T_reset get identical
    rotations; T_reset = 0 means no reset (phase = f).
    """
    if reset_period <= 0:
        return f
    return f % reset_period


def valid_slot_counts(frame_end: int, sink_frames: int, window_frames: int):
    """(valid sink slots, valid window slots) once frames 0..frame_end-1 exist.

    Sinks fill first; the window holds at most W frames.  Because window
    slots are used only after every sink slot is filled, the valid slots are
    always the prefix 0 .. sink_valid + window_valid - 1.
    """
    s_valid = min(frame_end, sink_frames)
    w_valid = min(max(frame_end - sink_frames, 0), window_frames)
    return s_valid, w_valid


def slot_frames(frame_end: int, sink_frames: int, window_frames: int) -> list[int]:
    """Frame held by each slot after frames 0..frame_end-1 (no refresh); -1 = empty."""
    slots = [-1] * (sink_frames + window_frames)
    for f in range(frame_end):
        slots[slot_of_frame(f, sink_frames, window_frames)] = f
    return slots


# --------------------------------------------------------------------------
# 3D RoPE (t, h, w)
# --------------------------------------------------------------------------

def rope_pair_split(head_dim: int) -> tuple[int, int, int]:
    """Rotation pairs per axis (t, h, w) for a head of ``head_dim`` dims.

    The pages name "RoPE" only.  With c = head_dim/2 pairs the split is
    (c - 2*floor(c/3), floor(c/3), floor(c/3)): (22, 21, 21) for 128 dims and
    (12, 10, 10) for 64 dims.
    """
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    c = head_dim // 2
    return (c - 2 * (c // 3), c // 3, c // 3)


def rope_axis_cos_sin(positions, n_pairs: int, base: float):
    """cos/sin tables [len(positions)][n_pairs] for one axis.

    Pair j of an axis with n pairs turns at frequency base**(-j/n) rad per
    position step; the angle is position * frequency.  Evaluated with the C
    library's pow/cos/sin through Python's math module, in fp64.
    """
    cos = np.empty((len(positions), n_pairs), dtype=np.float64)
    sin = np.empty_like(cos)
    for i, p in enumerate(positions):
        for j in range(n_pairs):
            omega = base ** (-j / n_pairs)
            ang = float(p) * omega
            cos[i, j] = math.cos(ang)
            sin[i, j] = math.sin(ang)
    return cos, sin


def rope_token_cos_sin(phases, frame_h: int, frame_w: int, pairs, base: float):
    """Per-token cos/sin [len(phases)*frame_h*frame_w][head_dim/2].

    Token n of a frame sits at (row, col) = (n // frame_w, n % frame_w).  The
    pairs are ordered t first, then h, then w; pair j rotates dims (2j, 2j+1).
    """
    n_t, n_h, n_w = pairs
    ct, st = rope_axis_cos_sin(list(phases), n_t, base)
    ch, sh = rope_axis_cos_sin(range(frame_h), n_h, base)
    cw, sw = rope_axis_cos_sin(range(frame_w), n_w, base)
    n_tok = frame_h * frame_w
    tok = np.arange(len(phases) * n_tok)
    fi = tok // n_tok
    row = (tok % n_tok) // frame_w
    col = (tok % n_tok) % frame_w
    cos = np.concatenate([ct[fi], ch[row], cw[col]], axis=1)
    sin = np.concatenate([st[fi], sh[row], sw[col]], axis=1)
    return cos, sin


def rope_rotate(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate interleaved pairs of x[..., tok, (head,) d] in fp64.

    r0 = x0*c - x1*s and r1 = x0*s + x1*c, each product and sum a separate
    fp64 operation (numpy never fuses them).  ``cos``/``sin`` are
    [tok][d/2]; x is [tok][d] or [tok][H][d].
    """
    x = np.asarray(x, dtype=np.float64)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    if x.ndim == 3:   # [tok][H][d]
        c = cos[:, None, :]
        s = sin[:, None, :]
    else:
        c = cos
        s = sin
    out = np.empty_like(x)
    out[..., 0::2] = (x0 * c) - (x1 * s)
    out[..., 1::2] = (x0 * s) + (x1 * c)
    return out


# --------------------------------------------------------------------------
# Cache state (a1, a2, a4)
# --------------------------------------------------------------------------

@dataclass
class CacheConfig:
    batch: int
    layers: int
    heads: int
    head_dim: int
    frame_h: int
    frame_w: int
    chunk_frames: int
    sink_frames: int
    window_frames: int
    rope_pairs: tuple = None
    rope_reset_period: int = 0
    embed_dim: int = 0
    rope_base: float = 10000.0

    def __post_init__(self):
        if self.rope_pairs is None:
            self.rope_pairs = rope_pair_split(self.head_dim)
        self.rope_pairs = tuple(int(p) for p in self.rope_pairs)

    @property
    def tokens_per_frame(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def slots(self) -> int:
        return self.sink_frames + self.window_frames

    @property
    def chunk_tokens(self) -> int:
        return self.chunk_frames * self.tokens_per_frame


@dataclass
class OracleCache:
    """K/V cache as bf16 bit patterns, [L][B][S+W][N][H][d], plus sink state."""
    cfg: CacheConfig
    k: np.ndarray = field(init=False)
    v: np.ndarray = field(init=False)
    next_frame: np.ndarray = field(init=False)      # [B][L] next frame expected per layer
    sink_embed: np.ndarray = field(init=False)      # [B][S][D] fp64 sink-set embeddings
    sink_embed_set: np.ndarray = field(init=False)  # [B][S] bool
    sink_frame: np.ndarray = field(init=False)      # [B][S] frame whose KV the sink holds

    def __post_init__(self):
        c = self.cfg
        shape = (c.layers, c.batch, c.slots, c.tokens_per_frame, c.heads, c.head_dim)
        self.k = np.zeros(shape, dtype=np.uint16)
        self.v = np.zeros(shape, dtype=np.uint16)
        self.next_frame = np.zeros((c.batch, c.layers), dtype=np.int64)
        self.sink_embed = np.zeros((c.batch, c.sink_frames, max(c.embed_dim, 1)), dtype=np.float64)
        self.sink_embed_set = np.zeros((c.batch, c.sink_frames), dtype=bool)
        self.sink_frame = np.full((c.batch, c.sink_frames), -1, dtype=np.int64)


def kv_append(cache: OracleCache, layer: int, k_bits: np.ndarray, v_bits: np.ndarray,
              chunk_first_frame) -> None:
    """a2: write the chunk's K (3D-RoPE rotated) and V into their ring slots.

    k_bits, v_bits: bf16 bits [B][T'*N][H][d].  Stream b's chunk holds frames
    chunk_first_frame[b] .. +T'-1; a negative entry skips the stream.  Frame
    f goes to slot_of_frame(f) (evicting what the slot held) and its keys are
    rotated at (phase(f), row, col), rounded to bf16 once.  V is stored as is.
    """
    c = cache.cfg
    N, Tp = c.tokens_per_frame, c.chunk_frames
    for b in range(c.batch):
        f0 = int(chunk_first_frame[b])
        if f0 < 0:
            continue
        if f0 != cache.next_frame[b, layer]:
            raise ValueError(f"stream {b} layer {layer}: expected frame {cache.next_frame[b, layer]}, got {f0}")
        for i in range(Tp):
            f = f0 + i
            s = slot_of_frame(f, c.sink_frames, c.window_frames)
            cos, sin = rope_token_cos_sin([rope_phase(f, c.rope_reset_period)],
                                          c.frame_h, c.frame_w, c.rope_pairs, c.rope_base)
            kx = bf16_decode(k_bits[b, i * N:(i + 1) * N])          # [N][H][d]
            cache.k[layer, b, s] = bf16_encode(rope_rotate(kx, cos, sin))
            cache.v[layer, b, s] = v_bits[b, i * N:(i + 1) * N]
            if s < c.sink_frames:
                cache.sink_frame[b, s] = f
        cache.next_frame[b, layer] = f0 + Tp


# --------------------------------------------------------------------------
# a3: chunk attention over sink + window keys
# --------------------------------------------------------------------------

def attention_reference(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """softmax(scale * q k^T) v for one head, fp64.  q [Lq][d], k/v [Lk][d].

    Returns (out [Lq][d], probabilities [Lq][Lk]).  The maximum is subtracted
    before exponentiating (exact in real arithmetic, keeps exp finite).
    """
    s = scale * (q @ k.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v, p


def chunk_queries_rotated(cfg: CacheConfig, q_bits_b: np.ndarray, first_frame: int) -> np.ndarray:
    """RoPE(q) in fp64 for one stream's chunk, [T'*N][H][d] (not rounded)."""
    phases = [rope_phase(first_frame + i, cfg.rope_reset_period) for i in range(cfg.chunk_frames)]
    cos, sin = rope_token_cos_sin(phases, cfg.frame_h, cfg.frame_w, cfg.rope_pairs, cfg.rope_base)
    return rope_rotate(bf16_decode(q_bits_b), cos, sin)


def valid_keys(cache: OracleCache, layer: int, b: int):
    """Valid cached K, V of stream b (fp64, [Lk][H][d]) after its last append."""
    c = cache.cfg
    s_valid, w_valid = valid_slot_counts(int(cache.next_frame[b, layer]), c.sink_frames, c.window_frames)
    n_slots = s_valid + w_valid
    k = bf16_decode(cache.k[layer, b, :n_slots]).reshape(n_slots * c.tokens_per_frame, c.heads, c.head_dim)
    v = bf16_decode(cache.v[layer, b, :n_slots]).reshape(n_slots * c.tokens_per_frame, c.heads, c.head_dim)
    return k, v


def chunk_attention(cache: OracleCache, layer: int, q_bits: np.ndarray, chunk_first_frame,
                    scale: float, rows=None) -> np.ndarray:
    """a3: O = softmax(scale * RoPE(q) K^T) V over the stream's valid slots.

    Block-causal at chunk granularity: every query of the chunk sees every
    valid cached key, its own chunk's included (the chunk was appended
    first).  Returns fp64 [B][Lq][H][d]; streams with a negative first frame
    are left as NaN.  ``rows`` (optional) restricts the computation to those
    query indices, for sampled checks at full size.
    """
    c = cache.cfg
    Lq = c.chunk_tokens
    out = np.full((c.batch, Lq, c.heads, c.head_dim), np.nan)
    for b in range(c.batch):
        f0 = int(chunk_first_frame[b])
        if f0 < 0:
            continue
        if cache.next_frame[b, layer] != f0 + c.chunk_frames:
            raise ValueError("attention must follow the append of the same chunk")
        qr = chunk_queries_rotated(c, q_bits[b], f0)
        k, v = valid_keys(cache, layer, b)
        sel = np.arange(Lq) if rows is None else np.asarray(rows)
        for h in range(c.heads):
            o, _ = attention_reference(qr[sel, h], k[:, h], v[:, h], scale)
            out[b, sel, h] = o
    return out


# --------------------------------------------------------------------------
# a4: adaptive sink refresh
# --------------------------------------------------------------------------

def cosine(a: np.ndarray, b: np.ndarray) -> float:
    """Cosine similarity in fp64; 1.0 when either vector has zero norm."""
    na = math.sqrt(float(np.dot(a, a)))
    nb = math.sqrt(float(np.dot(b, b)))
    if na == 0.0 or nb == 0.0:
        return 1.0
    return float(np.dot(a, b)) / (na * nb)


def sink_refresh(cache: OracleCache, hidden_bits: np.ndarray, tau: float, chunk_first_frame):
    """a4: refresh the least-similar sink when the chunk embedding drifts.

    qq8o.cn walkthrough, "Adaptive sink and RoPE refresh": the new chunk
    embedding is compared with the sink set by cosine similarity and the
    least-similar sink is replaced when the similarity is below the
    threshold tau (formulas blank on the page).  Readings:
      * chunk embedding h = mean over the chunk's tokens of hidden [Lq][D];
      * c_j = cos(h, e_j) over sinks j; j* = argmin c_j, lowest j on ties;
      * if c_{j*} < tau, sink slot j* takes the chunk's LAST frame K/V in
        every layer (already rotated at append) and e_{j*} = h;
      * a chunk that itself fills sink slots (stream start) only records
        e_j = h for those slots and refreshes nothing.
    Returns int array [B]: refreshed slot, or -1.
    """
    c = cache.cfg
    Lq = c.chunk_tokens
    out = np.full(c.batch, -1, dtype=np.int64)
    for b in range(c.batch):
        f0 = int(chunk_first_frame[b])
        if f0 < 0:
            continue
        for layer in range(c.layers):
            if cache.next_frame[b, layer] != f0 + c.chunk_frames:
                raise ValueError("refresh must follow the append of the chunk in every layer")
        h = bf16_decode(hidden_bits[b]).sum(axis=0) / Lq
        fills = [f for f in range(f0, f0 + c.chunk_frames) if f < c.sink_frames]
        if fills:
            for f in fills:
                cache.sink_embed[b, f] = h
                cache.sink_embed_set[b, f] = True
            continue
        sims = [cosine(h, cache.sink_embed[b, j]) for j in range(c.sink_frames)]
        j_star = int(np.argmin(sims))          # first index of the minimum
        if sims[j_star] < tau:
            f_last = f0 + c.chunk_frames - 1
            s_last = slot_of_frame(f_last, c.sink_frames, c.window_frames)
            cache.k[:, b, j_star] = cache.k[:, b, s_last]
            cache.v[:, b, j_star] = cache.v[:, b, s_last]
            cache.sink_embed[b, j_star] = h
            cache.sink_frame[b, j_star] = f_last
            out[b] = j_star
    return out


# --------------------------------------------------------------------------
# a5: motion estimate and EMA noise rate
# --------------------------------------------------------------------------

@dataclass
class MotionConfig:
    batch: int
    channels: int
    height: int
    width: int
    window: int = 4          # k: frames the motion estimate is stabilised over
    sigma: float = 2.0       # statistical scale the motion is normalised by
    lam: float = 0.9         # EMA weight of the new target
    s_min: float = 0.5
    s_max: float = 0.9
    s_init: float = 0.7


@dataclass
class MotionState:
    cfg: MotionConfig
    prev: np.ndarray = field(init=False)        # [B][C*H*W] last frame seen (fp32 values)
    has_prev: np.ndarray = field(init=False)    # [B] bool
    history: list = field(init=False)           # per stream: last k motion values
    rate: np.ndarray = field(init=False)        # [B] current noise rate

    def __post_init__(self):
        c = self.cfg
        self.prev = np.zeros((c.batch, c.channels * c.height * c.width), dtype=np.float64)
        self.has_prev = np.zeros(c.batch, dtype=bool)
        self.history = [[] for _ in range(c.batch)]
        self.rate = np.full(c.batch, c.s_init, dtype=np.float64)


def motion_noise_rate(state: MotionState, latents: np.ndarray):
    """a5: per-frame motion, window normalisation, clip and EMA update.

    admirer.cn article (method item 2) and qq8o.cn walkthrough, "Motion-aware
    noise scheduler": motion strength from the L2 distance of consecutive
    latent frames, normalised by a statistical scale over a short k-frame
    window and clipped to [0, 1]; the noise rate follows an EMA with
    0 < lambda < 1 between s_min and s_max, high motion -> lower noise
    (formulas blank on the page).  Readings:
      * d_t = ||x_t - x_{t-1}||_2 / sqrt(numel)  (an RMS),
      * dbar_t = max of the last k values d_{t-k+1..t},
      * dhat_t = clip(dbar_t / sigma, 0, 1),
      * target = s_max - (s_max - s_min) * dhat_t,
      * s_t = lam * target + (1 - lam) * s_{t-1}  (lam weights the new value),
      * the stream's first frame has no predecessor: no d, s unchanged.
    latents: [B][T'][C][H][W] (fp32 values).  Returns (rate [B], d [B][T'])
    with d = -1 where a frame had no predecessor.
    """
    c = state.cfg
    x = np.asarray(latents, dtype=np.float64).reshape(c.batch, -1, c.channels * c.height * c.width)
    Tp = x.shape[1]
    d_out = np.full((c.batch, Tp), -1.0)
    for b in range(c.batch):
        for t in range(Tp):
            cur = x[b, t]
            if state.has_prev[b]:
                diff = cur - state.prev[b]
                d = math.sqrt(float(np.dot(diff, diff)) / diff.size)
                d_out[b, t] = d
                state.history[b].append(d)
                if len(state.history[b]) > c.window:
                    state.history[b].pop(0)
                dbar = max(state.history[b])
                dhat = min(max(dbar / c.sigma, 0.0), 1.0)
                target = c.s_max - (c.s_max - c.s_min) * dhat
                state.rate[b] = c.lam * target + (1.0 - c.lam) * state.rate[b]
            state.prev[b] = cur
            state.has_prev[b] = True
    return state.rate.copy(), d_out

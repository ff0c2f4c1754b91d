/*
 * sdv2.h — C ABI of libsdv2: the streaming causal-DiT KV path of
 * StreamDiffusionV2 on NVIDIA B200 (sm_100a).
 *
 * The path, one latent chunk of T' frames per stream per step:
 *   for every DiT layer l:  sdv2_kv_append(l)  then  sdv2_chunk_attention(l)
 *                           (or both at once: sdv2_append_attention(l))
 *   once per step:          sdv2_sink_refresh, sdv2_motion_noise_rate
 *
 * Sources (page title, section):
 *   [A] admirer.cn article on StreamDiffusionV2 (MLSys 2026), sections
 *       "深入分析：內存帶寬約束導致的性能受限" (loading a long KV cache while
 *       computing only on the current input) and "方法：算法與系統層面的聯合優化"
 *       items 1 (sink tokens + rolling KV cache) and 2 (motion-aware noise).
 *   [Q] qq8o.cn walkthrough "直播革命來了！StreamDiffusionV2…", sections
 *       "Adaptive sink and RoPE refresh" and "Motion-aware noise scheduler".
 *   [G] agentlens project page "chenfengxu714/StreamDiffusionV2", component
 *       table (KV cache: ring buffer for sliding-window attention) and the
 *       single-GPU Python example (noise scale carried chunk to chunk).
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and owns every device buffer and every
 *     stream.  The library allocates only the small host-side handle.  Device
 *     buffers must outlive the handle that refers to them.
 *   - Asynchrony: compute calls enqueue work on the given stream and return
 *     without synchronising; decisions (e.g. which sink is refreshed) stay on
 *     the device.  A NULL stream means the legacy default stream.
 *   - Alignment: every device pointer must be 16-byte aligned (SDV2_E_ALIGN).
 *   - Errors: every call returns an sdv2_status; sdv2_last_error() gives a
 *     thread-local message for the last failure.  Kernels never trap: a wait
 *     that runs past its bound sets a device status word and the kernel
 *     returns; sdv2_cache_check()/sdv2_motion_check() read that word.
 *   - bf16 is IEEE bfloat16 (1 sign, 8 exponent, 7 fraction bits), passed as
 *     raw 16-bit words; fp32/fp64 are IEEE binary32/binary64.
 *   - No call allocates device memory.
 */
#ifndef SDV2_H
#define SDV2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

/* A CUDA stream (same type as cudaStream_t / CUstream). */
typedef struct CUstream_st *sdv2_stream;
/* A CUDA event (same type as cudaEvent_t / CUevent). */
typedef struct CUevent_st *sdv2_event;

typedef enum {
    SDV2_OK = 0,
    SDV2_E_ARG = -1,    /* null pointer or scalar out of range */
    SDV2_E_SHAPE = -2,  /* inconsistent config, or a size beyond the supported limits */
    SDV2_E_ALIGN = -3,  /* pointer not 16-byte aligned, or buffer smaller than required */
    SDV2_E_STATE = -4,  /* call out of order: frame index is not the expected one */
    SDV2_E_CUDA = -5,   /* a CUDA runtime call failed (message in sdv2_last_error) */
    SDV2_E_DEVICE = -6  /* a kernel reported an error through the device status word */
} sdv2_status;

/* ------------------------------------------------------------------------
 * KV cache: sink frames + rolling window, per layer, per stream.
 * ---------------------------------------------------------------------- */

typedef struct {
    int32_t batch;          /* B: independent streams, each with its own cache */
    int32_t layers;         /* L: DiT layers; each has its own K/V cache */
    int32_t heads;          /* H */
    int32_t head_dim;       /* d: 64 or 128 */
    int32_t frame_h;        /* latent token grid of one frame: N = frame_h * frame_w */
    int32_t frame_w;
    int32_t chunk_frames;   /* T': frames per chunk (per call) */
    int32_t sink_frames;    /* S: frames kept as sink tokens */
    int32_t window_frames;  /* W: rolling-window frames (W >= T') */
    int32_t rope_pairs[3];  /* rotation pairs on the (t, h, w) axes; sum = head_dim / 2 */
    int32_t rope_reset_period; /* T_reset: temporal phase = frame mod T_reset; 0 = never reset */
    int32_t embed_dim;      /* D: width of the hidden states used for sink refresh (0 = no refresh) */
    double rope_base;       /* RoPE base (10000 when <= 0) */
    int32_t kv_format;      /* SDV2_KV_BF16 (0) or SDV2_KV_FP8_E4M3 (1) */
} sdv2_cache_config;

/* Storage format of the cached K and V.
 * SDV2_KV_BF16: the rotated keys and the values as bf16.
 * SDV2_KV_FP8_E4M3: the same values quantised to FP8 E4M3 in blocks, a
 *   reading of the FP8 item on the roadmap of [G] (the page names the format
 *   only).  A slot's N tokens are padded to Np = ceil(N/128)*128 and cut into
 *   blocks of 128 tokens; each (layer, stream, slot, head, block) has one fp32
 *   scale for K and one for V: scale = amax/448 over the block's tokens and the
 *   head's d channels, code = E4M3(x * (448/amax)) with round-to-nearest-even
 *   and saturation (codes 0 for amax = 0); the dequantised value is
 *   code * scale.  K codes are token-major [B][S+W][Np][H][d]; V codes are
 *   transposed per slot, [B][S+W][H][d][Np], so both tensor-core operands are
 *   K-major; padding tokens hold code 0.  The attention rounds each rotated
 *   query row to E4M3 with its own scale and the probabilities to E4M3 before
 *   the products (fp32 accumulation).  With N = 64 (one half-full block per
 *   slot) the attention reads no padding: it takes two slots per 128-key tile,
 *   each half with its own scales.  Requires head_dim 128. */
enum { SDV2_KV_BF16 = 0, SDV2_KV_FP8_E4M3 = 1 };

typedef struct sdv2_cache sdv2_cache;

/* Byte offsets inside the caller's cache buffer (all 256-byte aligned). */
typedef struct {
    uint64_t k_offset;        /* K cache, bf16 [L][B][S+W][N][H][d] (rotated keys) */
    uint64_t v_offset;        /* V cache, bf16 [L][B][S+W][N][H][d] */
    uint64_t layer_stride;    /* bytes between consecutive layers of K (and of V) */
    uint64_t sink_embed_offset; /* fp64 [B][S][D]: sink-set embeddings e_j */
    uint64_t sink_frame_offset; /* int64 [B][S]: frame whose K/V each sink slot holds (-1 empty) */
    uint64_t status_offset;   /* uint32: device status word (0 = ok) */
    uint64_t scratch_offset;  /* attention split-KV partials and refresh reductions */
    uint64_t scratch_bytes;
    uint64_t total_bytes;     /* == sdv2_cache_bytes(cfg) */
    /* fp8 cache only (zero for bf16): k_offset / v_offset then hold the E4M3 codes,
     * K [L][B][S+W][Np][H][d] and V [L][B][S+W][H][d][Np], layer_stride bytes apart. */
    uint64_t k_scale_offset;  /* fp32 [L][B][S+W][scale_slot_stride]: head h, block j at h*(Np/128)+j */
    uint64_t v_scale_offset;
    uint64_t scale_layer_stride; /* bytes between layers of the scales */
    uint32_t scale_slot_stride;  /* floats per slot (H*Np/128 rounded up to a multiple of 4) */
    uint32_t tokens_padded;      /* Np */
} sdv2_cache_layout;

/* Device bytes the caller must allocate for a cache with this config;
 * 0 if the config is invalid (see sdv2_last_error). */
size_t sdv2_cache_bytes(const sdv2_cache_config *cfg);

/* Fill *out with the region offsets of a cache buffer for cfg. */
sdv2_status sdv2_cache_layout_of(const sdv2_cache_config *cfg, sdv2_cache_layout *out);

/* Bind a cache handle to the caller's device buffer dev_buf of `bytes`
 * bytes (>= sdv2_cache_bytes) on the current device.  Zero-fills the buffer
 * and uploads the RoPE row/column tables, synchronously (not on the hot
 * path).  Every stream starts empty at frame 0.
 * Limits: head_dim in {64, 128}; batch <= 64; N, H, L, S, W, T' >= 1,
 * W >= T'; sink refresh requires embed_dim >= 1; rope_pairs[0] (temporal
 * pairs) x min(T', floor(255 / N) + 2) <= 128 (the temporal angles of the
 * chunk frames that 256 consecutive queries span are kept on chip).
 * Errors: SDV2_E_ARG, SDV2_E_SHAPE, SDV2_E_ALIGN (buffer unaligned or too
 * small), SDV2_E_CUDA. */
sdv2_status sdv2_cache_create(const sdv2_cache_config *cfg, void *dev_buf, size_t bytes,
                              sdv2_cache **out);

/* Release the host handle.  The device buffer is the caller's to free. */
sdv2_status sdv2_cache_destroy(sdv2_cache *cache);

/* Append one chunk of keys and values for layer `layer`.
 * [A] method item 1, [G] component table, [Q] "Adaptive sink and RoPE refresh".
 * k, v: device bf16 [B][T'*N][H][d] (token t of the chunk is frame t / N,
 *       grid position (row, col) = ((t % N) / frame_w, (t % N) % frame_w)).
 * chunk_first_frame: HOST int64 [B]; stream b's chunk holds frames
 *       f0..f0+T'-1, and f0 must equal the number of frames already appended
 *       to that stream's layer (0 for a new stream).  A negative entry skips
 *       stream b for this call.
 * Frame f is written to slot f (f < S) or S + (f - S) mod W, evicting the
 * frame that slot held.  K is rotated by 3D RoPE at (phase(f), row, col) with
 * phase(f) = f mod T_reset, pairs interleaved (dims 2j, 2j+1), t pairs
 * first, then h, then w; frequency of pair j on an axis with n pairs is
 * base^(-j/n).  Each rotation is r0 = x0*c - x1*s, r1 = x0*s + x1*c in fp64
 * without fused multiply-add, rounded once to bf16 (nearest, ties to even).
 * V is copied unchanged.  With SDV2_KV_FP8_E4M3 the same rotated keys and
 * the values are then quantised per 128-token block and head (see
 * sdv2_cache_config.kv_format) and only the codes and scales are stored.
 * Errors: SDV2_E_ARG, SDV2_E_ALIGN, SDV2_E_STATE (wrong f0), SDV2_E_CUDA. */
sdv2_status sdv2_kv_append(sdv2_cache *cache, int32_t layer, const void *k, const void *v,
                           const int64_t *chunk_first_frame, sdv2_stream stream);

/* Attention of the chunk's queries over the valid sink + window keys of
 * layer `layer`: out = softmax(softmax_scale * RoPE(q) K^T) V.
 * [A] "深入分析" (KV-cache load per chunk), [Q] "Adaptive sink and RoPE refresh".
 * q:   device bf16 [B][T'*N][H][d], NOT rotated.  RoPE is applied on load:
 *      the attention kernel reads the raw tiles and rotates each row in fp32
 *      at the same (phase, row, col) as the chunk's keys, rounded to bf16 in
 *      shared memory for the tensor cores (q itself is never written).  With
 *      the fp8 cache each rotated row is coded as E4M3 with its own scale
 *      instead, the products run on E4M3 operands and the probabilities are
 *      coded as E4M3 too.  q must stay unchanged until the call's kernels
 *      have run (stream order).
 * out: device bf16 [B][T'*N][H][d].
 * chunk_first_frame: HOST int64 [B], the frames of this chunk; the chunk must
 *      already be appended to this layer (f0 + T' == frames appended).
 *      Negative entries skip the stream (its out rows are left untouched).
 * Every query sees every valid cached key of its stream, its own chunk
 * included (block-causal at chunk granularity): the valid slots are
 * 0 .. min(f_end,S) + min(max(f_end-S,0),W) - 1 with f_end = f0 + T'.
 * Accumulation is fp32; softmax_scale > 0 (1/sqrt(d) typically).
 * May use the cache buffer's scratch region (split-KV partials).
 * Errors: SDV2_E_ARG, SDV2_E_ALIGN, SDV2_E_STATE, SDV2_E_CUDA. */
sdv2_status sdv2_chunk_attention(sdv2_cache *cache, int32_t layer, const void *q, void *out,
                                 const int64_t *chunk_first_frame, float softmax_scale,
                                 sdv2_stream stream);

/* The KV append fused into the chunk attention: the same results as
 * sdv2_kv_append(layer, k, v) followed by sdv2_chunk_attention(layer, q, out)
 * (the cache bit for bit; out within the attention's fp32 accumulation, the
 * keys being taken in another order), in one launch where it applies.
 * [A] "深入分析" (each chunk loads the long KV cache but computes only on
 * the current input: the chunk's own K/V should not make a second trip),
 * [Q] "Adaptive sink and RoPE refresh".
 * q, k, v: device bf16 [B][T'*N][H][d] as for the two calls; out as for
 *      sdv2_chunk_attention.  chunk_first_frame as for sdv2_kv_append (the
 *      chunk is NOT yet appended); the call appends it.
 * Fused (bf16 cache, T'*N <= 256, T' <= 4, T' * temporal pairs <= 48, the
 * chunk's temporal phases below 4096 (the cache keeps their fp64 (cos, sin)),
 * 16 * (frame_h * row pairs + frame_w * column pairs) <= 256 * head_dim - 1024,
 * and the chunk's
 * rows of every stream within at most two 128-key tiles of its valid slot
 * prefix; see sdv2_append_attention_mode): the attention CTA that reads a KV
 * tile holding the chunk's rows builds those rows in shared memory from k and v
 * (keys rotated exactly as sdv2_kv_append rotates them), writes them to their
 * ring slots and feeds the same values to the tensor cores; the rest of the
 * cache comes by TMA as usual.  The chunk's K/V are read from k / v once
 * and never read back from the cache.  Otherwise the call makes the two calls.
 * Unlike sdv2_chunk_attention, the fused launch waits for the previous kernel
 * in the stream before reading q (q, k, v may come from it).
 * Errors: SDV2_E_ARG, SDV2_E_ALIGN, SDV2_E_STATE (wrong f0), SDV2_E_CUDA. */
sdv2_status sdv2_append_attention(sdv2_cache *cache, int32_t layer, const void *q, const void *k,
                                  const void *v, void *out, const int64_t *chunk_first_frame,
                                  float softmax_scale, sdv2_stream stream);

/* Adaptive sink refresh, after the chunk was appended to every layer.
 * [Q] "Adaptive sink and RoPE refresh".
 * hidden: device bf16 [B][T'*N][D] (D = embed_dim); the chunk embedding is
 *      its mean over tokens, in fp64.
 * tau: similarity threshold.
 * out_slot_dev: device int32 [B]: the refreshed sink slot, or -1.
 * For a chunk that fills sink slots itself (frames < S) the call records the
 * embedding of those slots and refreshes nothing.  Otherwise c_j =
 * cos(h, e_j) in fp64 (1 when a norm is zero), j* = argmin c_j with the
 * lowest j on ties, and if c_j* < tau the chunk's LAST frame K/V (every
 * layer, already rotated) is copied into sink slot j* and e_j* = h.  The
 * decision is taken on the device; no host synchronisation.
 * Errors: SDV2_E_ARG, SDV2_E_SHAPE (embed_dim 0), SDV2_E_ALIGN,
 * SDV2_E_STATE, SDV2_E_CUDA. */
sdv2_status sdv2_sink_refresh(sdv2_cache *cache, const void *hidden, float tau,
                              const int64_t *chunk_first_frame, int32_t *out_slot_dev,
                              sdv2_stream stream);

/* Host view of stream b, layer `layer`: slot_frame[S+W] = frame held by each
 * slot without refreshes (-1 empty), slot_phase[S+W] = its temporal RoPE
 * phase (-1 empty), *valid_slots = length of the valid slot prefix.  A sink
 * refreshed on the device is recorded in the sink_frame region instead.
 * Pure host call. */
sdv2_status sdv2_cache_query(const sdv2_cache *cache, int32_t b, int32_t layer,
                             int64_t *slot_frame, int32_t *slot_phase, int32_t *valid_slots);

/* Region offsets of this cache's buffer (see sdv2_cache_layout). */
sdv2_status sdv2_cache_layout_get(const sdv2_cache *cache, sdv2_cache_layout *out);

/* Synchronise the device and read the cache's status word: SDV2_OK, or
 * SDV2_E_DEVICE if a kernel gave up on a bounded wait (the word is then
 * cleared).  Not for the hot path. */
sdv2_status sdv2_cache_check(sdv2_cache *cache);

/* Failure-detection self-test (no counterpart in the pages): launches one
 * thread that waits on a device barrier nothing arrives on, bounded by
 * limit_ns (1 .. 2e9).  The wait gives up, sets a bit in the cache's status
 * word and the kernel returns normally, so the next sdv2_cache_check()
 * reports SDV2_E_DEVICE and clears the word; the CUDA context stays usable.
 * This is the path every real kernel wait takes when it runs out.
 * Errors: SDV2_E_ARG, SDV2_E_CUDA. */
sdv2_status sdv2_cache_selftest_wait(sdv2_cache *cache, uint64_t limit_ns, sdv2_stream stream);

/* Measurement hook (no counterpart in the pages): while set, every
 * sdv2_chunk_attention call (and fused sdv2_append_attention call) on this
 * cache records `start` on its stream right before the attention kernel's
 * launch and `stop` right after it, so
 * the time between them is that kernel alone (the split merge after it is
 * outside).  Recording events between the
 * call's launches serialises them; use it in a separate timing pass.  Pass
 * NULL for both to switch it off.  The events are the caller's.
 * Errors: SDV2_E_ARG (only one of the two given). */
sdv2_status sdv2_cache_time_attention(sdv2_cache *cache, sdv2_event start, sdv2_event stop);

/* ------------------------------------------------------------------------
 * Motion-aware noise rate.  [A] method item 2; [Q] "Motion-aware noise
 * scheduler"; [G] Python example (previous_noise_scale carried over).
 * ---------------------------------------------------------------------- */

typedef struct {
    int32_t batch;        /* B streams */
    int32_t chunk_frames; /* T' latent frames per call */
    int32_t channels;     /* latent frame shape C x H x W */
    int32_t height;
    int32_t width;
    int32_t window;       /* k: motion values the estimate is stabilised over (max) */
    double sigma;         /* statistical scale: dhat = clip(dbar / sigma, 0, 1) */
    double lambda;        /* EMA weight of the new target, 0 < lambda <= 1 */
    double s_min;         /* noise-rate bounds: target = s_max - (s_max - s_min) * dhat */
    double s_max;
    double s_init;        /* noise rate before the first motion value */
} sdv2_motion_config;

typedef struct sdv2_motion sdv2_motion;

/* Device bytes for the motion state of this config (0 if invalid). */
size_t sdv2_motion_bytes(const sdv2_motion_config *cfg);

/* Bind a motion handle to the caller's device buffer; initialises the state
 * (rate = s_init, no previous frame), synchronously.  Limits: batch <= 64,
 * chunk_frames <= 64, window in 1..64, sigma > 0, 0 < lambda <= 1.
 * Errors: SDV2_E_ARG, SDV2_E_SHAPE, SDV2_E_ALIGN, SDV2_E_CUDA. */
sdv2_status sdv2_motion_create(const sdv2_motion_config *cfg, void *dev_buf, size_t bytes,
                               sdv2_motion **out);
sdv2_status sdv2_motion_destroy(sdv2_motion *motion);

/* Per frame t of the chunk (in order), per stream:
 *   d_t   = ||x_t - x_{t-1}||_2 / sqrt(C*H*W)   (x_{t-1}: previous frame, from the
 *           previous call for t = 0; none for a stream's very first frame),
 *   dbar  = max of the last `window` d values, dhat = clip(dbar / sigma, 0, 1),
 *   s_t   = lambda * (s_max - (s_max - s_min) * dhat) + (1 - lambda) * s_{t-1}.
 * Sums and the recurrence run in fp64.
 * latents:      device fp32 [B][T'][C][H][W].
 * out_rate_dev: device fp32 [B], the noise rate after the chunk.
 * out_d_dev:    device fp32 [B][T'] (may be NULL): d_t, or -1 for a frame
 *               with no predecessor.
 * Errors: SDV2_E_ARG, SDV2_E_ALIGN, SDV2_E_CUDA. */
sdv2_status sdv2_motion_noise_rate(sdv2_motion *motion, const float *latents, float *out_rate_dev,
                                   float *out_d_dev, sdv2_stream stream);

/* Allocation-free variant of sdv2_motion_noise_rate.  The pages have no
 * counterpart: this is a deployment convenience of this library.
 * Same arguments, state and results as sdv2_motion_noise_rate, but the
 * per-call scratch (one fp64 partial sum per 2048-element block of each
 * frame, one ticket counter per stream) lives in a fixed 128 KB device array
 * that the library holds on every GPU that loads it, until the process exits.
 * For callers that cannot call cudaMalloc where they run the step: a host
 * framework that owns all device memory and hands out only fixed buffers, or
 * a real-time loop that must not allocate.  The array's device address is
 * looked up the first time the call runs on a device, so make that first
 * call before any stream capture.  Every call shares the one array: calls
 * whose work overlaps on the GPU (other streams, other threads) race and must
 * be serialised by the caller.  Limit: batch * chunk_frames *
 * ceil(C*H*W / 2048) <= 16384, else SDV2_E_SHAPE.  Allocates nothing.
 * Errors: SDV2_E_ARG, SDV2_E_SHAPE, SDV2_E_ALIGN, SDV2_E_CUDA. */
sdv2_status sdv2_motion_noise_rate_noalloc(sdv2_motion *motion, const float *latents, float *out_rate_dev,
                                           float *out_d_dev, sdv2_stream stream);

/* Synchronise and read the motion status word (as sdv2_cache_check). */
sdv2_status sdv2_motion_check(sdv2_motion *motion);

/* ------------------------------------------------------------------------
 * Host-only helpers (no device needed) and diagnostics.
 * ---------------------------------------------------------------------- */

/* Ring slot of frame f (-1 if f < 0). */
int32_t sdv2_slot_of_frame(int64_t f, int32_t sink_frames, int32_t window_frames);
/* Temporal RoPE phase of frame f (f mod T_reset, or f when T_reset <= 0). */
int64_t sdv2_rope_phase(int64_t f, int32_t rope_reset_period);
/* Valid sink and window slot counts once frames 0..frame_end-1 exist. */
void sdv2_valid_slots(int64_t frame_end, int32_t sink_frames, int32_t window_frames,
                      int32_t *sink_valid, int32_t *window_valid);
/* Work plan sdv2_chunk_attention would use on a GPU with sm_count SMs for
 * streams whose valid key counts are keys[0..batch-1] (0: stream skipped),
 * for the first launch (up to 64 streams).  Units are (stream, head, pair of
 * 128-query tiles); units [0, *whole_units) run whole and the rest are split
 * over the KV range into *pieces CTAs each (*pieces == 1: nothing split).
 * Host-side, no device needed.  Errors: SDV2_E_ARG, SDV2_E_SHAPE. */
sdv2_status sdv2_attention_plan(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count,
                                int32_t *whole_units, int32_t *pieces);
/* *pieces of sdv2_attention_plan (1 if no unit is split), or -1 on a bad
 * argument. */
int32_t sdv2_attention_splits(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count);
/* 1 if sdv2_chunk_attention would run that launch in the pair mode, 0 if not, -1
 * on a bad argument.  Pair mode (either cache format, chunks of at most 128 queries, more
 * (stream, head) units than SMs): one CTA takes heads 2k and 2k+1 of a stream,
 * each on its own query tile and accumulator set, their KV tiles interleaved, so
 * half as many CTAs start and the two heads' softmax and tensor-core work overlap.
 * Host-side, no device needed. */
int32_t sdv2_attention_pair_mode(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count);
/* How sdv2_append_attention runs chunks starting at chunk_first_frame[0..batch-1]
 * (negative: stream skipped) on a GPU with sm_count SMs: 0 as two launches (the
 * append, then the attention), 1 as the fused kernel, 2 as the fused kernel in
 * the pair mode (one KV tile per stream holds the chunk's rows); -1 on a bad
 * argument.  Host-side, no device needed. */
int32_t sdv2_append_attention_mode(const sdv2_cache_config *cfg, const int64_t *chunk_first_frame,
                                   int32_t sm_count);

/* Kernels launched by this library in this process so far. */
uint64_t sdv2_launch_count(void);
/* Thread-local message describing the last failing call ("" if none). */
const char *sdv2_last_error(void);
/* Library version string. */
const char *sdv2_version(void);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif
#endif /* SDV2_H */

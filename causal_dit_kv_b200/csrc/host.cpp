// libsdv2 host layer: config validation, buffer layout, the ring/phase
// bookkeeping of every stream, RoPE tables, TMA descriptors and kernel
// launches on the caller's stream.  Implements include/sdv2.h.
//
// Ring and phase rules (admirer.cn article on StreamDiffusionV2, method item
// 1; agentlens page "chenfengxu714/StreamDiffusionV2", component table;
// qq8o.cn walkthrough, "Adaptive sink and RoPE refresh"): frame f < S goes to
// sink slot f, later frames to S + (f - S) mod W; the temporal RoPE phase is
// f mod T_reset; the valid slots after frames 0..f_end-1 are the prefix of
// length min(f_end, S) + min(max(f_end - S, 0), W).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <memory>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "sdv2.h"
#include "sdv2_internal.h"

using namespace sdv2;

namespace {

thread_local std::string g_err;
std::atomic<uint64_t> g_launches{0};

sdv2_status fail(sdv2_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

sdv2_status cuda_fail(cudaError_t e, const char *what) {
    return fail(SDV2_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t slot_of(int64_t f, int32_t S, int32_t W) {
    if (f < 0) return -1;
    if (f < S) return static_cast<int32_t>(f);
    return S + static_cast<int32_t>((f - S) % W);
}

int64_t phase_of(int64_t f, int32_t reset) { return reset > 0 ? f % reset : f; }

void valid_counts(int64_t f_end, int32_t S, int32_t W, int32_t *sv, int32_t *wv) {
    const int64_t s = f_end < S ? f_end : S;
    int64_t w = f_end - S;
    if (w < 0) w = 0;
    if (w > W) w = W;
    *sv = static_cast<int32_t>(s < 0 ? 0 : s);
    *wv = static_cast<int32_t>(w);
}

// Angle of pair j on an axis with n pairs at integer position pos.  Same
// expression as the definition: pos * base^(-j/n), in fp64 with the C library.
double rope_angle(double base, int j, int n, int64_t pos) {
    const double omega = std::pow(base, -static_cast<double>(j) / static_cast<double>(n));
    return static_cast<double>(pos) * omega;
}

struct Geometry {
    int64_t N, slots, lq, frame_elems, layer_elems;
    bool f8;                 // fp8 (E4M3) block-scaled cache
    int64_t np_tokens;       // fp8: tokens per slot padded to whole 128-token blocks
    int n_blk, scale_slot_stride;
    bool pack2;              // fp8 with 64-token slots: two slots per KV tile (no padding read)
    uint64_t k_scale, v_scale, scale_layer_stride;
    int n_qpairs, lq_pad;
    int refresh_chunks;  // token chunks of the refresh reduction
    int64_t part_rows;  // capacity of the split-KV partial buffer, rows of d floats
    // region offsets
    uint64_t rope_h64, rope_w64, rope_h32, rope_w32;
    uint64_t omega;          // [n_t] fp64 temporal frequencies (query rotation)
    uint64_t rope_t64;       // [n_phase][n_t] fp64 (cos, sin) of the temporal pairs (fused append, bf16 cache)
    int64_t n_phase;
    uint64_t sink_embed, sink_frame, status;
    uint64_t scratch, refresh_mean, refresh_counter, part_ml, part_o, scratch_end;
    uint64_t k, v, layer_stride, total;
};

constexpr int64_t kPartRowsCap = 98304;   // split-KV partial rows: 384 blocks of 256 (~50 MB at d = 128)

sdv2_status check_config(const sdv2_cache_config *c, sdv2_cache_config *norm) {
    if (!c) return fail(SDV2_E_ARG, "config is NULL");
    sdv2_cache_config n = *c;
    if (n.batch < 1 || n.batch > kMaxBatch) return fail(SDV2_E_SHAPE, "batch must be in 1..%d", kMaxBatch);
    if (n.layers < 1 || n.heads < 1) return fail(SDV2_E_SHAPE, "layers and heads must be >= 1");
    if (n.head_dim != 64 && n.head_dim != 128) return fail(SDV2_E_SHAPE, "head_dim must be 64 or 128");
    if (n.frame_h < 1 || n.frame_w < 1) return fail(SDV2_E_SHAPE, "frame_h and frame_w must be >= 1");
    if (n.chunk_frames < 1 || n.sink_frames < 1 || n.window_frames < 1)
        return fail(SDV2_E_SHAPE, "chunk_frames, sink_frames and window_frames must be >= 1");
    if (n.window_frames < n.chunk_frames) return fail(SDV2_E_SHAPE, "window_frames must be >= chunk_frames");
    if (n.rope_reset_period < 0) return fail(SDV2_E_SHAPE, "rope_reset_period must be >= 0");
    if (n.embed_dim < 0 || (n.embed_dim & 1) || n.embed_dim > 16384)
        return fail(SDV2_E_SHAPE, "embed_dim must be even and in 0..16384");
    if (!(n.rope_base > 0.0)) n.rope_base = 10000.0;
    if (n.kv_format != SDV2_KV_BF16 && n.kv_format != SDV2_KV_FP8_E4M3)
        return fail(SDV2_E_SHAPE, "kv_format must be SDV2_KV_BF16 or SDV2_KV_FP8_E4M3");
    if (n.kv_format == SDV2_KV_FP8_E4M3 && n.head_dim != 128)
        return fail(SDV2_E_SHAPE, "the fp8 cache requires head_dim 128");
    const int c2 = n.head_dim / 2;
    if (n.rope_pairs[0] == 0 && n.rope_pairs[1] == 0 && n.rope_pairs[2] == 0) {
        n.rope_pairs[1] = c2 / 3;
        n.rope_pairs[2] = c2 / 3;
        n.rope_pairs[0] = c2 - 2 * (c2 / 3);
    }
    if (n.rope_pairs[0] < 0 || n.rope_pairs[1] < 0 || n.rope_pairs[2] < 0 ||
        n.rope_pairs[0] + n.rope_pairs[1] + n.rope_pairs[2] != c2)
        return fail(SDV2_E_SHAPE, "rope_pairs must be >= 0 and sum to head_dim/2");
    if (n.rope_pairs[0] < 1 || n.rope_pairs[0] > 64)
        return fail(SDV2_E_SHAPE, "the temporal axis needs 1..64 rotation pairs");
    const int64_t N = static_cast<int64_t>(n.frame_h) * n.frame_w;
    {
        // the temporal (cos, sin) of the chunk frames that one attention CTA's 256 query rows
        // can span are kept in shared memory
        const int64_t frames = std::min<int64_t>(n.chunk_frames, 255 / N + 2);
        if (frames * n.rope_pairs[0] > kAttnTabEntries)
            return fail(SDV2_E_SHAPE, "temporal pairs x chunk frames spanned by 256 queries exceeds %d",
                        kAttnTabEntries);
    }
    const int64_t slots = n.sink_frames + n.window_frames;
    const int64_t fe = N * n.heads * n.head_dim;
    const int64_t np_tok = (N + 127) / 128 * 128;
    if (slots * np_tok >= (1ll << 31) || fe * kAppendMaxFrames * 2 / 8 >= (1ll << 31) ||
        N * n.chunk_frames >= (1ll << 30))
        return fail(SDV2_E_SHAPE, "cache dimensions exceed the supported 32-bit index range");
    *norm = n;
    return SDV2_OK;
}

Geometry geometry(const sdv2_cache_config &c) {
    Geometry g{};
    g.N = static_cast<int64_t>(c.frame_h) * c.frame_w;
    g.slots = c.sink_frames + c.window_frames;
    g.lq = g.N * c.chunk_frames;
    g.frame_elems = g.N * c.heads * c.head_dim;
    g.layer_elems = static_cast<int64_t>(c.batch) * g.slots * g.frame_elems;
    g.f8 = c.kv_format == SDV2_KV_FP8_E4M3;
    g.np_tokens = (g.N + kBlockN - 1) / kBlockN * kBlockN;
    g.n_blk = static_cast<int>(g.np_tokens / kBlockN);
    g.scale_slot_stride = (c.heads * g.n_blk + 3) / 4 * 4;
    g.pack2 = g.f8 && g.N == kBlockN / 2;
    g.n_qpairs = static_cast<int>((g.lq + kBlockM * kQTilesPerCta - 1) / (kBlockM * kQTilesPerCta));
    g.lq_pad = g.n_qpairs * kBlockM * kQTilesPerCta;
    // partial blocks (256 rows each) for the split units of one launch
    g.part_rows = std::min<int64_t>(static_cast<int64_t>(std::min(c.batch, kMaxBatch)) * c.heads * g.n_qpairs *
                                        kMaxSplits, kPartRowsCap / 256) * 256;
    uint64_t off = 0;
    g.k = off;
    g.layer_stride = g.f8 ? static_cast<uint64_t>(c.batch) * g.slots * g.np_tokens * c.heads * c.head_dim
                          : static_cast<uint64_t>(g.layer_elems) * 2;
    off = align_up(off + g.layer_stride * c.layers, 256);
    g.v = off;
    off = align_up(off + g.layer_stride * c.layers, 256);
    if (g.f8) {
        g.scale_layer_stride = 4ull * c.batch * g.slots * g.scale_slot_stride;
        g.k_scale = off;
        off = align_up(off + g.scale_layer_stride * c.layers, 256);
        g.v_scale = off;
        off = align_up(off + g.scale_layer_stride * c.layers, 256);
    }
    g.rope_h64 = off;
    off = align_up(off + 16ull * c.frame_h * c.rope_pairs[1], 256);
    g.rope_w64 = off;
    off = align_up(off + 16ull * c.frame_w * c.rope_pairs[2], 256);
    g.rope_h32 = off;
    off = align_up(off + 8ull * c.frame_h * c.rope_pairs[1], 256);
    g.rope_w32 = off;
    off = align_up(off + 8ull * c.frame_w * c.rope_pairs[2], 256);
    g.omega = off;
    off = align_up(off + 8ull * c.rope_pairs[0], 256);
    g.n_phase = g.f8 ? 0 : std::min<int64_t>(c.rope_reset_period > 0 ? c.rope_reset_period : kFusePhaseCap, kFusePhaseCap);
    g.rope_t64 = off;
    off = align_up(off + 16ull * g.n_phase * c.rope_pairs[0], 256);
    g.sink_embed = off;
    off = align_up(off + 8ull * c.batch * c.sink_frames * (c.embed_dim > 0 ? c.embed_dim : 1), 256);
    g.sink_frame = off;
    off = align_up(off + 8ull * c.batch * c.sink_frames, 256);
    g.status = off;
    off = align_up(off + 4, 256);
    g.scratch = off;
    // token chunks of the chunk-mean reduction: about two blocks per SM of a 148-SM GPU
    {
        const int col_blocks = std::max(1, (c.embed_dim + 255) / 256);
        const int want = (296 + col_blocks * c.batch - 1) / (col_blocks * c.batch);
        g.refresh_chunks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({kRefreshMaxChunks, want, g.lq})));
    }
    g.refresh_mean = off;
    off = align_up(off + 8ull * c.batch * g.refresh_chunks * (c.embed_dim > 0 ? c.embed_dim : 1), 256);
    g.refresh_counter = off;
    off = align_up(off + 4ull * (kMaxBatch + static_cast<uint64_t>(c.batch) * kRefreshMaxColBlocks), 256);
    g.part_ml = off;
    off = align_up(off + 8ull * g.part_rows, 256);
    g.part_o = off;
    off = align_up(off + 4ull * c.head_dim * g.part_rows, 256);
    g.scratch_end = off;
    g.total = off;
    return g;
}

// Work decomposition of one attention launch over `units` (stream, head,
// query-tile pair) units of at most max_tiles KV tiles each.  Either every
// unit runs whole (one CTA each), or the units beyond the last complete wave
// (all of them, when there are fewer units than SMs) are split over the KV
// range into `pieces` CTAs each (2 .. kMaxSplits) and merged afterwards.
// Chosen by an estimate of the makespan, in KV-tile times: each wave of CTAs
// costs its longest CTA, i.e. a fixed start-up and epilogue (about 1.5 tiles)
// plus its tiles; the split pieces run in the waves after the whole units;
// the merge adds a fixed launch and the partials written and read back.
// Within the partial buffer's capacity.
struct AttnPlan {
    int64_t whole;
    int pieces;
};

AttnPlan plan_attention(const sdv2_cache_config &c, const Geometry &g, int64_t units, int64_t max_tiles,
                        int sm_count) {
    AttnPlan best{units, 1};
    if (units <= 0 || max_tiles <= 1 || sm_count <= 0) return best;
    const double tile_us = 2.0;            // one KV tile of one CTA (both query tiles) on a B200 SM
    const double cta_fixed_us = 3.0;       // CTA start-up (barriers, TMEM, first tiles) and epilogue
    const double merge_us = 3.0;           // the dependent merge launch
    const double bytes_per_us = 6.0e6;     // ~6 TB/s for the partials written and read back
    const int64_t cap = g.part_rows / 256;  // partial blocks of 256 rows
    auto waves = [&](int64_t ctas) { return (ctas + sm_count - 1) / sm_count; };
    auto wave_us = [&](int64_t tiles) { return cta_fixed_us + static_cast<double>(tiles) * tile_us; };
    double best_cost = static_cast<double>(waves(units)) * wave_us(max_tiles);
    const int64_t full = (units / sm_count) * sm_count;   // units that fill whole waves
    for (int s = 2; s <= kMaxSplits && s <= max_tiles; ++s) {
        const int64_t per = (max_tiles + s - 1) / s;
        for (int tail = 0; tail < 2; ++tail) {
            const int64_t whole = tail ? full : 0;
            if (tail && (full == 0 || full == units)) continue;
            const int64_t rest = units - whole;
            if (rest * s > cap) continue;
            const double cost = static_cast<double>(whole / sm_count) * wave_us(max_tiles) +
                                static_cast<double>(waves(rest * s)) * wave_us(per) + merge_us +
                                static_cast<double>(rest * s) * 256.0 * (c.head_dim + 2) * 8.0 / bytes_per_us;
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                best = {whole, s};
            }
        }
    }
    return best;
}

// Pair mode of the attention launch: with chunks of one query tile and more (stream, head)
// units than SMs, a CTA takes two heads of one stream, one accumulator set and query tile
// each, their KV tiles interleaved; half the CTAs, each start-up shared by two heads, and
// the two softmax / MMA chains of a CTA still overlap.  (Both cache formats.)
bool use_pair_mode(const Geometry &g, const sdv2_cache_config &c, int64_t units, int sm_count) {
    return g.n_qpairs == 1 && g.lq <= kBlockM && c.heads >= 2 && sm_count > 0 && units > sm_count;
}

// KV tiles of the longest stream: 128-key runs of its valid prefix, or for the fp8 cache
// the 128-token blocks of each valid slot (64-token slots: pairs of slots).
int64_t max_kv_tiles(const Geometry &g, const int64_t *keys, int n) {
    int64_t m = 0;
    for (int b = 0; b < n; ++b)
        if (keys[b] > 0)
            m = std::max<int64_t>(m, !g.f8    ? (keys[b] + kBlockN - 1) / kBlockN
                                     : g.pack2 ? (keys[b] / g.N + 1) / 2
                                               : keys[b] / g.N * g.n_blk);
    return m;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

}  // namespace

struct sdv2_cache {
    sdv2_cache_config cfg;
    Geometry g;
    uint8_t *base;
    int device;
    int sm_count;
    std::vector<int64_t> next_frame;  // [B][L]
    std::vector<CUtensorMap> tk, tv;  // [L]
    std::vector<CUtensorMap> tkh, tvh;  // [L][kFuseBoxes] bf16 cache: the same maps in boxes of 64, 32, 16, 8 rows (fused append)
    cudaEvent_t time_start = nullptr;  // measurement hook: events around the attention kernel
    cudaEvent_t time_stop = nullptr;
};

struct sdv2_motion {
    sdv2_motion_config cfg;
    uint8_t *base;
    int device;
    int n_blocks;
    int64_t frame_elems;
    uint64_t off_prev, off_has_prev, off_hist, off_hist_len, off_hist_pos, off_rate, off_partial, off_counter,
        off_status, total;
};

namespace {

sdv2_status check_device(int device) {
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (cur != device) return fail(SDV2_E_ARG, "current device %d is not the handle's device %d", cur, device);
    return SDV2_OK;
}

sdv2_status check_stream_frames(const sdv2_cache *c, int32_t layer, const int64_t *f0, bool after_append,
                                int *active_out) {
    if (!f0) return fail(SDV2_E_ARG, "chunk_first_frame is NULL");
    int active = 0;
    for (int b = 0; b < c->cfg.batch; ++b) {
        if (f0[b] < 0) continue;
        ++active;
        const int64_t expect = c->next_frame[static_cast<size_t>(b) * c->cfg.layers + layer];
        const int64_t want = after_append ? f0[b] + c->cfg.chunk_frames : f0[b];
        if (want != expect) {
            if (after_append)
                return fail(SDV2_E_STATE, "stream %d layer %d: chunk at frame %lld is not the last appended chunk", b,
                            layer, static_cast<long long>(f0[b]));
            return fail(SDV2_E_STATE, "stream %d layer %d: expected chunk at frame %lld, got %lld", b, layer,
                        static_cast<long long>(expect), static_cast<long long>(f0[b]));
        }
    }
    *active_out = active;
    return SDV2_OK;
}

// KV tiles of one stream that hold rows of its chunk's own frames (ascending), for the
// fused append: rows [slot * N, slot * N + N) of each chunk frame's ring slot, 128 keys
// per tile.  Returns their number (it may exceed `cap`; only `cap` are stored).
int chunk_tiles(const sdv2_cache_config &n, const Geometry &g, int64_t f0, int32_t *tiles, int cap) {
    int cnt = 0;
    for (int i = 0; i < n.chunk_frames; ++i) {
        const int64_t sl = slot_of(f0 + i, n.sink_frames, n.window_frames);
        for (int64_t t = sl * g.N / kBlockN; t <= (sl * g.N + g.N - 1) / kBlockN; ++t) {
            bool seen = false;
            for (int e = 0; e < std::min(cnt, cap); ++e) seen = seen || tiles[e] == t;
            if (seen) continue;
            if (cnt < cap) {
                int e = cnt;                      // insertion keeps them ascending
                while (e > 0 && tiles[e - 1] > t) {
                    tiles[e] = tiles[e - 1];
                    --e;
                }
                tiles[e] = static_cast<int32_t>(t);
            }
            ++cnt;
        }
    }
    return cnt;
}

// The 8-row groups of KV tile t of one stream (lk valid keys, chunk frame i in ring slot
// slots[i]) that hold rows of the chunk's own frames: *full gets the groups whose eight
// rows are consecutive tokens of one chunk frame (the fused kernel moves them by TMA),
// *part the others (built row by row).  Bit q: rows 8q .. 8q + 7 of the tile.
void chunk_groups(const sdv2_cache_config &n, const Geometry &g, const int32_t *slots, int64_t lk, int64_t t,
                  uint32_t *full, uint32_t *part) {
    *full = *part = 0u;
    for (int q = 0; q < kBlockN / 8; ++q) {
        const int64_t kr0 = t * kBlockN + 8 * q;
        bool any = false, whole = true;
        for (int k = 0; k < 8; ++k) {
            const int64_t kr = kr0 + k;
            if (kr >= lk) {
                whole = false;
                continue;
            }
            const int64_t sl = kr / g.N;
            bool is_new = false;
            for (int i = 0; i < n.chunk_frames; ++i) is_new = is_new || slots[i] == sl;
            any = any || is_new;
            whole = whole && is_new && sl == kr0 / g.N;
        }
        if (any) *(whole ? full : part) |= 1u << q;
    }
}

// Whether sdv2_append_attention runs the fused kernel for these chunk positions: bf16
// cache, at most two query tiles per stream (one CTA, or its KV pieces, per stream and
// head), at most kFuseMaxFrames chunk frames whose temporal tables fit the CTA's
// kFuseTabSmem entries and whose phases lie in the cache's phase table, row and column
// tables that fit fuse_tab_hw_bytes(head_dim), and at most
// kFuseMaxAsmTiles KV tiles per stream holding the chunk's rows.  0: the append and the attention run as two launches; 1: fused;
// 2: fused, pair mode (one tile per stream and more (stream, head) units than SMs).
int fuse_mode(const sdv2_cache_config &n, const Geometry &g, const int64_t *f0, int sm_count) {
    if (g.f8 || g.n_qpairs != 1 || n.chunk_frames > kFuseMaxFrames ||
        n.chunk_frames * n.rope_pairs[0] > kFuseTabSmem ||
        (static_cast<int64_t>(n.frame_h) * n.rope_pairs[1] + static_cast<int64_t>(n.frame_w) * n.rope_pairs[2]) * 16 >
            fuse_tab_hw_bytes(n.head_dim))
        return 0;
    bool one_tile = true;
    int64_t active = 0;
    for (int b = 0; b < n.batch; ++b) {
        if (f0[b] < 0) continue;
        ++active;
        for (int i = 0; i < n.chunk_frames; ++i)
            if (phase_of(f0[b] + i, n.rope_reset_period) >= g.n_phase) return 0;   // beyond the cache's phase table
        int32_t t[kFuseMaxAsmTiles];
        const int cnt = chunk_tiles(n, g, f0[b], t, kFuseMaxAsmTiles);
        if (cnt > kFuseMaxAsmTiles) return 0;
        one_tile = one_tile && cnt == 1;
    }
    return one_tile && use_pair_mode(g, n, active * n.heads * g.n_qpairs, sm_count) ? 2 : 1;
}

// One attention call over the streams with chunk_first_frame >= 0 (the caller checked
// the arguments and the stream positions).  With k and v given, the chunk's KV append
// is fused in (fuse_mode != 0).
sdv2_status run_attention(sdv2_cache *c, int32_t layer, const void *q, void *out, const int64_t *chunk_first_frame,
                          float softmax_scale, cudaStream_t s, const void *k, const void *v) {
    const sdv2_cache_config &n = c->cfg;
    const Geometry &g = c->g;
    const bool fuse = k != nullptr;
    std::vector<int64_t> keys(n.batch, 0);
    for (int b = 0; b < n.batch; ++b) {
        if (chunk_first_frame[b] < 0) continue;
        int32_t sv, wv;
        valid_counts(chunk_first_frame[b] + n.chunk_frames, n.sink_frames, n.window_frames, &sv, &wv);
        keys[b] = static_cast<int64_t>(sv + wv) * g.N;
    }
    const int n_t = n.rope_pairs[0];
    // The caller's un-rotated queries as a TMA tensor (d, H, Lq, B), bf16, in boxes of 64
    // channels x 128 rows with the 128-byte swizzle of the MMA's Q tiles; the kernel rotates
    // them on load.  Encoded per call: q is the caller's buffer.
    CUtensorMap tq;
    {
        PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
        if (!encode) return fail(SDV2_E_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        const cuuint64_t qdims[4] = {static_cast<cuuint64_t>(n.head_dim), static_cast<cuuint64_t>(n.heads),
                                     static_cast<cuuint64_t>(g.lq), static_cast<cuuint64_t>(n.batch)};
        const cuuint64_t qstrides[3] = {static_cast<cuuint64_t>(n.head_dim) * 2,
                                        static_cast<cuuint64_t>(n.heads) * n.head_dim * 2,
                                        static_cast<cuuint64_t>(g.lq) * n.heads * n.head_dim * 2};
        const cuuint32_t qbox[4] = {64u, 1, static_cast<cuuint32_t>(kBlockM), 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        CUresult r = encode(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), qdims, qstrides, qbox,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(SDV2_E_CUDA, "cuTensorMapEncodeTiled (queries) failed (%d)", static_cast<int>(r));
    }
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.out = static_cast<uint16_t *>(out);
    p.part_o = reinterpret_cast<float *>(c->base + g.part_o);
    p.part_ml = reinterpret_cast<float *>(c->base + g.part_ml);
    p.rope_h = reinterpret_cast<const float *>(c->base + g.rope_h32);
    p.rope_w = reinterpret_cast<const float *>(c->base + g.rope_w32);
    p.status = reinterpret_cast<uint32_t *>(c->base + g.status);
    p.batch = n.batch;
    p.heads = n.heads;
    p.lq = static_cast<int32_t>(g.lq);
    p.tokens_per_frame = static_cast<int32_t>(g.N);
    p.frame_h = n.frame_h;
    p.frame_w = n.frame_w;
    p.chunk_frames = n.chunk_frames;
    p.n_t = n_t;
    p.n_h = n.rope_pairs[1];
    p.n_w = n.rope_pairs[2];
    p.n_qpairs = g.n_qpairs;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.omega_t = reinterpret_cast<const double *>(c->base + g.omega);
    p.rope_reset = n.rope_reset_period;
    if (g.f8) {
        p.k_scale = reinterpret_cast<const float *>(c->base + g.k_scale + g.scale_layer_stride * layer);
        p.v_scale = reinterpret_cast<const float *>(c->base + g.v_scale + g.scale_layer_stride * layer);
        p.f8 = 1;
        p.slots = static_cast<int32_t>(g.slots);
        p.np_tokens = static_cast<int32_t>(g.np_tokens);
        p.n_blk = g.n_blk;
        p.scale_slot_stride = g.scale_slot_stride;
        p.pack2 = g.pack2 ? 1 : 0;
    }
    std::unique_ptr<FuseParams> fp;
    if (fuse) {
        fp.reset(new FuseParams());
        std::memset(fp.get(), 0, sizeof(FuseParams));
        fp->k_in = static_cast<const uint16_t *>(k);
        fp->v_in = static_cast<const uint16_t *>(v);
        fp->k_layer = reinterpret_cast<uint16_t *>(c->base + g.k + g.layer_stride * layer);
        fp->v_layer = reinterpret_cast<uint16_t *>(c->base + g.v + g.layer_stride * layer);
        fp->rope_h = reinterpret_cast<const double *>(c->base + g.rope_h64);
        fp->rope_w = reinterpret_cast<const double *>(c->base + g.rope_w64);
        fp->rope_t = reinterpret_cast<const double *>(c->base + g.rope_t64);
        fp->slots = static_cast<int32_t>(g.slots);
        for (int i = 0; i < kFuseBoxes; ++i) {
            fp->tmap_kc[i] = c->tkh[static_cast<size_t>(layer) * kFuseBoxes + i];
            fp->tmap_vc[i] = c->tvh[static_cast<size_t>(layer) * kFuseBoxes + i];
        }
        // the caller's k and v as TMA tensors (d, H, T'N, B), bf16, boxes of 64 channels x
        // (64 >> i) rows, 128-byte swizzle (the tiles' layout); encoded per call: k and v are
        // the caller's
        PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
        const cuuint64_t dims[4] = {static_cast<cuuint64_t>(n.head_dim), static_cast<cuuint64_t>(n.heads),
                                    static_cast<cuuint64_t>(g.lq), static_cast<cuuint64_t>(n.batch)};
        const cuuint64_t strides[3] = {static_cast<cuuint64_t>(n.head_dim) * 2,
                                       static_cast<cuuint64_t>(n.heads) * n.head_dim * 2,
                                       static_cast<cuuint64_t>(g.lq) * n.heads * n.head_dim * 2};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        for (int kv = 0; kv < 2; ++kv)
            for (int i = 0; i < kFuseBoxes; ++i) {
                const cuuint32_t box[4] = {64u, 1, static_cast<cuuint32_t>(64 >> i), 1};
                CUresult r = encode(kv ? &fp->tmap_vi[i] : &fp->tmap_ki[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                                    const_cast<void *>(kv ? v : k), dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
                if (r != CUDA_SUCCESS)
                    return fail(SDV2_E_CUDA, "cuTensorMapEncodeTiled (chunk k / v) failed (%d)", static_cast<int>(r));
            }
    }
    for (int b0 = 0; b0 < n.batch; b0 += kMaxBatch) {
        const int nb = std::min(kMaxBatch, n.batch - b0);     // the launch's streams: b0 .. b0 + nb - 1
        if (fuse)
            for (int bl = 0; bl < nb; ++bl) {
                const int64_t f0 = chunk_first_frame[b0 + bl];
                if (f0 < 0) continue;
                for (int i = 0; i < n.chunk_frames; ++i) {
                    fp->new_slot[bl][i] = slot_of(f0 + i, n.sink_frames, n.window_frames);
                    fp->phase[bl][i] = static_cast<int32_t>(phase_of(f0 + i, n.rope_reset_period));
                }
                int32_t t[kFuseMaxAsmTiles] = {-1, -1};
                chunk_tiles(n, g, f0, t, kFuseMaxAsmTiles);
                for (int e = 0; e < kFuseMaxAsmTiles; ++e) {
                    fp->asm_tile[bl][e] = t[e];
                    fp->grp_full[bl][e] = fp->grp_part[bl][e] = 0u;
                    if (t[e] >= 0)
                        chunk_groups(n, g, fp->new_slot[bl], keys[b0 + bl], t[e], &fp->grp_full[bl][e],
                                     &fp->grp_part[bl][e]);
                }
            }
        p.b_offset = b0;
        bool any = false, one_tile = true;
        int n_active = 0;
        for (int bl = 0; bl < kMaxBatch; ++bl) p.lk[bl] = 0;
        for (int bl = 0; bl < nb; ++bl) {
            const int b = b0 + bl;
            p.lk[bl] = static_cast<int32_t>(keys[b]);
            p.f0[bl] = chunk_first_frame[b];
            if (keys[b] > 0) {
                any = true;
                p.unit_stream[n_active++] = static_cast<uint8_t>(bl);
                if (fuse) one_tile = one_tile && fp->asm_tile[bl][1] < 0;
            }
        }
        if (!any) continue;
        p.n_units = n_active * n.heads * g.n_qpairs;
        // (the fused pair mode takes the one assembled tile of each stream for both heads)
        if (use_pair_mode(g, n, p.n_units, c->sm_count) && (!fuse || one_tile)) {
            p.pair = 1;
            p.n_whole = p.n_units;
            p.n_pieces = 1;
        } else {
            p.pair = 0;
            const AttnPlan plan =
                plan_attention(n, g, p.n_units, max_kv_tiles(g, keys.data() + b0, nb), c->sm_count);
            p.n_whole = static_cast<int32_t>(plan.whole);
            p.n_pieces = plan.pieces;
        }
        cudaError_t e = cudaSuccess;
        if (c->time_start && b0 == 0) {
            e = cudaEventRecord(c->time_start, s);
            if (e != cudaSuccess) return cuda_fail(e, "chunk_attention start event");
        }
        e = fuse ? launch_append_attention(p, *fp, tq, c->tk[layer], c->tv[layer], n.head_dim, s)
                 : launch_attention(p, tq, c->tk[layer], c->tv[layer], n.head_dim, s);
        if (e != cudaSuccess) return cuda_fail(e, fuse ? "append_attention launch" : "chunk_attention launch");
        if (c->time_stop && b0 + kMaxBatch >= n.batch) {
            e = cudaEventRecord(c->time_stop, s);
            if (e != cudaSuccess) return cuda_fail(e, "chunk_attention stop event");
        }
        g_launches.fetch_add(1);
        if (p.n_whole < p.n_units) {
            e = launch_combine(p, n.head_dim, s);
            if (e != cudaSuccess) return cuda_fail(e, "attention combine launch");
            g_launches.fetch_add(1);
        }
    }
    return SDV2_OK;
}

}  // namespace

extern "C" {

size_t sdv2_cache_bytes(const sdv2_cache_config *cfg) {
    sdv2_cache_config n;
    if (check_config(cfg, &n) != SDV2_OK) return 0;
    return static_cast<size_t>(geometry(n).total);
}

static void fill_layout(const sdv2_cache_config &n, const Geometry &g, sdv2_cache_layout *out) {
    out->k_offset = g.k;
    out->v_offset = g.v;
    out->layer_stride = g.layer_stride;
    out->sink_embed_offset = g.sink_embed;
    out->sink_frame_offset = g.sink_frame;
    out->status_offset = g.status;
    out->scratch_offset = g.scratch;
    out->scratch_bytes = g.scratch_end - g.scratch;
    out->total_bytes = g.total;
    out->k_scale_offset = g.f8 ? g.k_scale : 0;
    out->v_scale_offset = g.f8 ? g.v_scale : 0;
    out->scale_layer_stride = g.f8 ? g.scale_layer_stride : 0;
    out->scale_slot_stride = g.f8 ? static_cast<uint32_t>(g.scale_slot_stride) : 0;
    out->tokens_padded = g.f8 ? static_cast<uint32_t>(g.np_tokens) : 0;
    (void)n;
}

sdv2_status sdv2_cache_layout_of(const sdv2_cache_config *cfg, sdv2_cache_layout *out) {
    if (!out) return fail(SDV2_E_ARG, "out is NULL");
    sdv2_cache_config n;
    sdv2_status st = check_config(cfg, &n);
    if (st != SDV2_OK) return st;
    fill_layout(n, geometry(n), out);
    return SDV2_OK;
}

sdv2_status sdv2_cache_create(const sdv2_cache_config *cfg, void *dev_buf, size_t bytes, sdv2_cache **out) {
    if (!out) return fail(SDV2_E_ARG, "out is NULL");
    *out = nullptr;
    sdv2_cache_config n;
    sdv2_status st = check_config(cfg, &n);
    if (st != SDV2_OK) return st;
    if (!dev_buf) return fail(SDV2_E_ARG, "dev_buf is NULL");
    if ((reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) return fail(SDV2_E_ALIGN, "dev_buf must be 256-byte aligned");
    const Geometry g = geometry(n);
    if (bytes < g.total)
        return fail(SDV2_E_ALIGN, "buffer of %zu bytes is smaller than the %llu bytes required", bytes,
                    static_cast<unsigned long long>(g.total));
    PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
    if (!encode) return fail(SDV2_E_CUDA, "cuTensorMapEncodeTiled is not available from the driver");

    sdv2_cache *c = new sdv2_cache();
    c->cfg = n;
    c->g = g;
    c->base = static_cast<uint8_t *>(dev_buf);
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device);
    if (e == cudaSuccess) e = cudaMemset(dev_buf, 0, g.total);
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail(e, "cache_create");
    }
    // RoPE row / column tables (fp64 for the bit-exact key rotation, fp32 for queries).
    const int nh = n.rope_pairs[1], nw = n.rope_pairs[2];
    std::vector<double> h64(2ull * n.frame_h * nh), w64(2ull * n.frame_w * nw);
    std::vector<float> h32(h64.size()), w32(w64.size());
    for (int r = 0; r < n.frame_h; ++r)
        for (int j = 0; j < nh; ++j) {
            const double a = rope_angle(n.rope_base, j, nh, r);
            h64[2 * (r * nh + j)] = std::cos(a);
            h64[2 * (r * nh + j) + 1] = std::sin(a);
        }
    for (int col = 0; col < n.frame_w; ++col)
        for (int j = 0; j < nw; ++j) {
            const double a = rope_angle(n.rope_base, j, nw, col);
            w64[2 * (col * nw + j)] = std::cos(a);
            w64[2 * (col * nw + j) + 1] = std::sin(a);
        }
    // fp32 copies for the queries, pair-major ([pair][position] (cos, sin)): the attention
    // kernel rotates one query row per thread, so for a given pair the 32 lanes of a warp
    // (consecutive tokens, consecutive columns) read consecutive entries
    for (int r = 0; r < n.frame_h; ++r)
        for (int j = 0; j < nh; ++j)
            for (int k = 0; k < 2; ++k)
                h32[2 * (static_cast<size_t>(j) * n.frame_h + r) + k] = static_cast<float>(h64[2 * (r * nh + j) + k]);
    for (int col = 0; col < n.frame_w; ++col)
        for (int j = 0; j < nw; ++j)
            for (int k = 0; k < 2; ++k)
                w32[2 * (static_cast<size_t>(j) * n.frame_w + col) + k] =
                    static_cast<float>(w64[2 * (col * nw + j) + k]);
    std::vector<int64_t> sink_frames(static_cast<size_t>(n.batch) * n.sink_frames, -1);
    // temporal frequencies (the queries' angles are formed on the device), and the fp64
    // (cos, sin) of every temporal pair at phases 0 .. n_phase - 1 (the fused append
    // rotates keys with these, the same values the append's per-call table carries)
    const int nt = n.rope_pairs[0];
    std::vector<double> omega(nt), t64(2ull * g.n_phase * nt);
    for (int j = 0; j < nt; ++j) omega[j] = rope_angle(n.rope_base, j, nt, 1);
    for (int64_t ph = 0; ph < g.n_phase; ++ph)
        for (int j = 0; j < nt; ++j) {
            const double a = rope_angle(n.rope_base, j, nt, ph);
            t64[2 * (ph * nt + j)] = std::cos(a);
            t64[2 * (ph * nt + j) + 1] = std::sin(a);
        }
    struct Up { uint64_t off; const void *src; size_t bytes; } ups[] = {
        {g.rope_h64, h64.data(), h64.size() * 8}, {g.rope_w64, w64.data(), w64.size() * 8},
        {g.rope_h32, h32.data(), h32.size() * 4}, {g.rope_w32, w32.data(), w32.size() * 4},
        {g.omega, omega.data(), omega.size() * 8}, {g.rope_t64, t64.data(), t64.size() * 8},
        {g.sink_frame, sink_frames.data(), sink_frames.size() * 8}};
    for (const Up &u : ups) {
        if (u.bytes == 0) continue;
        e = cudaMemcpy(c->base + u.off, u.src, u.bytes, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            delete c;
            return cuda_fail(e, "cache_create upload");
        }
    }
    // One TMA descriptor per layer for K and for V.  bf16: dims (d, H, slots*N, B), boxes of
    // 64 channels x 128 keys.  fp8: K codes (d, H, slots*Np, B) and transposed V codes
    // (Np, d, H, slots, B), boxes of 128 bytes x 128 rows; with 64-token slots (two per KV
    // tile) boxes of 64 K rows, and of 64 V bytes (one slot's keys) x 128 rows, 64-byte
    // swizzled.
    c->tk.resize(n.layers);
    c->tv.resize(n.layers);
    c->tkh.resize(g.f8 ? 0 : static_cast<size_t>(n.layers) * kFuseBoxes);
    c->tvh.resize(g.f8 ? 0 : static_cast<size_t>(n.layers) * kFuseBoxes);
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    for (int l = 0; l < n.layers; ++l) {
        for (int kv = 0; kv < 2; ++kv) {
            void *ptr = c->base + (kv ? g.v : g.k) + g.layer_stride * l;
            CUresult r;
            if (!g.f8) {
                const cuuint64_t dims[4] = {static_cast<cuuint64_t>(n.head_dim), static_cast<cuuint64_t>(n.heads),
                                            static_cast<cuuint64_t>(g.slots * g.N), static_cast<cuuint64_t>(n.batch)};
                const cuuint64_t strides[3] = {static_cast<cuuint64_t>(n.head_dim) * 2,
                                               static_cast<cuuint64_t>(n.heads) * n.head_dim * 2,
                                               static_cast<cuuint64_t>(g.slots * g.frame_elems) * 2};
                const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kBlockN), 1};
                r = encode(kv ? &c->tv[l] : &c->tk[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
                for (int i = 0; r == CUDA_SUCCESS && i < kFuseBoxes; ++i) {
                    const cuuint32_t boxh[4] = {64, 1, static_cast<cuuint32_t>(64 >> i), 1};
                    CUtensorMap *m = &(kv ? c->tvh : c->tkh)[static_cast<size_t>(l) * kFuseBoxes + i];
                    r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims, strides, boxh, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
                }
            } else if (kv == 0) {
                const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(n.heads),
                                            static_cast<cuuint64_t>(g.slots * g.np_tokens),
                                            static_cast<cuuint64_t>(n.batch)};
                const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(n.heads) * 128,
                                               static_cast<cuuint64_t>(g.slots * g.np_tokens * n.heads) * 128};
                const cuuint32_t box[4] = {128, 1, static_cast<cuuint32_t>(g.pack2 ? kBlockN / 2 : kBlockN), 1};
                r = encode(&c->tk[l], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, ptr, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            } else {
                const cuuint64_t dims[5] = {static_cast<cuuint64_t>(g.np_tokens), 128,
                                            static_cast<cuuint64_t>(n.heads), static_cast<cuuint64_t>(g.slots),
                                            static_cast<cuuint64_t>(n.batch)};
                const cuuint64_t strides[4] = {static_cast<cuuint64_t>(g.np_tokens),
                                               static_cast<cuuint64_t>(g.np_tokens) * 128,
                                               static_cast<cuuint64_t>(g.np_tokens) * 128 * n.heads,
                                               static_cast<cuuint64_t>(g.np_tokens) * 128 * n.heads * g.slots};
                const cuuint32_t box[5] = {static_cast<cuuint32_t>(g.pack2 ? kBlockN / 2 : kBlockN), 128, 1, 1, 1};
                // (64-token slots: 64-byte L2 fills, so that a row's padding half is not read)
                r = encode(&c->tv[l], CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, ptr, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           g.pack2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                           g.pack2 ? CU_TENSOR_MAP_L2_PROMOTION_L2_64B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            }
            if (r != CUDA_SUCCESS) {
                delete c;
                return fail(SDV2_E_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
            }
        }
    }
    c->next_frame.assign(static_cast<size_t>(n.batch) * n.layers, 0);
    *out = c;
    return SDV2_OK;
}

sdv2_status sdv2_cache_destroy(sdv2_cache *cache) {
    delete cache;
    return SDV2_OK;
}

sdv2_status sdv2_kv_append(sdv2_cache *c, int32_t layer, const void *k, const void *v,
                           const int64_t *chunk_first_frame, sdv2_stream stream) {
    if (!c || !k || !v) return fail(SDV2_E_ARG, "NULL argument");
    if (layer < 0 || layer >= c->cfg.layers) return fail(SDV2_E_ARG, "layer %d out of range", layer);
    if (!aligned16(k) || !aligned16(v)) return fail(SDV2_E_ALIGN, "k and v must be 16-byte aligned");
    int active = 0;
    sdv2_status st = check_stream_frames(c, layer, chunk_first_frame, false, &active);
    if (st != SDV2_OK) return st;
    if ((st = check_device(c->device)) != SDV2_OK) return st;
    const sdv2_cache_config &n = c->cfg;
    const int n_t = n.rope_pairs[0];
    const int max_rows = kAppendTabEntries / n_t;     // distinct phases per launch
    int64_t row_phase[kAppendTabEntries];
    int n_rows = 0;
    AppendParams p;
    std::memset(&p, 0, sizeof(p));
    p.k_in = static_cast<const uint16_t *>(k);
    p.v_in = static_cast<const uint16_t *>(v);
    p.k_layer = reinterpret_cast<uint16_t *>(c->base + c->g.k + c->g.layer_stride * layer);
    p.v_layer = reinterpret_cast<uint16_t *>(c->base + c->g.v + c->g.layer_stride * layer);
    p.rope_h = reinterpret_cast<const double *>(c->base + c->g.rope_h64);
    p.rope_w = reinterpret_cast<const double *>(c->base + c->g.rope_w64);
    p.frame_elems = c->g.frame_elems;
    p.chunk_tokens = static_cast<int32_t>(c->g.lq);
    p.heads = n.heads;
    p.head_dim = n.head_dim;
    p.frame_w = n.frame_w;
    p.n_t = n_t;
    p.n_h = n.rope_pairs[1];
    p.n_w = n.rope_pairs[2];
    p.slots = static_cast<int32_t>(c->g.slots);
    if (c->g.f8) {
        p.k_layer = p.v_layer = nullptr;
        p.k8_layer = reinterpret_cast<uint8_t *>(c->base + c->g.k + c->g.layer_stride * layer);
        p.v8t_layer = reinterpret_cast<uint8_t *>(c->base + c->g.v + c->g.layer_stride * layer);
        p.k_scale_layer = reinterpret_cast<float *>(c->base + c->g.k_scale + c->g.scale_layer_stride * layer);
        p.v_scale_layer = reinterpret_cast<float *>(c->base + c->g.v_scale + c->g.scale_layer_stride * layer);
        p.tokens = static_cast<int32_t>(c->g.N);
        p.np_tokens = static_cast<int32_t>(c->g.np_tokens);
        p.n_blk = c->g.n_blk;
        p.scale_slot_stride = c->g.scale_slot_stride;
    }
    auto flush = [&]() -> sdv2_status {
        if (p.n_frames == 0) return SDV2_OK;
        cudaError_t e = launch_append(p, c->sm_count, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "kv_append launch");
        g_launches.fetch_add(1);
        p.n_frames = 0;
        n_rows = 0;
        return SDV2_OK;
    };
    for (int b = 0; b < n.batch; ++b) {
        const int64_t f0 = chunk_first_frame[b];
        if (f0 < 0) continue;
        for (int i = 0; i < n.chunk_frames; ++i) {
            const int64_t f = f0 + i;
            const int64_t ph = phase_of(f, n.rope_reset_period);
            // streams at the same phase share one row of the temporal table
            int row = 0;
            while (row < n_rows && row_phase[row] != ph) ++row;
            if (row == n_rows) {
                if (n_rows == max_rows) {
                    if ((st = flush()) != SDV2_OK) return st;
                    row = 0;
                }
                row_phase[row] = ph;
                for (int j = 0; j < n_t; ++j) {
                    const double a = rope_angle(n.rope_base, j, n_t, ph);
                    p.tab_t[row * n_t + j][0] = std::cos(a);
                    p.tab_t[row * n_t + j][1] = std::sin(a);
                }
                n_rows = row + 1;
            }
            const int fi = p.n_frames;
            p.src_b[fi] = b;
            p.src_i[fi] = i;
            p.dst_slot[fi] = slot_of(f, n.sink_frames, n.window_frames);
            p.tab_row[fi] = static_cast<uint8_t>(row);
            ++p.n_frames;
            if (p.n_frames == kAppendMaxFrames && (st = flush()) != SDV2_OK) return st;
        }
    }
    if ((st = flush()) != SDV2_OK) return st;
    for (int b = 0; b < n.batch; ++b)
        if (chunk_first_frame[b] >= 0) c->next_frame[static_cast<size_t>(b) * n.layers + layer] += n.chunk_frames;
    return SDV2_OK;
}

sdv2_status sdv2_chunk_attention(sdv2_cache *c, int32_t layer, const void *q, void *out,
                                 const int64_t *chunk_first_frame, float softmax_scale, sdv2_stream stream) {
    if (!c || !q || !out) return fail(SDV2_E_ARG, "NULL argument");
    if (layer < 0 || layer >= c->cfg.layers) return fail(SDV2_E_ARG, "layer %d out of range", layer);
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return fail(SDV2_E_ARG, "softmax_scale must be > 0");
    if (!aligned16(q) || !aligned16(out)) return fail(SDV2_E_ALIGN, "q and out must be 16-byte aligned");
    int active = 0;
    sdv2_status st = check_stream_frames(c, layer, chunk_first_frame, true, &active);
    if (st != SDV2_OK) return st;
    if ((st = check_device(c->device)) != SDV2_OK) return st;
    if (active == 0) return SDV2_OK;
    return run_attention(c, layer, q, out, chunk_first_frame, softmax_scale, reinterpret_cast<cudaStream_t>(stream),
                         nullptr, nullptr);
}

sdv2_status sdv2_append_attention(sdv2_cache *c, int32_t layer, const void *q, const void *k, const void *v,
                                  void *out, const int64_t *chunk_first_frame, float softmax_scale,
                                  sdv2_stream stream) {
    if (!c || !q || !k || !v || !out) return fail(SDV2_E_ARG, "NULL argument");
    if (layer < 0 || layer >= c->cfg.layers) return fail(SDV2_E_ARG, "layer %d out of range", layer);
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return fail(SDV2_E_ARG, "softmax_scale must be > 0");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k) || !aligned16(v))
        return fail(SDV2_E_ALIGN, "q, k, v and out must be 16-byte aligned");
    int active = 0;
    sdv2_status st = check_stream_frames(c, layer, chunk_first_frame, false, &active);
    if (st != SDV2_OK) return st;
    if ((st = check_device(c->device)) != SDV2_OK) return st;
    if (active == 0) return SDV2_OK;
    if (fuse_mode(c->cfg, c->g, chunk_first_frame, c->sm_count) == 0) {
        // not covered by the fused kernel: the append, then the attention (same results)
        if ((st = sdv2_kv_append(c, layer, k, v, chunk_first_frame, stream)) != SDV2_OK) return st;
        return sdv2_chunk_attention(c, layer, q, out, chunk_first_frame, softmax_scale, stream);
    }
    st = run_attention(c, layer, q, out, chunk_first_frame, softmax_scale, reinterpret_cast<cudaStream_t>(stream), k, v);
    if (st != SDV2_OK) return st;
    for (int b = 0; b < c->cfg.batch; ++b)
        if (chunk_first_frame[b] >= 0) c->next_frame[static_cast<size_t>(b) * c->cfg.layers + layer] += c->cfg.chunk_frames;
    return SDV2_OK;
}

sdv2_status sdv2_sink_refresh(sdv2_cache *c, const void *hidden, float tau, const int64_t *chunk_first_frame,
                              int32_t *out_slot_dev, sdv2_stream stream) {
    if (!c || !hidden || !out_slot_dev) return fail(SDV2_E_ARG, "NULL argument");
    if (c->cfg.embed_dim <= 0) return fail(SDV2_E_SHAPE, "the cache was created with embed_dim 0");
    if (!aligned16(hidden) || (reinterpret_cast<uintptr_t>(out_slot_dev) & 3u))
        return fail(SDV2_E_ALIGN, "hidden must be 16-byte aligned and out_slot_dev 4-byte aligned");
    if (!std::isfinite(tau)) return fail(SDV2_E_ARG, "tau must be finite");
    if (!chunk_first_frame) return fail(SDV2_E_ARG, "chunk_first_frame is NULL");
    const sdv2_cache_config &n = c->cfg;
    for (int l = 0; l < n.layers; ++l) {
        int active = 0;
        sdv2_status st = check_stream_frames(c, l, chunk_first_frame, true, &active);
        if (st != SDV2_OK) return st;
    }
    sdv2_status st = check_device(c->device);
    if (st != SDV2_OK) return st;
    const Geometry &g = c->g;
    RefreshParams p;
    std::memset(&p, 0, sizeof(p));
    p.hidden = static_cast<const uint16_t *>(hidden);
    p.partial = reinterpret_cast<double *>(c->base + g.refresh_mean);
    p.counter = reinterpret_cast<uint32_t *>(c->base + g.refresh_counter);
    p.sink_embed = reinterpret_cast<double *>(c->base + g.sink_embed);
    p.sink_frame = reinterpret_cast<int64_t *>(c->base + g.sink_frame);
    p.out_slot = out_slot_dev;
    // slot-to-slot copy regions: K and V (codes, for the fp8 cache, plus their scales)
    const int64_t kv_slot_bytes = g.layer_stride / (static_cast<int64_t>(n.batch) * g.slots);
    p.copy_base[0] = c->base + g.k;
    p.copy_base[1] = c->base + g.v;
    p.copy_layer_bytes[0] = p.copy_layer_bytes[1] = static_cast<int64_t>(g.layer_stride);
    p.copy_slot_bytes[0] = p.copy_slot_bytes[1] = kv_slot_bytes;
    p.n_copy = 2;
    if (g.f8) {
        p.copy_base[2] = c->base + g.k_scale;
        p.copy_base[3] = c->base + g.v_scale;
        p.copy_layer_bytes[2] = p.copy_layer_bytes[3] = static_cast<int64_t>(g.scale_layer_stride);
        p.copy_slot_bytes[2] = p.copy_slot_bytes[3] = 4ll * g.scale_slot_stride;
        p.n_copy = 4;
    }
    p.batch = n.batch;
    p.lq = static_cast<int32_t>(g.lq);
    p.dim = n.embed_dim;
    p.sinks = n.sink_frames;
    p.slots = static_cast<int32_t>(g.slots);
    p.layers = n.layers;
    p.row_chunks = g.refresh_chunks;
    p.tau = static_cast<double>(tau);
    for (int b = 0; b < n.batch; ++b) {
        const int64_t f0 = chunk_first_frame[b];
        p.fill_first[b] = -1;
        if (f0 < 0) continue;
        p.active[b] = 1;
        if (f0 < n.sink_frames) {
            p.fill_first[b] = static_cast<int32_t>(f0);
            const int64_t end = std::min<int64_t>(n.sink_frames, f0 + n.chunk_frames);
            p.fill_count[b] = static_cast<int32_t>(end - f0);
        }
        p.last_frame[b] = f0 + n.chunk_frames - 1;
        p.last_slot[b] = slot_of(p.last_frame[b], n.sink_frames, n.window_frames);
    }
    int launches = 0;
    cudaError_t e = launch_refresh(p, c->sm_count, reinterpret_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(static_cast<uint64_t>(launches));
    if (e != cudaSuccess) return cuda_fail(e, "sink_refresh launch");
    return SDV2_OK;
}

sdv2_status sdv2_cache_time_attention(sdv2_cache *c, sdv2_event start, sdv2_event stop) {
    if (!c) return fail(SDV2_E_ARG, "cache is NULL");
    if ((start == nullptr) != (stop == nullptr)) return fail(SDV2_E_ARG, "give both events or neither");
    c->time_start = reinterpret_cast<cudaEvent_t>(start);
    c->time_stop = reinterpret_cast<cudaEvent_t>(stop);
    return SDV2_OK;
}

sdv2_status sdv2_cache_query(const sdv2_cache *c, int32_t b, int32_t layer, int64_t *slot_frame, int32_t *slot_phase,
                             int32_t *valid_slots) {
    if (!c) return fail(SDV2_E_ARG, "cache is NULL");
    const sdv2_cache_config &n = c->cfg;
    if (b < 0 || b >= n.batch || layer < 0 || layer >= n.layers) return fail(SDV2_E_ARG, "stream or layer out of range");
    const int64_t f_end = c->next_frame[static_cast<size_t>(b) * n.layers + layer];
    const int slots = n.sink_frames + n.window_frames;
    for (int s = 0; s < slots; ++s) {
        if (slot_frame) slot_frame[s] = -1;
        if (slot_phase) slot_phase[s] = -1;
    }
    for (int64_t f = f_end - n.window_frames - n.sink_frames; f < f_end; ++f) {
        if (f < 0) continue;
        const int s = slot_of(f, n.sink_frames, n.window_frames);
        if (slot_frame) slot_frame[s] = f;
        if (slot_phase) slot_phase[s] = static_cast<int32_t>(phase_of(f, n.rope_reset_period));
    }
    for (int s = 0; s < n.sink_frames && s < f_end; ++s) {
        if (slot_frame) slot_frame[s] = s;
        if (slot_phase) slot_phase[s] = static_cast<int32_t>(phase_of(s, n.rope_reset_period));
    }
    int32_t sv, wv;
    valid_counts(f_end, n.sink_frames, n.window_frames, &sv, &wv);
    if (valid_slots) *valid_slots = sv + wv;
    return SDV2_OK;
}

sdv2_status sdv2_cache_layout_get(const sdv2_cache *c, sdv2_cache_layout *out) {
    if (!c || !out) return fail(SDV2_E_ARG, "NULL argument");
    fill_layout(c->cfg, c->g, out);
    return SDV2_OK;
}

sdv2_status sdv2_cache_check(sdv2_cache *c) {
    if (!c) return fail(SDV2_E_ARG, "cache is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cache_check");
    uint32_t word = 0;
    e = cudaMemcpy(&word, c->base + c->g.status, 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cache_check");
    if (word != 0) {
        // A block that gave up may have left the refresh ticket half counted: re-arm it.
        cudaMemset(c->base + c->g.status, 0, 4);
        cudaMemset(c->base + c->g.refresh_counter, 0,
                   4ull * (kMaxBatch + static_cast<uint64_t>(c->cfg.batch) * kRefreshMaxColBlocks));
        cudaDeviceSynchronize();
        return fail(SDV2_E_DEVICE, "device status 0x%x (a kernel gave up on a bounded wait)", word);
    }
    return SDV2_OK;
}

sdv2_status sdv2_cache_selftest_wait(sdv2_cache *c, uint64_t limit_ns, sdv2_stream stream) {
    if (!c) return fail(SDV2_E_ARG, "cache is NULL");
    if (limit_ns == 0 || limit_ns > kWaitLimitNs) return fail(SDV2_E_ARG, "limit_ns must be in 1..%llu",
                                                               static_cast<unsigned long long>(kWaitLimitNs));
    sdv2_status st = check_device(c->device);
    if (st != SDV2_OK) return st;
    cudaError_t e = launch_wait_selftest(reinterpret_cast<uint32_t *>(c->base + c->g.status), limit_ns,
                                         reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
    g_launches.fetch_add(1);
    return SDV2_OK;
}

// ------------------------------------------------------------------ motion

static sdv2_status check_motion(const sdv2_motion_config *m) {
    if (!m) return fail(SDV2_E_ARG, "config is NULL");
    if (m->batch < 1 || m->batch > kMaxBatch) return fail(SDV2_E_SHAPE, "batch must be in 1..%d", kMaxBatch);
    if (m->chunk_frames < 1 || m->chunk_frames > 64) return fail(SDV2_E_SHAPE, "chunk_frames must be in 1..64");
    if (m->channels < 1 || m->height < 1 || m->width < 1) return fail(SDV2_E_SHAPE, "latent shape must be >= 1");
    if (m->window < 1 || m->window > 64) return fail(SDV2_E_SHAPE, "window must be in 1..64");
    if (!(m->sigma > 0.0) || !(m->lambda > 0.0) || !(m->lambda <= 1.0))
        return fail(SDV2_E_ARG, "need sigma > 0 and 0 < lambda <= 1");
    if (!std::isfinite(m->s_min) || !std::isfinite(m->s_max) || !std::isfinite(m->s_init))
        return fail(SDV2_E_ARG, "noise-rate bounds must be finite");
    return SDV2_OK;
}

static void motion_layout(const sdv2_motion_config &m, sdv2_motion *h) {
    h->frame_elems = static_cast<int64_t>(m.channels) * m.height * m.width;
    h->n_blocks = static_cast<int>((h->frame_elems + kMotionBlockElems - 1) / kMotionBlockElems);
    uint64_t off = 0;
    h->off_prev = off;
    off = align_up(off + 4ull * m.batch * h->frame_elems, 256);
    h->off_has_prev = off;
    off = align_up(off + 4ull * m.batch, 256);
    h->off_hist = off;
    off = align_up(off + 8ull * m.batch * m.window, 256);
    h->off_hist_len = off;
    off = align_up(off + 4ull * m.batch, 256);
    h->off_hist_pos = off;
    off = align_up(off + 4ull * m.batch, 256);
    h->off_rate = off;
    off = align_up(off + 8ull * m.batch, 256);
    h->off_status = off;
    off = align_up(off + 4, 256);
    h->off_partial = off;
    off = align_up(off + 8ull * m.batch * m.chunk_frames * h->n_blocks, 256);
    h->off_counter = off;
    off = align_up(off + 4ull * m.batch, 256);
    h->total = off;
}

size_t sdv2_motion_bytes(const sdv2_motion_config *cfg) {
    if (check_motion(cfg) != SDV2_OK) return 0;
    sdv2_motion h{};
    motion_layout(*cfg, &h);
    return static_cast<size_t>(h.total);
}

sdv2_status sdv2_motion_create(const sdv2_motion_config *cfg, void *dev_buf, size_t bytes, sdv2_motion **out) {
    if (!out) return fail(SDV2_E_ARG, "out is NULL");
    *out = nullptr;
    sdv2_status st = check_motion(cfg);
    if (st != SDV2_OK) return st;
    if (!dev_buf) return fail(SDV2_E_ARG, "dev_buf is NULL");
    if ((reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) return fail(SDV2_E_ALIGN, "dev_buf must be 256-byte aligned");
    sdv2_motion *h = new sdv2_motion();
    h->cfg = *cfg;
    motion_layout(*cfg, h);
    if (bytes < h->total) {
        const unsigned long long need = h->total;
        delete h;
        return fail(SDV2_E_ALIGN, "buffer of %zu bytes is smaller than the %llu bytes required", bytes, need);
    }
    h->base = static_cast<uint8_t *>(dev_buf);
    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess) e = cudaMemset(dev_buf, 0, h->total);
    std::vector<double> rate(cfg->batch, cfg->s_init);
    if (e == cudaSuccess) e = cudaMemcpy(h->base + h->off_rate, rate.data(), 8ull * cfg->batch, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "motion_create");
    }
    *out = h;
    return SDV2_OK;
}

sdv2_status sdv2_motion_destroy(sdv2_motion *m) {
    delete m;
    return SDV2_OK;
}

sdv2_status sdv2_motion_noise_rate(sdv2_motion *m, const float *latents, float *out_rate_dev, float *out_d_dev,
                                   sdv2_stream stream) {
    if (!m || !latents || !out_rate_dev) return fail(SDV2_E_ARG, "NULL argument");
    if (!aligned16(latents) || (reinterpret_cast<uintptr_t>(out_rate_dev) & 3u) ||
        (reinterpret_cast<uintptr_t>(out_d_dev) & 3u))
        return fail(SDV2_E_ALIGN, "latents must be 16-byte aligned, outputs 4-byte aligned");
    sdv2_status st = check_device(m->device);
    if (st != SDV2_OK) return st;
    MotionParams p;
    std::memset(&p, 0, sizeof(p));
    p.latents = latents;
    p.prev = reinterpret_cast<float *>(m->base + m->off_prev);
    p.has_prev = reinterpret_cast<int32_t *>(m->base + m->off_has_prev);
    p.hist = reinterpret_cast<double *>(m->base + m->off_hist);
    p.hist_len = reinterpret_cast<int32_t *>(m->base + m->off_hist_len);
    p.hist_pos = reinterpret_cast<int32_t *>(m->base + m->off_hist_pos);
    p.rate = reinterpret_cast<double *>(m->base + m->off_rate);
    p.partial = reinterpret_cast<double *>(m->base + m->off_partial);
    p.counter = reinterpret_cast<uint32_t *>(m->base + m->off_counter);
    p.out_rate = out_rate_dev;
    p.out_d = out_d_dev;
    p.frame_elems = m->frame_elems;
    p.batch = m->cfg.batch;
    p.chunk_frames = m->cfg.chunk_frames;
    p.window = m->cfg.window;
    p.n_blocks = m->n_blocks;
    p.sigma = m->cfg.sigma;
    p.lambda = m->cfg.lambda;
    p.s_min = m->cfg.s_min;
    p.s_max = m->cfg.s_max;
    cudaError_t e = launch_motion(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "motion launch");
    g_launches.fetch_add(1);
    return SDV2_OK;
}

sdv2_status sdv2_motion_check(sdv2_motion *m) {
    if (!m) return fail(SDV2_E_ARG, "motion is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "motion_check");
    uint32_t word = 0;
    e = cudaMemcpy(&word, m->base + m->off_status, 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "motion_check");
    if (word != 0) return fail(SDV2_E_DEVICE, "device status 0x%x", word);
    return SDV2_OK;
}

sdv2_status sdv2_motion_noise_rate_noalloc(sdv2_motion *m, const float *latents, float *out_rate_dev,
                                           float *out_d_dev, sdv2_stream stream) {
    if (!m || !latents || !out_rate_dev) return fail(SDV2_E_ARG, "NULL argument");
    if (!aligned16(latents) || (reinterpret_cast<uintptr_t>(out_rate_dev) & 3u) ||
        (reinterpret_cast<uintptr_t>(out_d_dev) & 3u))
        return fail(SDV2_E_ALIGN, "latents must be 16-byte aligned, outputs 4-byte aligned");
    const int64_t partials = static_cast<int64_t>(m->cfg.batch) * m->cfg.chunk_frames * m->n_blocks;
    if (partials > motion_noalloc_max_partials())
        return fail(SDV2_E_SHAPE,
                    "batch * chunk_frames * ceil(C*H*W / %d) = %lld exceeds the %d partial sums of the "
                    "library's fixed scratch; use sdv2_motion_noise_rate",
                    kMotionBlockElems, static_cast<long long>(partials), motion_noalloc_max_partials());
    sdv2_status st = check_device(m->device);
    if (st != SDV2_OK) return st;
    MotionParams p;
    std::memset(&p, 0, sizeof(p));
    p.latents = latents;
    p.prev = reinterpret_cast<float *>(m->base + m->off_prev);
    p.has_prev = reinterpret_cast<int32_t *>(m->base + m->off_has_prev);
    p.hist = reinterpret_cast<double *>(m->base + m->off_hist);
    p.hist_len = reinterpret_cast<int32_t *>(m->base + m->off_hist_len);
    p.hist_pos = reinterpret_cast<int32_t *>(m->base + m->off_hist_pos);
    p.rate = reinterpret_cast<double *>(m->base + m->off_rate);
    p.out_rate = out_rate_dev;
    p.out_d = out_d_dev;
    p.frame_elems = m->frame_elems;
    p.batch = m->cfg.batch;
    p.chunk_frames = m->cfg.chunk_frames;
    p.window = m->cfg.window;
    p.n_blocks = m->n_blocks;
    p.sigma = m->cfg.sigma;
    p.lambda = m->cfg.lambda;
    p.s_min = m->cfg.s_min;
    p.s_max = m->cfg.s_max;
    cudaError_t e = launch_motion_noalloc(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "motion (no-alloc) launch");
    g_launches.fetch_add(1);
    return SDV2_OK;
}

// ------------------------------------------------------------------ host-only helpers

int32_t sdv2_slot_of_frame(int64_t f, int32_t sink_frames, int32_t window_frames) {
    if (sink_frames < 1 || window_frames < 1) return -1;
    return slot_of(f, sink_frames, window_frames);
}

int64_t sdv2_rope_phase(int64_t f, int32_t rope_reset_period) { return phase_of(f, rope_reset_period); }

void sdv2_valid_slots(int64_t frame_end, int32_t sink_frames, int32_t window_frames, int32_t *sink_valid,
                      int32_t *window_valid) {
    int32_t sv = 0, wv = 0;
    valid_counts(frame_end, sink_frames, window_frames, &sv, &wv);
    if (sink_valid) *sink_valid = sv;
    if (window_valid) *window_valid = wv;
}

int32_t sdv2_attention_pair_mode(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count) {
    sdv2_cache_config n;
    if (check_config(cfg, &n) != SDV2_OK || !keys) return -1;
    const Geometry g = geometry(n);
    int64_t active = 0;
    for (int b = 0; b < std::min(n.batch, kMaxBatch); ++b)
        if (keys[b] > 0) ++active;
    return use_pair_mode(g, n, active * n.heads * g.n_qpairs, sm_count) ? 1 : 0;
}

int32_t sdv2_append_attention_mode(const sdv2_cache_config *cfg, const int64_t *chunk_first_frame, int32_t sm_count) {
    sdv2_cache_config n;
    if (check_config(cfg, &n) != SDV2_OK || !chunk_first_frame) return -1;
    return fuse_mode(n, geometry(n), chunk_first_frame, sm_count);
}

int32_t sdv2_attention_splits(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count) {
    int32_t whole = 0, pieces = 0;
    if (sdv2_attention_plan(cfg, keys, sm_count, &whole, &pieces) != SDV2_OK) return -1;
    return pieces;
}

sdv2_status sdv2_attention_plan(const sdv2_cache_config *cfg, const int64_t *keys, int32_t sm_count,
                                int32_t *whole_units, int32_t *pieces) {
    sdv2_cache_config n;
    if (!keys || !whole_units || !pieces) return fail(SDV2_E_ARG, "NULL argument");
    sdv2_status st = check_config(cfg, &n);
    if (st != SDV2_OK) return st;
    const Geometry g = geometry(n);
    int active = 0;
    for (int b = 0; b < std::min(n.batch, kMaxBatch); ++b)
        if (keys[b] > 0) ++active;
    const int64_t units = static_cast<int64_t>(active) * n.heads * g.n_qpairs;
    if (use_pair_mode(g, n, units, sm_count)) {     // pair mode: every unit whole
        *whole_units = static_cast<int32_t>(units);
        *pieces = 1;
        return SDV2_OK;
    }
    const AttnPlan plan = plan_attention(n, g, units, max_kv_tiles(g, keys, std::min(n.batch, kMaxBatch)), sm_count);
    *whole_units = static_cast<int32_t>(plan.whole);
    *pieces = plan.pieces;
    return SDV2_OK;
}

uint64_t sdv2_launch_count(void) { return g_launches.load(); }

const char *sdv2_last_error(void) { return g_err.c_str(); }

const char *sdv2_version(void) { return "sdv2 0.1.0 (sm_100a)"; }

}  // extern "C"

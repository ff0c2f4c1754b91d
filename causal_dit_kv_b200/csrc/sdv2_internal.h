// Internal declarations shared by the host library (host.cpp) and the
// kernel translation units.  Nothing here is part of the public C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>

#include <cuda.h>           // CUtensorMap (type only; the driver is reached at run time)
#include <cuda_runtime.h>

namespace sdv2 {

constexpr int kMaxBatch = 64;
// fp64 (cos, sin) entries of the temporal axis carried in one append launch.
constexpr int kAppendTabEntries = 256;    // 4 KB of kernel parameters (rows of distinct phases)
constexpr int kAppendMaxFrames = 64;
// fp32 (cos, sin) entries of the temporal axis that one attention CTA keeps in shared
// memory: n_t pairs for each chunk frame its (up to 256) query rows span.
constexpr int kAttnTabEntries = 128;
constexpr int kMaxSplits = 16;                // KV pieces of one split unit, at most
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits give up after 2 s

// Device status word bits (set with atomicOr, never cleared by kernels).
enum : uint32_t {
    kStatusTmaWait = 1u << 0,
    kStatusMmaWait = 1u << 1,
    kStatusSoftmaxWait = 1u << 2,
    kStatusBadArgs = 1u << 3,
    kStatusSelfTest = 1u << 4,
};

struct AppendParams {
    const uint16_t *k_in;       // [B][T'N][H][d]
    const uint16_t *v_in;
    uint16_t *k_layer;          // [B][slots][N][H][d] of this layer
    uint16_t *v_layer;
    const double *rope_h;       // [frame_h][n_h][2] fp64 (cos, sin)
    const double *rope_w;       // [frame_w][n_w][2]
    int64_t frame_elems;        // N*H*d
    int32_t chunk_tokens;       // T'N
    int32_t heads, head_dim, frame_w, n_t, n_h, n_w, slots;
    int32_t n_frames;           // frames handled by this launch
    int32_t src_b[kAppendMaxFrames];     // stream of each frame
    int32_t src_i[kAppendMaxFrames];     // index of the frame in the chunk
    int32_t dst_slot[kAppendMaxFrames];  // ring slot it goes to
    uint8_t tab_row[kAppendMaxFrames];   // row of tab_t with the frame's phase
    double tab_t[kAppendTabEntries][2];  // [distinct phase][n_t] temporal cos, sin
    // fp8 (E4M3) cache only: codes and per-(slot, head, 128-token block) scales of this layer
    uint8_t *k8_layer;          // [B][slots][Np][H][d]
    uint8_t *v8t_layer;         // [B][slots][H][d][Np]
    float *k_scale_layer;       // [B][slots][scale_slot_stride] (head h, block j at h * n_blk + j)
    float *v_scale_layer;
    int32_t tokens, np_tokens, n_blk, scale_slot_stride;
};

struct AttnParams {
    uint16_t *out;              // [B][Lq][H][d]
    float *part_o;              // [piece][split unit][d/4][256] float4 (split units only)
    float *part_ml;             // [piece][split unit][256] float2 (row max in log2 units, row sum)
    const float *rope_h;        // [n_h][frame_h][2] fp32, pair-major
    const float *rope_w;        // [n_w][frame_w][2]
    uint32_t *status;
    int32_t batch, heads, lq, tokens_per_frame, frame_h, frame_w, chunk_frames;
    int32_t n_t, n_h, n_w;
    int32_t n_qpairs, b_offset;
    // Work units u = (i * heads + h) * n_qpairs + qpair over the launch's active streams
    // unit_stream[i]: units [0, n_whole) run whole, one CTA each; units [n_whole,
    // n_units) are split over the KV range into n_pieces CTAs each and merged by
    // attention_combine_kernel.
    int32_t n_units, n_whole, n_pieces;
    // 1: pair mode (chunks of one query tile, nothing split): CTA x takes heads 2k and
    // 2k + 1 of stream unit_stream[x / ceil(H / 2)], one accumulator set and query tile each
    int32_t pair;
    uint8_t unit_stream[kMaxBatch];
    float scale_log2;           // softmax_scale * log2(e)
    int32_t lk[kMaxBatch];      // valid keys per stream of this launch (0 = skip)
    const double *omega_t;      // [n_t] temporal frequencies base^(-j / n_t), fp64 (in the cache buffer)
    int32_t rope_reset;         // temporal phase period (0: none)
    int64_t f0[kMaxBatch];      // first frame of each stream's chunk
    // fp8 (E4M3) cache only: KV tiles are 128-token blocks of one slot (slot s, block j at
    // tile s * n_blk + j), each with its own K and V scale; the kernel rounds each rotated
    // query row to E4M3 with its own scale
    const float *k_scale;       // this layer: [B][slots][scale_slot_stride]
    const float *v_scale;
    int32_t slots, np_tokens, n_blk, scale_slot_stride;
    int32_t f8;                 // 1: fp8 cache (E4M3 queries, keys, values and probabilities)
    // fp8 with 64-token slots: tile g packs slots 2g and 2g + 1 (64 keys each, the second
    // absent past the valid slots), so no padding token is read; the K map's boxes are 64
    // rows, the V map's 64 keys (64-byte swizzle)
    int32_t pack2;
};

// Append fused into the attention (bf16 cache, chunks of at most two query tiles):
// the CTA that reads a KV tile holding rows of the chunk's own frames brings those rows
// from the caller's k / v into the tile instead (by TMA, or row by row where an 8-row
// group straddles slots), rotates the keys there by the append's rule and writes the
// rows to their ring slots (keys from the rotating threads' registers, values copied
// from v); the tile's other rows come from the cache.  Such
// "assembled" tiles go first in each CTA's tile order; every other tile comes by TMA as
// in the plain attention.
constexpr int kFuseMaxFrames = 4;          // chunk frames, at most
constexpr int kFuseMaxAsmTiles = 2;        // assembled KV tiles of one stream, at most
constexpr int kFuseTabSmem = 48;           // fp64 temporal (cos, sin) entries a CTA keeps: T' * n_t, at most
// fp64 row and column tables a CTA keeps, (frame_h n_h + frame_w n_w) 16 B, at most: one
// KV tile's shared memory (128 x head_dim bf16) less 1 KB for the temporal entries
constexpr int fuse_tab_hw_bytes(int head_dim) { return 256 * head_dim - 1024; }
constexpr int kFusePhaseCap = 4096;        // temporal phases in the cache's fp64 (cos, sin) table for the fused append

constexpr int kFuseBoxes = 4;              // TMA box heights of the fused append: 64, 32, 16, 8 rows

struct FuseParams {
    // this layer's K and V, and the caller's k and v as (d, H, T'N, B), as tensor maps in
    // boxes of 64 channels x (64 >> i) rows: runs of whole 8-row groups of an assembled tile
    // move by TMA in a few boxes each
    CUtensorMap tmap_kc[kFuseBoxes];
    CUtensorMap tmap_vc[kFuseBoxes];
    CUtensorMap tmap_ki[kFuseBoxes];
    CUtensorMap tmap_vi[kFuseBoxes];
    const uint16_t *k_in;       // [B][T'N][H][d] (caller's, un-rotated)
    const uint16_t *v_in;
    uint16_t *k_layer;          // [B][slots][N][H][d] of this layer
    uint16_t *v_layer;
    const double *rope_h;       // [frame_h][n_h][2] fp64 (cos, sin)
    const double *rope_w;       // [frame_w][n_w][2]
    const double *rope_t;       // [phase][n_t][2] fp64 (cos, sin) of the temporal pairs (phases < kFusePhaseCap)
    int32_t slots;
    int32_t new_slot[kMaxBatch][kFuseMaxFrames];       // ring slot of chunk frame i of each stream
    int32_t phase[kMaxBatch][kFuseMaxFrames];          // temporal phase of chunk frame i of each stream
    int32_t asm_tile[kMaxBatch][kFuseMaxAsmTiles];     // KV tiles holding the chunk's rows (-1: none), ascending
    // 8-row groups of those tiles (bit q: rows 8q .. 8q + 7) that hold the chunk's rows:
    // full = all eight are consecutive tokens of one chunk frame (TMA in, keys rotated in
    // place, TMA out); part = the others (built row by row)
    uint32_t grp_full[kMaxBatch][kFuseMaxAsmTiles];
    uint32_t grp_part[kMaxBatch][kFuseMaxAsmTiles];
};

// The non-fused attention instantiations take this in place of FuseParams.
struct FuseNone {
    int32_t unused;
};

struct RefreshParams {
    const uint16_t *hidden;     // [B][Lq][D]
    double *partial;            // scratch [B][row_chunks][D]: column sums of each token chunk
    uint32_t *counter;          // scratch: [kMaxBatch] per-stream tickets, then [B][kRefreshMaxColBlocks] per column block
    double *sink_embed;         // [B][S][D]
    int64_t *sink_frame;        // [B][S]
    int32_t *out_slot;          // [B] (caller's)
    // Regions copied slot to slot on a refresh (bf16 cache: K, V; fp8 cache: K, V codes and
    // their scales); region r of stream b, slot s, layer l starts at
    // copy_base[r] + l * copy_layer_bytes[r] + (b * slots + s) * copy_slot_bytes[r].
    uint8_t *copy_base[4];
    int64_t copy_layer_bytes[4];
    int64_t copy_slot_bytes[4]; // multiples of 16
    int32_t n_copy;
    int32_t batch, lq, dim, sinks, slots, layers, row_chunks;
    double tau;
    int32_t active[kMaxBatch];  // 1 if stream takes part in this call
    int32_t fill_first[kMaxBatch];  // first sink slot this chunk fills itself (-1 none)
    int32_t fill_count[kMaxBatch];  // number of sink slots it fills
    int32_t last_slot[kMaxBatch];   // ring slot of the chunk's last frame
    int64_t last_frame[kMaxBatch];  // frame index of the chunk's last frame
};

struct MotionParams {
    const float *latents;       // [B][T'][CHW]
    float *prev;                // [B][CHW] state: last frame seen
    int32_t *has_prev;          // [B]
    double *hist;               // [B][window] ring of motion values
    int32_t *hist_len;          // [B]
    int32_t *hist_pos;          // [B]
    double *rate;               // [B]
    double *partial;            // scratch [B][T'][n_blocks]
    uint32_t *counter;          // scratch: [kMaxBatch] per-stream tickets, then [B][kRefreshMaxColBlocks] per column block
    float *out_rate;            // [B]
    float *out_d;               // [B][T'] or null
    int64_t frame_elems;        // CHW
    int32_t batch, chunk_frames, window, n_blocks;
    double sigma, lambda, s_min, s_max;
};

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it calls grid_dependency_wait()
// before touching anything that kernel may write.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launchers (defined next to their kernels).  Each returns the CUDA error
// of the launch; the host layer turns it into an sdv2_status.
cudaError_t launch_append(const AppendParams &p, int sm_count, cudaStream_t s);
cudaError_t launch_wait_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t s);
// Merge of the KV-split partials into out (a dependent launch after the attention kernel).
cudaError_t launch_combine(const AttnParams &p, int head_dim, cudaStream_t s);
// Attention of the launch's streams; tq maps the caller's (un-rotated) bf16 queries as
// (d, H, Lq, B) in boxes of 64 channels x 128 rows, 128-byte swizzle.
cudaError_t launch_attention(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, int head_dim, cudaStream_t s);
// The same launch with the chunk's KV append fused in (bf16 cache, FuseParams above).
cudaError_t launch_append_attention(const AttnParams &p, const FuseParams &f, const CUtensorMap &tq,
                                    const CUtensorMap &tk, const CUtensorMap &tv, int head_dim, cudaStream_t s);
cudaError_t launch_refresh(const RefreshParams &p, int sm_count, cudaStream_t s, int *launches);
cudaError_t launch_motion(const MotionParams &p, cudaStream_t s);
// Same kernel with partial/counter in the library's static device array.
cudaError_t launch_motion_noalloc(MotionParams p, cudaStream_t s);
int motion_noalloc_max_partials();

// Attention tiling shared by host planning and kernels.
constexpr int kBlockM = 128;      // query rows per tile (one TMEM lane each)
constexpr int kBlockN = 128;      // keys per KV tile
constexpr int kQTilesPerCta = 2;  // two query tiles ping-pong over the tensor core
constexpr int kAttnThreads = 384;
int attention_smem_bytes(int head_dim);

constexpr int kRefreshMaxChunks = 32;     // token chunks the chunk-mean reduction is split into, at most
constexpr int kRefreshMaxColBlocks = 64;  // 256-column blocks of the refresh reduction (embed_dim <= 16384)
constexpr int kMotionBlockElems = 2048;   // latent elements per motion block
constexpr int kMotionThreads = 256;
constexpr int kMotionMaxFrames = 64;      // chunk_frames of a motion state, at most

}  // namespace sdv2

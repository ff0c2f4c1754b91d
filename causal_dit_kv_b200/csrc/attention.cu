// Chunk attention over the sink + rolling-window KV cache on the sm_100a
// tensor cores (tcgen05 MMA, accumulators in TMEM, K/V tiles by TMA).
//
// Sources: admirer.cn article on StreamDiffusionV2, "深入分析：內存帶寬約束
// 導致的性能受限" (each chunk loads the long KV cache while computing only on
// the current input); qq8o.cn walkthrough, "Adaptive sink and RoPE refresh"
// (sink tokens, RoPE); agentlens page "chenfengxu714/StreamDiffusionV2"
// (ring-buffer KV cache with sliding-window attention).
//
// out = softmax(scale * RoPE(q) K^T) V over the valid slots of the stream.
// The valid slots are always the prefix 0..n_valid-1 of the ring (sinks fill
// first, window slots after), and attention is invariant to the order of the
// keys, so the kernel reads keys 0..lk-1 of the slot-major cache directly,
// without unrolling the ring.
//
// One CTA = one work unit (stream, head, pair of 128-row query tiles) or one
// KV-range piece of a unit: the host runs as many units whole as fill complete
// waves of the GPU and splits the remaining ones (or all of them, when there
// are fewer units than SMs) over the KV range, so the last wave is not left
// mostly empty.
//   warp 0      TMA producer: K tiles (128 keys x d) into a 2-slot ring, V tiles
//               into a 3-slot ring
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V
//   warps 4..7  softmax + epilogue of query tile 0 (thread i owns row i)
//   warps 8..11 softmax + epilogue of query tile 1
// The producer/MMA warpgroup gives registers to the two softmax warpgroups
// (setmaxnreg 80 / 208).
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1, 128 columns each; P_t (bf16)
// is written over the first 64 columns of S_t and fed to the PV MMA from
// TMEM.  The MMA order PV(0,j), QK(0,j+1), PV(1,j), QK(1,j+1) lets one tile's
// softmax run while the tensor core works on the other tile.
// Online softmax in base 2 with lazy rescaling: the running max only moves
// (and O is rescaled in TMEM) when a tile's max exceeds it by more than 8,
// so P stays <= 256.  The exponent arguments and row sums use packed f32x2
// arithmetic.
// A CTA whose query-tile pair holds a single tile (chunks of <= 128 queries,
// or the last pair of a ragged chunk) runs the same pipeline with both
// accumulator sets on that tile: even KV tiles go to S_0/O_0, odd ones to
// S_1/O_1, so the softmax of one still overlaps the MMAs of the other; the
// two partial results are merged in the epilogue.
// Q: RoPE is applied on load.  The producer TMA-loads the chunk's raw bf16
// query tiles (128-byte-swizzled, the layout the MMA reads) before the kernel
// waits for the KV append it depends on; the softmax warps, idle until the
// first scores arrive, rotate their own rows in place in fp32 (rounded to
// bf16) from a per-CTA table of the temporal (cos, sin), evaluated in fp64 for
// the chunk frames the CTA's rows span, and the cache's fp32 row and column
// tables; they fence the writes for the tensor core and release the first MMA.
// fp8 (E4M3) cache (the F8 instantiation, head_dim 128): the raw queries land in
// a staging area and each rotated row is coded as E4M3 with its own scale
// (amax / 448 over the row) into the Q tile.  KV tiles are the
// 128-token blocks of each valid slot (tile g = block g % n_blk of slot
// g / n_blk, padding tokens masked), V tiles come from the slot's transposed
// codes, and Q, K, P and V enter kind::f8f6f4 MMAs (K = 32 per instruction).
// Slots of 64 tokens are packed two to a tile instead (tile g: slots 2g and
// 2g + 1): K rows 0..63 and 64..127 come from the two slots, and the V tile is
// two 64-byte-swizzled halves, one per slot, read by the PV MMAs as keys 0..63
// and 64..127.  Each tile's (each half's) K scale and the query row's scale
// fold into the softmax scale of its columns; its V scale divided by the CTA's
// largest V scale multiplies P before its E4M3 coding, and the epilogue
// multiplies O back by that largest scale.  P takes columns [0, 32) of S_t.
// KV splits: each split CTA writes its unnormalised O, row max and row sum;
// attention_combine_kernel (a dependent launch) merges them over the whole
// GPU.
// Every wait is bounded (2 s), after which the CTA records an error in the
// device status word and unwinds; TMEM is always released.
#include <cmath>
#include <type_traits>

#include "ptx.cuh"

namespace sdv2 {

template <int D, bool F8 = false, bool FUSE = false>
struct AttnLayout {
    static constexpr int kElem = F8 ? 1 : 2;          // bytes per element of Q, K, V in the MMA tiles
    static constexpr int kQTile = kBlockM * D * kElem;    // bytes of one Q tile
    static constexpr int kKVTile = kBlockN * D * kElem;   // bytes of one K (or V) tile
    static constexpr int kSub = kBlockM * 128;        // one 64-column (128-byte) sub-tile
    static constexpr int kKStages = 2;                // K tile i is needed one half-iteration before V tile i,
    static constexpr int kVStages = 3;                // so V gets the deeper ring to hide its load latency
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQTilesPerCta * kQTile;
    static constexpr int kV = kK + kKStages * kKVTile;
    // raw bf16 query tiles as loaded (fp8: a staging area; bf16: the Q tiles themselves,
    // rotated in place)
    static constexpr int kQRaw = F8 ? kV + kVStages * kKVTile : kQ;
    static constexpr int kQRawTile = kBlockM * D * 2;
    static constexpr int kTab = F8 ? kQRaw + kQTilesPerCta * kQRawTile : kV + kVStages * kKVTile;
    // fused append: fp64 (cos, sin) for the keys (temporal entries of the chunk's frames,
    // then the cache's row table and column table) in V stage 2, which no tile uses before
    // the assembled tiles are built (the producer loads it only after kAsm)
    static constexpr int kTab64 = kV + 2 * kKVTile;
    static constexpr int kTabHW = kTab64 + kFuseTabSmem * 16;
    static_assert(!FUSE || kFuseTabSmem * 16 + fuse_tab_hw_bytes(D) <= kKVTile, "key tables fit V stage 2");
    static constexpr int kBar = kTab + kAttnTabEntries * 8;
    // barriers
    static constexpr int kQFull = 0;                  // raw query tiles landed (TMA)
    static constexpr int kQReady = 1;                 // rotated query tiles written and fenced (softmax threads)
    static constexpr int kKFull = 2;
    static constexpr int kKEmpty = kKFull + kKStages;
    static constexpr int kVFull = kKEmpty + kKStages;
    static constexpr int kVEmpty = kVFull + kVStages;
    static constexpr int kSFull = kVEmpty + kVStages;
    static constexpr int kPFull = kSFull + 2;
    static constexpr int kOFull = kPFull + 2;
    static constexpr int kDrain = kOFull + 2;
    static constexpr int kAsm = kDrain + 1;           // fused append: assembled tiles written (one arrival per warp 2..11)
    static constexpr int kTabReady = kAsm + 1;        // fused append: fp64 key tables in shared memory
    static constexpr int kNumBars = kAsm + (FUSE ? 2 : 0);
    static constexpr int kMisc = kBar + kNumBars * 8;   // tmem base, abort flag, a spare word (zeroed by the fused launch)
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;      // room to align the base to 1024 bytes
    static_assert(kAlloc <= 232448, "shared memory of one CTA");
};

int attention_smem_bytes(int head_dim) {
    return head_dim == 64 ? AttnLayout<64>::kAlloc : AttnLayout<128>::kAlloc;
}

constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale only when the max grows by > 2^8

// All 32 lanes wait; the warp proceeds only if every lane saw the phase
// complete, so the .sync.aligned tcgen05 ops that follow stay warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile uint32_t *abort, uint32_t *status,
                                          uint32_t code) {
    const bool ok = mbar_wait(bar, parity, abort, status, code);
    return __all_sync(0xffffffffu, ok);
}

// Tables of one query row's rotation: the temporal (cos, sin) of its frame in the
// CTA's shared-memory table (tab_t: pair 0), and the cache's pair-major fp32 row
// and column tables ([pair][position]), offset to the row's position (h: prow, w:
// pcol) and to pair 0 of their axis.
struct RopeRow {
    const float2 *tab_t;
    const float2 *h;
    const float2 *w;
    int n_t, n_th, frame_h, frame_w;
};

// (cos, sin) of pair j.  j is the same in every lane at a given step (one thread per
// row): the temporal entry is a broadcast and the lanes' row / column entries
// (consecutive tokens) are consecutive in the pair-major tables.  With the axis
// split known at compile time (NT temporal pairs, NTH temporal + row pairs), j is a
// constant after unrolling and each load goes straight to its table; otherwise
// (NT = 0) the address is selected without a branch, so all of a row's loads can
// still be in flight together.
template <int NT, int NTH>
__device__ __forceinline__ float2 rope_cs(const RopeRow &t, int j) {
    if constexpr (NT > 0) {
        if (j < NT) return t.tab_t[j];
        if (j < NTH) return __ldg(t.h + (j - NT) * t.frame_h);
        return __ldg(t.w + (j - NTH) * t.frame_w);
    } else {
        const float2 *ptr = j < t.n_t ? t.tab_t + j
                                      : (j < t.n_th ? t.h + (j - t.n_t) * t.frame_h : t.w + (j - t.n_th) * t.frame_w);
        return *ptr;
    }
}

// Load one 64-column sub-tile row (8 chunks of 16 bytes at the 128-byte-swizzled
// positions c ^ (r & 7) of the row) and the (cos, sin) of its 32 pairs j0 .. j0 + 31;
// every load is issued before any use.
template <int NT, int NTH>
__device__ __forceinline__ void rope_load(const uint8_t *row, int r, int j0, const RopeRow &t, uint4 (&x)[8],
                                          float2 (&cs)[32]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) x[c] = *reinterpret_cast<const uint4 *>(row + ((c ^ (r & 7)) << 4));
#pragma unroll
    for (int q = 0; q < 32; ++q) cs[q] = rope_cs<NT, NTH>(t, j0 + q);
}

// Pair q of chunk c of a loaded sub-tile row, rotated in fp32.
__device__ __forceinline__ float2 rope_apply(const uint4 (&x)[8], const float2 (&cs)[32], int c, int q) {
    const uint32_t w = q == 0 ? x[c].x : (q == 1 ? x[c].y : (q == 2 ? x[c].z : x[c].w));
    const float x0 = bf16_lo(w), x1 = bf16_hi(w);
    const float2 k = cs[4 * c + q];
    return make_float2(x0 * k.x - x1 * k.y, x0 * k.y + x1 * k.x);
}

// Rotate the 32 pairs of one 64-column sub-tile of row r in place (bf16 in, fp32
// rotation, bf16 out).
template <int NT, int NTH>
__device__ __forceinline__ void rope_subtile_bf16(uint8_t *sub, int r, int j0, const RopeRow &t) {
    uint8_t *row = sub + r * 128;
    uint4 x[8];
    float2 cs[32];
    rope_load<NT, NTH>(row, r, j0, t, x, cs);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 v = rope_apply(x, cs, c, q);
            o[q] = pack_bf16x2(v.x, v.y);
        }
        *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// fp8 cache (head_dim 128): rotate the raw bf16 row r (two 64-column swizzled
// sub-tiles at shared address raw) in fp32, code it as E4M3 with the row's own
// scale amax / 448 into the 128-byte-swizzled E4M3 row of q8 (when `write`), and
// return the scale.  Two passes over the row (the maximum, then the codes), one
// sub-tile at a time, keep the register use low.
template <int NT, int NTH>
__device__ __forceinline__ float rope_row_e4m3(const uint8_t *raw, uint8_t *q8, int r, bool write, const RopeRow &t) {
    float am = 0.0f;
#pragma unroll 1
    for (int kb = 0; kb < 2; ++kb) {
        uint4 x[8];
        float2 cs[32];
        rope_load<NT, NTH>(raw + kb * (kBlockM * 128) + r * 128, r, kb * 32, t, x, cs);
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 v = rope_apply(x, cs, c, q);
                am = fmaxf(am, fmaxf(fabsf(v.x), fabsf(v.y)));
            }
    }
    float scale, inv;
    e4m3_scale_inv(am, scale, inv);
    if (write) {
#pragma unroll 1
        for (int kb = 0; kb < 2; ++kb) {
            uint4 x[8];
            float2 cs[32];
            rope_load<NT, NTH>(raw + kb * (kBlockM * 128) + r * 128, r, kb * 32, t, x, cs);
            // E4M3 chunk e (16 codes, pairs 8e .. 8e + 7) takes raw chunks 2e, 2e + 1 of this sub-tile
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t w[4];
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    const float2 v0 = rope_apply(x, cs, 2 * e + hlf, 0), v1 = rope_apply(x, cs, 2 * e + hlf, 1);
                    const float2 v2 = rope_apply(x, cs, 2 * e + hlf, 2), v3 = rope_apply(x, cs, 2 * e + hlf, 3);
                    w[2 * hlf] = pack_e4m3x2(v0.x * inv, v0.y * inv) | (pack_e4m3x2(v1.x * inv, v1.y * inv) << 16);
                    w[2 * hlf + 1] = pack_e4m3x2(v2.x * inv, v2.y * inv) | (pack_e4m3x2(v3.x * inv, v3.y * inv) << 16);
                }
                const int cq = kb * 4 + e;              // E4M3 chunk of the 128-byte row
                *reinterpret_cast<uint4 *>(q8 + r * 128 + ((cq ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    return scale;
}

// P = 2^(s*scale_log2 - m) for one row of 128 scores (raw fp32 bits in sr),
// packed to bf16 into TMEM columns [0, 64) of the row's S region; returns
// the row sum (fp32).  Exponentials on the MUFU ex2; pairs of columns share
// one f32x2 FMA for the exponent argument and one f32x2 add for the sum.
__device__ __forceinline__ float softmax_exp_store(const uint32_t (&sr)[kBlockN / 32][32], float scale_log2,
                                                   float neg_m, uint32_t s_tmem) {
    const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
    const uint64_t negm2 = f2_pack(neg_m, neg_m);
    uint64_t acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0ull;
#pragma unroll
    for (int cb = 0; cb < kBlockN / 32; ++cb) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[cb][2 * i]), __uint_as_float(sr[cb][2 * i + 1])),
                                      scale2, negm2);
            float x0, x1, p0, p1;
            f2_unpack(x, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
            pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(s_tmem + cb * 16, pk);
    }
    float a0, a1;
    f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
    return a0 + a1;
}

// fp8 cache: P = 2^(s*c - m) as above, the row sum from P, and P * r coded as
// E4M3 (four keys per 32-bit TMEM column, key order in the bytes) into columns
// [0, 32) of the row's S region; r = (this tile's V scale) / (the CTA's
// largest V scale) folds the tile's V scale into P, so one O accumulates
// tiles of different scales.
template <bool PK>
__device__ __forceinline__ float softmax_exp_store_f8(const uint32_t (&sr)[kBlockN / 32][32], float c, float neg_m,
                                                      float r, float r_hi, uint32_t s_tmem) {
    const uint64_t scale2 = f2_pack(c, c);
    const uint64_t negm2 = f2_pack(neg_m, neg_m);
    const uint64_t zero2 = f2_pack(0.0f, 0.0f);
    uint64_t acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0ull;
#pragma unroll
    for (int cb = 0; cb < kBlockN / 32; ++cb) {
        // columns 64 .. 127 at their own V ratio (a tile of two 64-token slots)
        const float rc = PK && cb >= kBlockN / 64 ? r_hi : r;
        const uint64_t r2 = f2_pack(rc, rc);
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[cb][2 * i]), __uint_as_float(sr[cb][2 * i + 1])),
                                      scale2, negm2);
            float x0, x1;
            f2_unpack(x, x0, x1);
            const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
            acc[i & 3] = f2_add(acc[i & 3], pp);
            float q0, q1;
            f2_unpack(f2_fma(pp, r2, zero2), q0, q1);
            const uint32_t h16 = pack_e4m3x2(q0, q1);
            if (i & 1)
                pk[i >> 1] |= h16 << 16;
            else
                pk[i >> 1] = h16;
        }
        tmem_st8(s_tmem + cb * 8, pk);
    }
    float a0, a1;
    f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
    return a0 + a1;
}

// Single-tile mode: 32 columns of w0 O_0 + w1 O_1 for this thread's row, as
// fp32 bits in r0 (O_1 is read only if its set received keys).
__device__ __forceinline__ void merge_sets(uint32_t o0, uint32_t o1, bool has1, float w0, float w1,
                                           uint32_t (&r0)[32]) {
    uint32_t r1[32];
    tmem_ld32(o0, r0);
    if (has1) {
        tmem_ld32(o1, r1);
        tmem_wait_ld_bind(r0);
        reg_bind(r1);
    } else {
        tmem_wait_ld_bind(r0);
#pragma unroll
        for (int i = 0; i < 32; ++i) r1[i] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) r0[i] = __float_as_uint(w0 * __uint_as_float(r0[i]) + w1 * __uint_as_float(r1[i]));
}

// Fused append: TMA loads of the 8-row groups `groups` of an assembled tile (bit q: rows
// 8q .. 8q + 7), as runs: consecutive groups whose rows are consecutive in the tensor go
// together, each run in boxes of 64, 32, 16, 8 rows, largest first (maps[i]: boxes of
// 64 >> i rows x 64 channels; row_of(q): the tensor row of group q's first row).  A box
// of rows starting at tile row 8q lands at byte 1024 q of each 128-byte-swizzled sub-tile
// of the tile at dst, where a whole-tile load puts those rows.
template <int D, typename L, typename RowOf>
__device__ __forceinline__ void load_row_groups(uint8_t *dst, const CUtensorMap *maps, uint64_t *bar, uint32_t groups,
                                                int hh, int bg, RowOf row_of) {
    int q = 0;
    while (q < 16) {
        if (!((groups >> q) & 1u)) {
            ++q;
            continue;
        }
        const int row0 = row_of(q);
        int e = q + 1;                                // the run: groups q .. e - 1
        while (e < 16 && ((groups >> e) & 1u) && row_of(e) == row0 + 8 * (e - q)) ++e;
        for (int g = q; g < e;) {
            const int left = e - g;                   // groups left in the run
            const int i = left >= 8 ? 0 : (left >= 4 ? 1 : (left >= 2 ? 2 : 3));
            const int row = row0 + 8 * (g - q);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
                tma_load_4d(dst + kb * L::kSub + g * 1024, &maps[i], bar, kb * 64, hh, row, bg);
            g += 8 >> i;
        }
        q = e;
    }
}

// Fused append, the rows of the assembled tiles that straddle slots (the "part" 8-row
// groups mp0, mp1 of tiles g0, g1; rare: only where a slot boundary is not a multiple of
// 8 rows).  They are cut into slots of kRowsPerIter rows, dealt round-robin to warps
// 2 .. 11 (wi = warp - 2); in a slot kLanes lanes share a row and lane c takes pairs c,
// c + kLanes, c + 2 kLanes, c + 3 kLanes (one 32-bit word of K and of V each), so a
// row's loads are contiguous words and neighbouring lanes read neighbouring entries of
// the shared-memory tables (no bank conflicts).  A warp issues the loads of up to kBatch
// slots at once, then rotates and stores them.  A row of one of the chunk's frames is
// read from the caller's k / v (keys rotated pair by pair with the append's fp64 rule),
// written to its ring slot and to the tile; another valid row is read from the cache;
// rows past the valid prefix are zero (masked, and finite under the zero
// probabilities).  Words land at the 128-byte-swizzled positions a TMA load gives them.
template <int D, typename L>
__device__ __forceinline__ void build_part_groups(uint8_t *smem, uint64_t *bars, const AttnParams &p,
                                                  const FuseParams &f, int bg, int lk, int h, int h_pair, bool paired,
                                                  int g0, int g1, uint32_t mp0, uint32_t mp1,
                                                  const int (&ns)[kFuseMaxFrames], int wi, int lane,
                                                  volatile uint32_t *abort_flag, bool &have_tab) {
    constexpr int kLanes = D / 8;                     // lanes per row (4 pairs each)
    constexpr int kRowsPerIter = 32 / kLanes;         // rows of one slot
    constexpr int kIters = 8 / kRowsPerIter;          // slots of an 8-row group
    constexpr int kWarps = (kAttnThreads - 64) / 32;  // warps 2 .. 11
    constexpr int kBatch = 4;                         // slots of one warp whose loads are in flight together
    const int c0 = __popc(mp0);
    const int n_slots = kIters * (c0 + __popc(mp1));
    if (wi >= n_slots) return;
    const int c = lane % kLanes;
    const int rr = lane / kLanes;
    const int N = p.tokens_per_frame;
    const int n_t = p.n_t, n_th = p.n_t + p.n_h, n_h = p.n_h, n_w = p.n_w, fw = p.frame_w;
    const int64_t row_elems = static_cast<int64_t>(p.heads) * D;
    const int64_t cache_row0 = static_cast<int64_t>(bg) * f.slots * N;   // first key row of this stream
    const int64_t in_row0 = static_cast<int64_t>(bg) * p.lq;
    const double2 *tab_t = reinterpret_cast<const double2 *>(smem + L::kTab64);
    const double2 *tab_h = reinterpret_cast<const double2 *>(smem + L::kTabHW);
    const double2 *tab_w = tab_h + p.frame_h * n_h;
    for (int s0 = wi; s0 < n_slots; s0 += kWarps * kBatch) {
        uint32_t xk[kBatch][4], xv[kBatch][4];
        int fi[kBatch], nn[kBatch], rw[kBatch];       // chunk frame (-1: not the chunk's, -2: no slot); token; tile row | tile << 8
        int64_t dst[kBatch];                          // element offset of this lane's row in the layer (pair 0)
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int s = s0 + b * kWarps;
            fi[b] = -2;
            nn[b] = 0;
            rw[b] = 0;
            dst[b] = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) xk[b][q] = xv[b][q] = 0u;
            if (s < n_slots) {
                const int a = s < kIters * c0 ? 0 : 1;
                const int sa = a ? s - kIters * c0 : s;
                uint32_t m = a ? mp1 : mp0;
                for (int k = sa / kIters; k > 0; --k) m &= m - 1u;
                const int r = (__ffs(m) - 1) * 8 + (sa % kIters) * kRowsPerIter + rr;
                const int kr = (a ? g1 : g0) * kBlockN + r;
                const int hs = paired && a == 1 ? h_pair : h;
                rw[b] = r | (a << 8);
                fi[b] = -1;
                if (kr < lk) {
                    const int sl = kr / N;
                    const int n = kr - sl * N;
#pragma unroll
                    for (int i = 0; i < kFuseMaxFrames; ++i)
                        if (ns[i] == sl) fi[b] = i;
                    nn[b] = n;
                    dst[b] = (cache_row0 + kr) * row_elems + hs * D;
                    const int64_t src =
                        fi[b] >= 0 ? (in_row0 + static_cast<int64_t>(fi[b]) * N + n) * row_elems + hs * D : dst[b];
                    const uint32_t *ks = reinterpret_cast<const uint32_t *>((fi[b] >= 0 ? f.k_in : f.k_layer) + src);
                    const uint32_t *vs = reinterpret_cast<const uint32_t *>((fi[b] >= 0 ? f.v_in : f.v_layer) + src);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        xk[b][q] = ld_nc_u32(ks + c + kLanes * q);
                        xv[b][q] = ld_nc_u32(vs + c + kLanes * q);
                    }
                }
            }
        }
        if (!have_tab) {                              // the key tables, once
            have_tab = warp_wait(&bars[L::kTabReady], 0, abort_flag, p.status, kStatusSoftmaxWait);
            if (!have_tab) return;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (fi[b] == -2) continue;
            const int r = rw[b] & 0xFF, a = rw[b] >> 8;
            uint8_t *krow = smem + L::kK + a * L::kKVTile + r * 128;
            uint8_t *vrow = smem + L::kV + a * L::kKVTile + r * 128;
            const int prow = nn[b] / fw;
            const int pcol = nn[b] - prow * fw;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = c + kLanes * q;         // pair: dims 2j, 2j + 1
                uint32_t wk = xk[b][q];
                if (fi[b] >= 0) {
                    const double2 cs = j < n_t ? tab_t[fi[b] * n_t + j]
                                               : (j < n_th ? tab_h[prow * n_h + (j - n_t)] : tab_w[pcol * n_w + (j - n_th)]);
                    wk = rotate_pair(wk, cs.x, cs.y);
                    reinterpret_cast<uint32_t *>(f.k_layer + dst[b])[j] = wk;
                    reinterpret_cast<uint32_t *>(f.v_layer + dst[b])[j] = xv[b][q];
                }
                // 128-byte-swizzled position of pair j: sub-tile j / 32, 16-byte chunk (j % 32) / 4
                const int off = (j >> 5) * L::kSub + ((((j & 31) >> 2) ^ (r & 7)) << 4) + ((j & 3) << 2);
                *reinterpret_cast<uint32_t *>(krow + off) = wk;
                *reinterpret_cast<uint32_t *>(vrow + off) = xv[b][q];
            }
        }
    }
}

// Fused append, the "full" 8-row groups mf0, mf1 of the assembled tiles (eight
// consecutive tokens of one chunk frame each): their un-rotated keys and values came by
// TMA from the caller's k / v into the tiles; once a tile's key loads have landed (its
// kKFull phase), the keys are rotated in place, pair by pair with the append's fp64
// rule, and written from registers to their ring slots; the values go to their ring
// slots straight from the caller's v (loaded before the wait, so that latency is hidden).
// Rows are dealt round-robin to warps 2 .. 11 in slots of kRowsPerIter rows, kBatch slots
// of a warp at a time; lane c of a row takes pairs c + kLanes q (32-bit words of the
// swizzled row; neighbouring table entries; contiguous global words).
template <int D, typename L>
__device__ __forceinline__ void rotate_full_groups(uint8_t *smem, uint64_t *bars, const AttnParams &p,
                                                   const FuseParams &f, int bg, int h, int h_pair, bool paired, int g0,
                                                   int g1, uint32_t mf0, uint32_t mf1, const int (&ns)[kFuseMaxFrames],
                                                   int wi, int lane, volatile uint32_t *abort_flag, bool &have_tab) {
    constexpr int kLanes = D / 8;
    constexpr int kRowsPerIter = 32 / kLanes;
    constexpr int kIters = 8 / kRowsPerIter;
    constexpr int kWarps = (kAttnThreads - 64) / 32;
    constexpr int kBatch = 4;
    const int c0 = __popc(mf0);
    const int n_slots = kIters * (c0 + __popc(mf1));
    if (wi >= n_slots) return;
    const int c = lane % kLanes;
    const int rr = lane / kLanes;
    const int N = p.tokens_per_frame;
    const int n_t = p.n_t, n_th = p.n_t + p.n_h, n_h = p.n_h, n_w = p.n_w, fw = p.frame_w;
    const int64_t row_elems = static_cast<int64_t>(p.heads) * D;
    const double2 *tab_t = reinterpret_cast<const double2 *>(smem + L::kTab64);
    const double2 *tab_h = reinterpret_cast<const double2 *>(smem + L::kTabHW);
    const double2 *tab_w = tab_h + p.frame_h * n_h;
    uint32_t landed = 0u;                             // tiles whose key loads this warp has seen land
    for (int s0 = wi; s0 < n_slots; s0 += kWarps * kBatch) {
        uint32_t xv[kBatch][4];
        int rw[kBatch], pos[kBatch];                  // tile row | tile << 8 | chunk frame << 12; row, col packed
        int64_t dst[kBatch];                          // element offset of this lane's row in the layer (-1: no slot)
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int s = s0 + b * kWarps;
            dst[b] = -1;
            rw[b] = pos[b] = 0;
            if (s >= n_slots) continue;
            const int a = s < kIters * c0 ? 0 : 1;
            const int sa = a ? s - kIters * c0 : s;
            uint32_t m = a ? mf1 : mf0;
            for (int k = sa / kIters; k > 0; --k) m &= m - 1u;
            const int r = (__ffs(m) - 1) * 8 + (sa % kIters) * kRowsPerIter + rr;
            const int kr = (a ? g1 : g0) * kBlockN + r;
            const int sl = kr / N;
            const int n = kr - sl * N;
            int fi = 0;
#pragma unroll
            for (int i = 0; i < kFuseMaxFrames; ++i)
                if (ns[i] == sl) fi = i;
            const int prow = n / fw;
            const int hs = paired && a == 1 ? h_pair : h;
            rw[b] = r | (a << 8) | (fi << 12);
            pos[b] = (prow << 16) | (n - prow * fw);
            dst[b] = (static_cast<int64_t>(bg) * f.slots * N + kr) * row_elems + hs * D;
            const uint32_t *vs = reinterpret_cast<const uint32_t *>(
                f.v_in + (static_cast<int64_t>(bg) * p.lq + static_cast<int64_t>(fi) * N + n) * row_elems + hs * D);
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[b][q] = ld_nc_u32(vs + c + kLanes * q);
        }
        if (!have_tab) {
            have_tab = warp_wait(&bars[L::kTabReady], 0, abort_flag, p.status, kStatusSoftmaxWait);
            if (!have_tab) return;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (dst[b] < 0) continue;
            const int r = rw[b] & 0xFF, a = (rw[b] >> 8) & 0xF, fi = rw[b] >> 12;
            if (!((landed >> a) & 1u)) {
                if (!warp_wait(&bars[L::kKFull + a], 0, abort_flag, p.status, kStatusSoftmaxWait)) return;
                landed |= 1u << a;
            }
            const int prow = pos[b] >> 16, pcol = pos[b] & 0xFFFF;
            uint8_t *krow = smem + L::kK + a * L::kKVTile + r * 128;
            uint32_t *kdst = reinterpret_cast<uint32_t *>(f.k_layer + dst[b]);
            uint32_t *vdst = reinterpret_cast<uint32_t *>(f.v_layer + dst[b]);
            uint32_t w[4];
            int off[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = c + kLanes * q;
                off[q] = (j >> 5) * L::kSub + ((((j & 31) >> 2) ^ (r & 7)) << 4) + ((j & 3) << 2);
                w[q] = *reinterpret_cast<const uint32_t *>(krow + off[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = c + kLanes * q;
                const double2 cs = j < n_t ? tab_t[fi * n_t + j]
                                           : (j < n_th ? tab_h[prow * n_h + (j - n_t)] : tab_w[pcol * n_w + (j - n_th)]);
                const uint32_t wr = rotate_pair(w[q], cs.x, cs.y);
                *reinterpret_cast<uint32_t *>(krow + off[q]) = wr;
                kdst[j] = wr;
                vdst[j] = xv[b][q];
            }
        }
    }
}

// Fused append: a warp's writes to the assembled tiles are done; fence them for the
// tensor core, then one arrival on kAsm (warps 2 .. 11).
template <typename L>
__device__ __forceinline__ void assembled(uint64_t *bars, int lane) {
    fence_proxy_async_shared();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[L::kAsm]);
}

template <int D, bool F8, bool FUSE, bool PK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    chunk_attention_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                           const __grid_constant__ std::conditional_t<FUSE, FuseParams, FuseNone> f) {
    using L = AttnLayout<D, F8, FUSE>;
    static_assert(!F8 || D == 128, "the fp8 cache is built for head_dim 128");
    static_assert(!(F8 && FUSE), "the fused append is built for the bf16 cache");
    static_assert(!PK || F8, "two slots per KV tile: the fp8 cache's 64-token slots");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // work unit of this CTA: whole units first, then the pieces of the split ones; in the
    // pair mode (single-tile chunks, no split) CTA x takes heads 2k and 2k+1 of one stream
    int unit, split, n_split;
    int h_pair = -1;                            // pair mode: head of accumulator set 1
    if (p.pair) {
        const int hp = (p.heads + 1) >> 1;
        const int k = blockIdx.x % hp;
        unit = (blockIdx.x / hp) * p.heads + 2 * k;   // (n_qpairs == 1)
        if (2 * k + 1 < p.heads) h_pair = 2 * k + 1;
        split = 0;
        n_split = 1;
    } else if (static_cast<int>(blockIdx.x) < p.n_whole) {
        unit = blockIdx.x;
        split = 0;
        n_split = 1;
    } else {
        const int j = blockIdx.x - p.n_whole;
        unit = p.n_whole + j / p.n_pieces;
        split = j - (j / p.n_pieces) * p.n_pieces;
        n_split = p.n_pieces;
    }
    const int su = unit - p.n_whole;            // index among the split units (split CTAs only)
    const int n_su = p.n_units - p.n_whole;
    const int qpair = unit % p.n_qpairs;
    const int h = (unit / p.n_qpairs) % p.heads;
    const int bl = p.unit_stream[unit / (p.n_qpairs * p.heads)];   // stream within this launch
    const int bg = p.b_offset + bl;             // stream index in the cache
    const int lk = p.lk[bl];
    if (lk <= 0) return;                        // (active streams only; uniform per CTA)

    // KV tiles: 128-key runs of the valid prefix (bf16), or the 128-token blocks of each
    // valid slot (fp8: tile g is block g % n_blk of slot g / n_blk; 64-token slots: slots
    // 2g and 2g + 1)
    const int n_vslots = F8 ? lk / p.tokens_per_frame : 0;
    const int n_kv = F8 ? (PK ? (n_vslots + 1) >> 1 : n_vslots * p.n_blk) : (lk + kBlockN - 1) / kBlockN;
    const int per = (n_kv + n_split - 1) / n_split;
    const int kv_begin = split * per;
    const int kv_end = min(n_kv, kv_begin + per);
    const bool paired = h_pair >= 0;            // set t: head (t ? h_pair : h), its own query tile and KV tiles
    // KV tiles of this CTA, in the order the sets take them: in the pair mode both heads'
    // tiles interleaved (even: head h, odd: head h_pair), otherwise this piece's range
    const int n_local = paired ? 2 * n_kv : (kv_end > kv_begin ? kv_end - kv_begin : 0);
    const int q_row0 = qpair * (kBlockM * kQTilesPerCta);
    const int n_qt = paired || (q_row0 + kBlockM < p.lq) ? 2 : 1;
    // the two accumulator sets alternate over the KV tiles when there is one query tile
    // (both sets on that tile, merged at the end) or in the pair mode (one head each)
    const bool alt = n_qt == 1 || paired;
    const bool one_q = n_qt == 1;               // one query tile, two accumulator sets merged in the epilogue
    // Fused append: the KV tiles of this CTA's range that hold the chunk's own rows (a0 < a1;
    // pair mode: the stream's one such tile, for both heads) are assembled in shared memory
    // and taken first; n_asm local tiles (K and V stages 0 .. n_asm - 1) come that way.
    int n_asm = 0, na = 0, a0 = -1, a1 = -1;
    int ns[kFuseMaxFrames];                     // fused append: ring slots of the chunk's frames (-1: none),
    int phs[kFuseMaxFrames];                    // their temporal phases,
    uint32_t mf0 = 0u, mf1 = 0u, mp0 = 0u, mp1 = 0u;   // and the full / part 8-row groups of the assembled tiles
    if constexpr (FUSE) {
        const int t0 = f.asm_tile[bl][0], t1 = f.asm_tile[bl][1];
#pragma unroll
        for (int i = 0; i < kFuseMaxFrames; ++i) {
            ns[i] = i < p.chunk_frames ? f.new_slot[bl][i] : -1;
            phs[i] = i < p.chunk_frames ? f.phase[bl][i] : 0;
        }
        if (paired) {
            a0 = t0;
            na = 1;
            n_asm = 2;
        } else {
            if (t0 >= kv_begin && t0 < kv_end) a0 = t0;
            if (t1 >= kv_begin && t1 < kv_end) (a0 < 0 ? a0 : a1) = t1;
            na = (a0 >= 0) + (a1 >= 0);
            n_asm = na;
        }
        if (n_asm > 0) {
            const int e = a0 == t0 ? 0 : 1;
            mf0 = f.grp_full[bl][e];
            mp0 = f.grp_part[bl][e];
        }
        if (n_asm > 1) {
            mf1 = paired ? mf0 : f.grp_full[bl][1];
            mp1 = paired ? mp0 : f.grp_part[bl][1];
        }
    }
    // KV tile of the i-th position of a head's sequence: the assembled tiles, then the rest
    // of the range in order (the plain attention: the range in order)
    auto tile_at = [&](int i) -> int {
        if constexpr (!FUSE) {
            return kv_begin + i;
        } else {
            if (i < na) return i == 0 ? a0 : a1;
            int g = kv_begin + i - na;
            if (a0 >= 0 && a0 <= g) ++g;
            if (a1 >= 0 && a1 <= g) ++g;
            return g;
        }
    };

    if (threadIdx.x == 0) {
        mbar_init(&bars[L::kQFull], 1);
        mbar_init(&bars[L::kQReady], kAttnThreads - 128);
        for (int s = 0; s < L::kKStages; ++s) {
            mbar_init(&bars[L::kKFull + s], 1);
            mbar_init(&bars[L::kKEmpty + s], 1);
        }
        for (int s = 0; s < L::kVStages; ++s) {
            mbar_init(&bars[L::kVFull + s], 1);
            mbar_init(&bars[L::kVEmpty + s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[L::kSFull + t], 1);
            mbar_init(&bars[L::kPFull + t], kBlockM);
            mbar_init(&bars[L::kOFull + t], 1);
        }
        mbar_init(&bars[L::kDrain], 1);
        if constexpr (FUSE) {
            mbar_init(&bars[L::kAsm], (kAttnThreads - 64) / 32);
            mbar_init(&bars[L::kTabReady], 1);
            *reinterpret_cast<int *>(smem + L::kMisc + 8) = 0;
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if constexpr (FUSE) {
        // the fused append's descriptors (cache and chunk K / V, four box heights each)
        if (warp == 0 && lane < 4 * kFuseBoxes && n_asm > 0) {
            const int i = lane % kFuseBoxes;
            const CUtensorMap *m = lane < kFuseBoxes       ? &f.tmap_kc[i]
                                   : lane < 2 * kFuseBoxes ? &f.tmap_vc[i]
                                   : lane < 3 * kFuseBoxes ? &f.tmap_ki[i]
                                                           : &f.tmap_vi[i];
            tma_prefetch_desc(m);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    __syncwarp();                               // thread 0 took the set-up branches alone
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- queries: raw tiles by TMA, RoPE on load by the softmax warps.  Neither the
    // queries nor the cache's row / column tables are written by the kernels this launch
    // depends on (the KV append), so this overlaps them, before the dependency wait.
    // The fused launch has no append before it: its inputs may come from the kernel just
    // before, so it waits first.
    if constexpr (FUSE) {
        grid_dependency_wait();
        grid_launch_dependents();
    }
    if (warp == 0 && lane == 0 && n_local > 0) {
        mbar_arrive_expect_tx(&bars[L::kQFull], n_qt * L::kQRawTile);
        for (int t = 0; t < n_qt; ++t)
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
                tma_load_4d(smem + L::kQRaw + t * L::kQRawTile + kb * L::kSub, &tmap_q, &bars[L::kQFull], kb * 64,
                            paired && t ? h_pair : h, q_row0 + (paired ? 0 : t * kBlockM), bg);
        if constexpr (FUSE) {
            if (n_asm > 0) {
                // the fp64 tables of the keys the CTA rotates: the temporal (cos, sin) rows of the
                // chunk's phases (T' n_t <= kFuseTabSmem entries), the cache's row and column tables
                const uint32_t tb = static_cast<uint32_t>(p.n_t) * 16u;
                const uint32_t hb = static_cast<uint32_t>(p.frame_h * p.n_h) * 16u;
                const uint32_t wb = static_cast<uint32_t>(p.frame_w * p.n_w) * 16u;   // (checked on the host)
                mbar_arrive_expect_tx(&bars[L::kTabReady], p.chunk_frames * tb + hb + wb);
#pragma unroll
                for (int i = 0; i < kFuseMaxFrames; ++i)
                    if (i < p.chunk_frames)
                        bulk_load(smem + L::kTab64 + i * tb, f.rope_t + static_cast<int64_t>(phs[i]) * p.n_t * 2, tb,
                                  &bars[L::kTabReady]);
                if (hb > 0) bulk_load(smem + L::kTabHW, f.rope_h, hb, &bars[L::kTabReady]);
                if (wb > 0) bulk_load(smem + L::kTabHW + hb, f.rope_w, wb, &bars[L::kTabReady]);
                // the assembled tiles (K and V stages 0 .. n_asm - 1): the cache's rows in the
                // 8-row groups without the chunk's rows, the caller's rows in the full groups
                // (the part groups are built by the CTA's warps)
                const int N = p.tokens_per_frame;
                // every K before any V: the keys are rotated, and the first products taken,
                // before the values are needed
                for (int u = 0; u < 2 * n_asm; ++u) {
                    const bool is_v = u >= n_asm;
                    const int i = is_v ? u - n_asm : u;
                    const int hi = paired && i == 1 ? h_pair : h;
                    const int ti = i == 0 || paired ? a0 : a1;
                    const uint32_t mf = i ? mf1 : mf0, mp = i ? mp1 : mp0;
                    const uint32_t old = ~(mf | mp) & 0xFFFFu;
                    const uint32_t bytes = static_cast<uint32_t>(__popc(old) + __popc(mf)) * 8u * 128u * (D / 64);
                    auto cache_row = [&](int q) { return ti * kBlockN + 8 * q; };
                    auto chunk_token = [&](int q) {           // first row of a full group: its chunk token
                        const int kr = ti * kBlockN + 8 * q, sl = kr / N;
                        int fi = 0;
#pragma unroll
                        for (int e = 0; e < kFuseMaxFrames; ++e)
                            if (ns[e] == sl) fi = e;
                        return fi * N + (kr - sl * N);
                    };
                    uint8_t *tile = smem + (is_v ? L::kV : L::kK) + i * L::kKVTile;
                    uint64_t *bar = &bars[(is_v ? L::kVFull : L::kKFull) + i];
                    mbar_arrive_expect_tx(bar, bytes);
                    load_row_groups<D, L>(tile, is_v ? f.tmap_vc : f.tmap_kc, bar, old, hi, bg, cache_row);
                    load_row_groups<D, L>(tile, is_v ? f.tmap_vi : f.tmap_ki, bar, mf, hi, bg, chunk_token);
                }
            }
        }
    }
    bool have_tab = false;
    // RoPE on load by the softmax warps (idle until the first scores arrive): thread
    // (t, row) rotates its own query row (the single-tile mode: sub-tile t of tile 0's row)
    float q_row_scale = 0.0f;                   // fp8: E4M3 scale of this thread's query row
    if (warp >= 4 && n_local > 0) {
        const int t = (warp - 4) >> 2;
        const int row = ((warp & 3) << 5) + lane;
        const int qt = one_q ? 0 : t;           // query tile of this thread's row
        const int n_rows = min(p.lq - q_row0, alt ? kBlockM : 2 * kBlockM);
        const int fi_lo = q_row0 / p.tokens_per_frame;
        const int fi_hi = (q_row0 + n_rows - 1) / p.tokens_per_frame;
        // temporal (cos, sin) of the chunk frames this CTA's rows span.  The angle
        // phase * base^(-j/n_t) is formed and reduced modulo 2 pi in fp64 (an FMA with
        // the nearest multiple), then sine and cosine are taken in fp32.
        float2 *tab = reinterpret_cast<float2 *>(smem + L::kTab);
        const int n_tab = (fi_hi - fi_lo + 1) * p.n_t;           // <= kAttnTabEntries (checked on the host)
        for (int e = threadIdx.x - 128; e < n_tab; e += kAttnThreads - 128) {
            const int fi = e / p.n_t, j = e - fi * p.n_t;
            const int64_t f = p.f0[bl] + fi_lo + fi;
            const int64_t ph = p.rope_reset > 0 ? f % p.rope_reset : f;
            const double a = static_cast<double>(ph) * __ldg(p.omega_t + j);
            const double turns = rint(a * 0.15915494309189535);  // a / (2 pi), nearest integer
            const float r = static_cast<float>(fma(-turns, 6.283185307179586, a));
            float sn, cs;
            sincosf(r, &sn, &cs);
            tab[e] = make_float2(cs, sn);
        }
        const int token = q_row0 + (paired ? 0 : qt * kBlockM) + row;   // (pair mode: both tiles hold rows 0..)
        const bool in_chunk = token < p.lq;
        RopeRow rt;
        {
            const int fi = in_chunk ? token / p.tokens_per_frame : fi_lo;
            const int n = in_chunk ? token - fi * p.tokens_per_frame : 0;
            const int prow = n / p.frame_w;
            const int pcol = n - prow * p.frame_w;
            rt.tab_t = tab + (fi - fi_lo) * p.n_t;
            rt.h = reinterpret_cast<const float2 *>(p.rope_h) + prow;
            rt.w = reinterpret_cast<const float2 *>(p.rope_w) + pcol;
            rt.n_t = p.n_t;
            rt.n_th = p.n_t + p.n_h;
            rt.frame_h = p.frame_h;
            rt.frame_w = p.frame_w;
        }
        uint8_t *qtile = smem + L::kQ + qt * L::kQTile;
        // the default axis split (c - 2 floor(c/3), floor(c/3), floor(c/3)) pairs, c = d/2
        constexpr int kNt = D / 2 - 2 * (D / 6), kNth = kNt + D / 6;
        const bool def_split = p.n_t == kNt && p.n_t + p.n_h == kNth;
        bool ok = true;
        if (!F8 && D == 128 && def_split) {
            // sub-tile 1 holds only row and column pairs: rotated while the temporal table
            // is still being written, then sub-tile 0 after the barrier
            ok = warp_wait(&bars[L::kQFull], 0, abort_flag, p.status, kStatusSoftmaxWait);
            if (ok && in_chunk && (!one_q || t == 1)) rope_subtile_bf16<kNt, kNth>(qtile + L::kSub, row, 32, rt);
            named_bar_sync(2, kAttnThreads - 128);
            if (ok && in_chunk && (!one_q || t == 0)) rope_subtile_bf16<kNt, kNth>(qtile, row, 0, rt);
        } else {
            named_bar_sync(2, kAttnThreads - 128);
            ok = warp_wait(&bars[L::kQFull], 0, abort_flag, p.status, kStatusSoftmaxWait);
            if (ok && in_chunk) {
                if constexpr (F8) {
                    // both threads of a row in the single-tile mode need its scale; one writes the codes
                    const uint8_t *raw = smem + L::kQRaw + qt * L::kQRawTile;
                    q_row_scale = def_split ? rope_row_e4m3<kNt, kNth>(raw, qtile, row, !one_q || t == 0, rt)
                                            : rope_row_e4m3<0, 0>(raw, qtile, row, !one_q || t == 0, rt);
                } else {
                    // two-tile mode: the whole row; single-tile mode: thread t takes sub-tile t
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb) {
                        if (one_q && kb != t) continue;
                        if (def_split)
                            rope_subtile_bf16<kNt, kNth>(qtile + kb * L::kSub, row, kb * 32, rt);
                        else
                            rope_subtile_bf16<0, 0>(qtile + kb * L::kSub, row, kb * 32, rt);
                    }
                }
            } else if (F8 && ok && (!one_q || t == 0)) {
                // rows past the chunk: E4M3 zeros (the bf16 tiles were zero-filled by the TMA)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(qtile + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        fence_proxy_async_shared();             // the tensor core reads these rows next
        mbar_arrive(&bars[L::kQReady]);
    }
    // Fused append: warps 2 and 3 at once, the softmax warps after the query rotation, build
    // the assembled tiles' chunk rows, all from this one place in the code (one copy of it
    // in the instruction cache)
    if constexpr (FUSE) {
        if (warp >= 2 && n_asm > 0) {
            build_part_groups<D, L>(smem, bars, p, f, bg, lk, h, h_pair, paired, a0, paired ? a0 : a1, mp0, mp1, ns,
                                    warp - 2, lane, abort_flag, have_tab);
            rotate_full_groups<D, L>(smem, bars, p, f, bg, h, h_pair, paired, a0, paired ? a0 : a1, mf0, mf1, ns,
                                     warp - 2, lane, abort_flag, have_tab);
            assembled<L>(bars, lane);
        }
    }

    // Everything above overlaps the previous kernels (dependent launch); the cache and
    // the split partials are only touched below.
    if constexpr (!FUSE) {
        grid_dependency_wait();
        grid_launch_dependents();
    }

    if (warp < 4) {
      regs_dec<80>();
      if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_local > 0) {
            // K tile `it` and V tile `it` are issued as soon as their own ring slot is free
            // (fused append: the first n_asm were issued with the queries).
            int k_issued = n_asm, v_issued = n_asm;
            bool ok = true;
            if constexpr (FUSE) {
                // nothing goes into V stage 2 (the key tables) before the assembled tiles are built
                if (n_asm > 0) ok = mbar_wait(&bars[L::kAsm], 0, abort_flag, p.status, kStatusTmaWait);
            }
            while (ok && v_issued < n_local) {
                if (k_issued < n_local && k_issued <= v_issued + 1) {
                    const int st = k_issued % L::kKStages;
                    const uint32_t ph = (k_issued / L::kKStages) & 1;
                    if (!mbar_wait(&bars[L::kKEmpty + st], ph ^ 1u, abort_flag, p.status, kStatusTmaWait)) {
                        ok = false;
                        break;
                    }
                    if constexpr (F8) {
                        // (pair mode: sequence tile i is tile i / 2 of head h or h_pair)
                        const int hk = paired && (k_issued & 1) ? h_pair : h;
                        mbar_arrive_expect_tx(&bars[L::kKFull + st], L::kKVTile);
                        const int g = paired ? k_issued >> 1 : kv_begin + k_issued, sl = g / p.n_blk;
                        if constexpr (PK) {
                            // rows 64 .. 127 from slot 2g + 1, or past the ring (zero-filled, masked)
                            const int s1 = 2 * g + 1 < n_vslots ? 2 * g + 1 : p.slots;
                            tma_load_4d(smem + L::kK + st * L::kKVTile, &tmap_k, &bars[L::kKFull + st], 0, hk,
                                        2 * g * p.np_tokens, bg);
                            tma_load_4d(smem + L::kK + st * L::kKVTile + L::kKVTile / 2, &tmap_k,
                                        &bars[L::kKFull + st], 0, hk, s1 * p.np_tokens, bg);
                        } else {
                            tma_load_4d(smem + L::kK + st * L::kKVTile, &tmap_k, &bars[L::kKFull + st], 0, hk,
                                        sl * p.np_tokens + (g - sl * p.n_blk) * kBlockN, bg);
                        }
                    } else {
                        // (pair mode: sequence tile i is tile i / 2 of head h or h_pair)
                        const int hk = paired && (k_issued & 1) ? h_pair : h;
                        const int tk = paired ? tile_at(k_issued >> 1) : tile_at(k_issued);
                        mbar_arrive_expect_tx(&bars[L::kKFull + st], L::kKVTile);
#pragma unroll
                        for (int kb = 0; kb < D / 64; ++kb)
                            tma_load_4d(smem + L::kK + st * L::kKVTile + kb * L::kSub, &tmap_k, &bars[L::kKFull + st],
                                        kb * 64, hk, tk * kBlockN, bg);
                    }
                    ++k_issued;
                }
                const int st = v_issued % L::kVStages;
                const uint32_t ph = (v_issued / L::kVStages) & 1;
                if (!mbar_wait(&bars[L::kVEmpty + st], ph ^ 1u, abort_flag, p.status, kStatusTmaWait)) {
                    ok = false;
                    break;
                }
                if constexpr (F8) {
                    const int hv = paired && (v_issued & 1) ? h_pair : h;
                    mbar_arrive_expect_tx(&bars[L::kVFull + st], L::kKVTile);
                    const int g = paired ? v_issued >> 1 : kv_begin + v_issued, sl = g / p.n_blk;
                    if constexpr (PK) {
                        // two 64-key halves (128 channel rows of 64 bytes each), one per slot
                        const int s1 = 2 * g + 1 < n_vslots ? 2 * g + 1 : p.slots;
                        tma_load_5d(smem + L::kV + st * L::kKVTile, &tmap_v, &bars[L::kVFull + st], 0, 0, hv, 2 * g,
                                    bg);
                        tma_load_5d(smem + L::kV + st * L::kKVTile + L::kKVTile / 2, &tmap_v, &bars[L::kVFull + st],
                                    0, 0, hv, s1, bg);
                    } else {
                        tma_load_5d(smem + L::kV + st * L::kKVTile, &tmap_v, &bars[L::kVFull + st],
                                    (g - sl * p.n_blk) * kBlockN, 0, hv, sl, bg);
                    }
                } else {
                    const int hv = paired && (v_issued & 1) ? h_pair : h;
                    const int tv = paired ? tile_at(v_issued >> 1) : tile_at(v_issued);
                    mbar_arrive_expect_tx(&bars[L::kVFull + st], L::kKVTile);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_4d(smem + L::kV + st * L::kKVTile + kb * L::kSub, &tmap_v, &bars[L::kVFull + st],
                                    kb * 64, hv, tv * kBlockN, bg);
                }
                ++v_issued;
            }
            if (!ok) {
                // Let every copy already in flight land before the CTA leaves.
                const uint64_t t0 = global_timer_ns();
                for (int i = k_issued - L::kKStages; i < k_issued; ++i) {
                    if (i < 0) continue;
                    while (!mbar_try_wait(&bars[L::kKFull + i % L::kKStages], (i / L::kKStages) & 1))
                        if (global_timer_ns() - t0 > kWaitLimitNs) break;
                }
                for (int i = v_issued - L::kVStages; i < v_issued; ++i) {
                    if (i < 0) continue;
                    while (!mbar_try_wait(&bars[L::kVFull + i % L::kVStages], (i / L::kVStages) & 1))
                        if (global_timer_ns() - t0 > kWaitLimitNs) break;
                }
                if constexpr (FUSE) {
                    if (n_asm > 0)
                        while (!mbar_try_wait(&bars[L::kTabReady], 0))
                            if (global_timer_ns() - t0 > kWaitLimitNs) break;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n_local > 0) {
            // fp8: E4M3 operands, K = 32 per MMA; V is stored transposed, so both B operands
            // are K-major 128-byte rows
            constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(kBlockM, kBlockN, 0, 0) : idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t idesc_pv = F8 ? idesc_e4m3_f32(kBlockM, D, 0, 0) : idesc_bf16_f32(kBlockM, D, 0, 1);
            // Descriptors are built once; each MMA only adds a constant to the start-address
            // field (bits 0..13, address >> 4; every operand lies below 256 KB, so no carry
            // leaves the field).  This keeps the issuing thread's instruction count low: it
            // shares its SM sub-partition with busy softmax warps.
            const uint64_t dq = smem_desc_sw128(smem_addr(smem + L::kQ), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_addr(smem + L::kK), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_addr(smem + L::kV), F8 ? 16 : L::kSub, 1024);
            auto issue_qk = [&](int t, int st) {
                const uint64_t a0 = dq + static_cast<uint64_t>((one_q ? 0 : t) * (L::kQTile >> 4));
                const uint64_t b0 = dk + static_cast<uint64_t>(st * (L::kKVTile >> 4));
                if constexpr (F8) {
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        umma_ss_f8(tmem + t * 128, a0 + kk * 2, b0 + kk * 2, idesc_qk, kk > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * L::kSub + (kk & 3) * 32) >> 4);
                        umma_ss(tmem + t * 128, a0 + off, b0 + off, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                }
            };
            auto issue_pv = [&](int t, int st, bool acc) {
                const uint64_t b0 = dv + static_cast<uint64_t>(st * (L::kKVTile >> 4));
                if constexpr (F8) {
                    if constexpr (PK) {
                        // 64-token slots: the V tile's two halves, 128 rows of 64 bytes each;
                        // keys 32 kk .. 32 kk + 31 are half kk / 2, byte 32 (kk % 2) of its rows
                        const uint64_t b1 = smem_desc_sw64(smem_addr(smem + L::kV), 16, 512) +
                                            static_cast<uint64_t>(st * (L::kKVTile >> 4));
#pragma unroll
                        for (int kk = 0; kk < kBlockN / 32; ++kk)
                            umma_ts_f8(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                       b1 + static_cast<uint64_t>((kk >> 1) * (L::kKVTile >> 5) + (kk & 1) * 2),
                                       idesc_pv, (acc || kk > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kBlockN / 32; ++kk)
                            umma_ts_f8(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, b0 + kk * 2, idesc_pv,
                                       (acc || kk > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk)
                        umma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(&bars[L::kQReady], 0, abort_flag, p.status, kStatusMmaWait);
            if constexpr (FUSE) {
                // the chunk's rows of the first n_asm tiles (their other rows come by TMA)
                if (ok && n_asm > 0) ok = mbar_wait(&bars[L::kAsm], 0, abort_flag, p.status, kStatusMmaWait);
            }
            if (alt) {
                // KV tile i -> accumulator set i & 1.  Prologue: S_0 = Q K_0^T, S_1 = Q K_1^T.
                for (int i = 0; ok && i < n_local && i < 2; ++i) {
                    ok = mbar_wait(&bars[L::kKFull + i % L::kKStages], (i / L::kKStages) & 1, abort_flag, p.status,
                                   kStatusMmaWait);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(i, i % L::kKStages);
                    umma_commit(&bars[L::kSFull + i]);
                    umma_commit(&bars[L::kKEmpty + i % L::kKStages]);
                }
                for (int i = 0; ok && i < n_local; ++i) {
                    const int t = i & 1;
                    const int st = i % L::kVStages;
                    if (!mbar_wait(&bars[L::kVFull + st], (i / L::kVStages) & 1, abort_flag, p.status, kStatusMmaWait))
                        break;
                    if (!mbar_wait(&bars[L::kPFull + t], (i >> 1) & 1, abort_flag, p.status, kStatusMmaWait)) break;
                    tc_fence_after();
                    issue_pv(t, st, i >= 2);
                    umma_commit(&bars[L::kVEmpty + st]);
                    const int nk = i + 2;
                    if (nk < n_local) {
                        const int kst = nk % L::kKStages;
                        if (!mbar_wait(&bars[L::kKFull + kst], (nk / L::kKStages) & 1, abort_flag, p.status,
                                       kStatusMmaWait))
                            break;
                        tc_fence_after();
                        issue_qk(t, kst);
                        umma_commit(&bars[L::kSFull + t]);
                        umma_commit(&bars[L::kKEmpty + kst]);
                    } else {
                        umma_commit(&bars[L::kOFull + t]);
                    }
                }
                ok = false;                              // the two-tile schedule below is skipped
            }
            if (ok) {
                tc_fence_after();
                ok = mbar_wait(&bars[L::kKFull + 0], 0, abort_flag, p.status, kStatusMmaWait);
            }
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < n_qt; ++t) {
                    issue_qk(t, 0);
                    umma_commit(&bars[L::kSFull + t]);
                }
                umma_commit(&bars[L::kKEmpty + 0]);
            }
            for (int it = 0; ok && it < n_local; ++it) {
                const int st = it % L::kVStages;            // V slot of tile it
                const uint32_t ph = (it / L::kVStages) & 1;
                const int nst = (it + 1) % L::kKStages;     // K slot of tile it+1
                const uint32_t nph = ((it + 1) / L::kKStages) & 1;
                const bool more = it + 1 < n_local;
                if (!mbar_wait(&bars[L::kVFull + st], ph, abort_flag, p.status, kStatusMmaWait)) break;
                tc_fence_after();
                for (int t = 0; t < n_qt; ++t) {
                    if (!mbar_wait(&bars[L::kPFull + t], it & 1, abort_flag, p.status, kStatusMmaWait)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(t, st, it > 0);
                    if (more) {
                        if (t == 0) {
                            if (!mbar_wait(&bars[L::kKFull + nst], nph, abort_flag, p.status, kStatusMmaWait)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        issue_qk(t, nst);
                        umma_commit(&bars[L::kSFull + t]);
                    } else {
                        umma_commit(&bars[L::kOFull + t]);
                    }
                }
                if (!ok) break;
                umma_commit(&bars[L::kVEmpty + st]);
                if (more) umma_commit(&bars[L::kKEmpty + nst]);
            }
            // Drain: every MMA issued so far has finished before TMEM is released.
            umma_commit(&bars[L::kDrain]);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&bars[L::kDrain], 0)) {
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(p.status, kStatusMmaWait);
                    break;
                }
            }
        }
      }
    } else {
        regs_inc<208>();
        // ------------------------------------------------ softmax / epilogue
        const int t = (warp - 4) >> 2;               // query tile of this warpgroup
        const int row = ((warp & 3) << 5) + lane;    // TMEM lane == query row in the tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) << 5) << 16;
        if (t < n_qt || alt) {
            // in the single-tile mode, tile 1's warps take the odd KV tiles of tile 0's rows
            const int token = q_row0 + (alt ? 0 : t) * kBlockM + row;
            const int hs = paired && t ? h_pair : h;   // head of this set's rows
            const bool valid = token < p.lq;
            const int n_mine = alt ? (n_local + 1 - t) / 2 : n_local;
            float m_run = -INFINITY;   // running max of scale*log2(e)*s
            float l_run = 0.0f;
            bool ok = true;
            const uint32_t s_tmem = tmem + lane_base + t * 128;
            const uint32_t o_tmem = tmem + lane_base + 256 + t * 128;
            // fp8: this row's query scale, and the largest V scale of the CTA's tiles (every
            // tile's P is multiplied by its V scale over this one; the epilogue multiplies back)
            float sq = 1.0f, sv_ref = 1.0f;
            int64_t scale_base = 0;
            if constexpr (F8) {
                sq = valid ? q_row_scale : 0.0f;
                scale_base = static_cast<int64_t>(bg) * p.slots * p.scale_slot_stride + hs * p.n_blk;
                sv_ref = 0.0f;
                // this set's tiles (pair mode: all of its own head's; otherwise the CTA's range,
                // which both sets of a single query tile share)
                for (int i = 0; i < (paired ? n_kv : n_local); ++i) {
                    const int g = kv_begin + i, sl = g / p.n_blk;
                    if constexpr (PK) {
                        // (one block per slot: the scale of slot s at scale_base + s * stride)
                        sv_ref = fmaxf(sv_ref, p.v_scale[scale_base + 2 * g * p.scale_slot_stride]);
                        if (2 * g + 1 < n_vslots)
                            sv_ref = fmaxf(sv_ref, p.v_scale[scale_base + (2 * g + 1) * p.scale_slot_stride]);
                    } else {
                        sv_ref = fmaxf(sv_ref, p.v_scale[scale_base + sl * (p.scale_slot_stride - p.n_blk) + g]);
                    }
                }
                sv_ref = fmaxf(sv_ref, 1e-30f);
            }
            // bf16: the one iteration of this set whose KV tile is the valid prefix's ragged
            // last tile (keys past lk masked), found once: the tile's position in the CTA's
            // tile order (the inverse of tile_at), then the set's iteration of that position
            int rag_it = -1;
            const int rag_cols = lk - (n_kv - 1) * kBlockN;
            if constexpr (!F8) {
                const int gl = n_kv - 1;
                int pos = -1;
                if (rag_cols < kBlockN && gl >= kv_begin && gl < kv_end) {
                    if (gl == a0)
                        pos = 0;
                    else if (gl == a1)
                        pos = 1;
                    else
                        pos = gl - kv_begin + na - (a0 >= 0 && a0 < gl) - (a1 >= 0 && a1 < gl);
                }
                if (pos >= 0) rag_it = paired || !alt ? pos : ((pos & 1) == t ? pos >> 1 : -1);
            }
            for (int it = 0; it < n_mine; ++it) {
                float c_t = p.scale_log2, r_t = 1.0f;
                float c_h = 0.0f, r_h = 0.0f;           // two slots per tile: scales of columns 64 .. 127
                int valid_cols;
                if constexpr (F8) {
                    const int g = kv_begin + (paired ? it : (alt ? 2 * it + t : it));   // KV tile of this iteration
                    const int sl = g / p.n_blk;
                    if constexpr (PK) {
                        const int64_t si = scale_base + static_cast<int64_t>(2 * g) * p.scale_slot_stride;
                        c_t = fmaxf(p.scale_log2 * sq * p.k_scale[si], 1e-30f);
                        r_t = p.v_scale[si] / sv_ref;
                        valid_cols = 2 * g + 1 < n_vslots ? kBlockN : kBlockN / 2;
                        c_h = c_t;
                        r_h = r_t;
                        if (valid_cols == kBlockN) {
                            const int64_t sj = si + p.scale_slot_stride;
                            c_h = fmaxf(p.scale_log2 * sq * p.k_scale[sj], 1e-30f);
                            r_h = p.v_scale[sj] / sv_ref;
                        }
                    } else {
                        const int64_t si = scale_base + sl * (p.scale_slot_stride - p.n_blk) + g;
                        c_t = fmaxf(p.scale_log2 * sq * p.k_scale[si], 1e-30f);
                        r_t = p.v_scale[si] / sv_ref;
                        valid_cols = p.tokens_per_frame - (g - sl * p.n_blk) * kBlockN;
                    }
                } else {
                    valid_cols = it == rag_it ? rag_cols : kBlockN;
                }
                if (!warp_wait(&bars[L::kSFull + t], it & 1, abort_flag, p.status, kStatusSoftmaxWait)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t sr[kBlockN / 32][32];
#pragma unroll
                for (int cb = 0; cb < kBlockN / 32; ++cb) tmem_ld32(s_tmem + cb * 32, sr[cb]);
                tmem_wait_ld_bind(sr[0]);
#pragma unroll
                for (int cb = 1; cb < kBlockN / 32; ++cb) reg_bind(sr[cb]);
                if (valid_cols < kBlockN) {
#pragma unroll
                    for (int cb = 0; cb < kBlockN / 32; ++cb)
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (cb * 32 + i >= valid_cols) sr[cb][i] = 0xff800000u;   // -inf
                }
                // row max: four 3-input max chains, then combine
                float m4[4];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float m = __uint_as_float(sr[cb][0]);
#pragma unroll
                    for (int i = 1; i < 31; i += 2)
                        m = fmax3(m, __uint_as_float(sr[cb][i]), __uint_as_float(sr[cb][i + 1]));
                    m4[cb] = fmaxf(m, __uint_as_float(sr[cb][31]));
                }
                if (PK && c_h != c_t) {
                    // fp8, a tile of two slots: the half with the smaller scale is brought to
                    // the larger one (a factor below 1, so nothing overflows), so that one
                    // scale serves the whole row below; a positive factor keeps the maxima
                    const int lo = c_h > c_t ? 0 : 1;       // the half scaled down
                    const float k = lo ? c_h / c_t : c_t / c_h;
#pragma unroll
                    for (int cb = 0; cb < kBlockN / 32; ++cb) {
                        if (cb / (kBlockN / 64) != lo) continue;
#pragma unroll
                        for (int i = 0; i < 32; ++i) sr[cb][i] = __float_as_uint(__uint_as_float(sr[cb][i]) * k);
                        m4[cb] *= k;
                    }
                    c_t = fmaxf(c_t, c_h);
                }
                const float m_tile = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c_t;
                bool rescale = false;
                float alpha = 1.0f;
                if (it == 0) {
                    m_run = m_tile;
                } else if (m_tile > m_run + kRescaleThreshold) {
                    rescale = true;
                    alpha = ex2_approx(m_run - m_tile);
                    l_run *= alpha;
                    m_run = m_tile;
                }
                if constexpr (F8)
                    l_run += softmax_exp_store_f8<PK>(sr, c_t, -m_run, r_t, r_h, s_tmem);
                else
                    l_run += softmax_exp_store(sr, c_t, -m_run, s_tmem);
                // O_t is idle here (PV(t, it-1) completed before S(t, it) was signalled and
                // PV(t, it) waits for this thread's arrival below), so it can be rescaled now.
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                    for (int cb = 0; cb < D / 32; ++cb) {
                        uint32_t r[32];
                        tmem_ld32(o_tmem + cb * 32, r);
                        tmem_wait_ld_bind(r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(o_tmem + cb * 32, r);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[L::kPFull + t]);
            }

            if (one_q) {
                // ---- single-tile epilogue: merge the two accumulator sets of the row; thread
                // (t, row) produces output columns [t d/2, (t+1) d/2)
                const int n0 = (n_local + 1) / 2, n1 = n_local / 2;
                if (ok && n0 > 0) ok = warp_wait(&bars[L::kOFull + 0], 0, abort_flag, p.status, kStatusSoftmaxWait);
                if (ok && n1 > 0) ok = warp_wait(&bars[L::kOFull + 1], 0, abort_flag, p.status, kStatusSoftmaxWait);
                // (max, sum) of both sets through the unused second query-tile slot
                float2 *xm = reinterpret_cast<float2 *>(smem + L::kQ + L::kQTile);
                xm[t * kBlockM + row] = make_float2(n_mine > 0 ? m_run : -INFINITY, l_run);
                ok = named_bar_and(1, 2 * 4 * 32, ok);
                const float2 a0 = xm[row], a1 = xm[kBlockM + row];
                const float m = fmaxf(a0.x, a1.x);
                const float w0 = a0.x == -INFINITY ? 0.0f : ex2_approx(a0.x - m);
                const float w1 = a1.x == -INFINITY ? 0.0f : ex2_approx(a1.x - m);
                const float l = w0 * a0.y + w1 * a1.y;
                const float svr = F8 ? sv_ref : 1.0f;      // fp8: undo the V-scale normalisation of P
                if (ok) tc_fence_after();
                const uint32_t o0 = tmem + lane_base + 256 + t * (D / 2);
                const uint32_t o1 = o0 + 128;
                if (n_split == 1) {
                    if (ok) {
                        const float inv = svr / l;
                        uint16_t *orow =
                            p.out + ((static_cast<int64_t>(bg) * p.lq + token) * p.heads + h) * D + t * (D / 2);
#pragma unroll 1
                        for (int cb = 0; cb < D / 64; ++cb) {
                            uint32_t v[32];
                            merge_sets(o0 + cb * 32, o1 + cb * 32, n1 > 0, w0, w1, v);
                            if (valid) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    uint4 w;
                                    w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
                                    w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
                                    w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
                                    w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
                                    *reinterpret_cast<uint4 *>(orow + cb * 32 + q * 8) = w;
                                }
                            }
                        }
                    }
                } else if (ok) {
                    // KV split: this split's merged, unnormalised partial (layout as below)
                    float4 *po = reinterpret_cast<float4 *>(p.part_o) +
                                 (static_cast<int64_t>(split) * n_su + su) * (D / 4) * 256 + t * (D / 8) * 256 + row;
                    if (n_local > 0) {
#pragma unroll 1
                        for (int cb = 0; cb < D / 64; ++cb) {
                            uint32_t v[32];
                            merge_sets(o0 + cb * 32, o1 + cb * 32, n1 > 0, w0 * svr, w1 * svr, v);
                            if (valid) {
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    po[(cb * 8 + q) * 256] =
                                        make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                    __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                            }
                        }
                    } else if (valid) {
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) po[c * 256] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    }
                    if (valid && t == 0)
                        reinterpret_cast<float2 *>(p.part_ml)[(static_cast<int64_t>(split) * n_su + su) * 256 + row] =
                            make_float2(n_local > 0 ? m : -INFINITY, l);
                }
            } else {
                // ---- epilogue
                if (ok && n_local > 0) ok = warp_wait(&bars[L::kOFull + t], 0, abort_flag, p.status, kStatusSoftmaxWait);
                if (ok) tc_fence_after();
                const float svr = F8 ? sv_ref : 1.0f;          // fp8: undo the V-scale normalisation of P
                if (n_split == 1) {
                    if (ok) {
                        const float inv = svr / l_run;
                        uint16_t *orow = p.out + ((static_cast<int64_t>(bg) * p.lq + token) * p.heads + hs) * D;
#pragma unroll
                        for (int cb = 0; cb < D / 32; ++cb) {
                            uint32_t r[32];
                            tmem_ld32(o_tmem + cb * 32, r);
                            tmem_wait_ld_bind(r);
                            if (valid) {
#pragma unroll
                                for (int v = 0; v < 4; ++v) {
                                    uint4 w;
                                    w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
                                    w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
                                    w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
                                    w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
                                    *reinterpret_cast<uint4 *>(orow + cb * 32 + v * 8) = w;
                                }
                            }
                        }
                    }
                } else if (ok) {
                    // ---- KV split: write this split's unnormalised partial for attention_combine_kernel.
                    // part_o: one block per (piece, split unit) of [D/4 float4 columns][256 rows]
                    // (rows t*128 + lane; a warp's 32 rows are 512 contiguous bytes);
                    // part_ml[piece][split unit][256] float2 = (row max in log2 units, sum).
                    const int64_t blk = static_cast<int64_t>(split) * n_su + su;
                    const int srow = t * kBlockM + row;
                    if (n_local > 0) {                         // warp-uniform: every lane takes part in tcgen05.ld
                        float4 *po = reinterpret_cast<float4 *>(p.part_o) + blk * (D / 4) * 256 + srow;
                        uint32_t r[D / 32][32];
#pragma unroll
                        for (int cb = 0; cb < D / 32; ++cb) tmem_ld32(o_tmem + cb * 32, r[cb]);
                        tmem_wait_ld_bind(r[0]);
#pragma unroll
                        for (int cb = 1; cb < D / 32; ++cb) reg_bind(r[cb]);
                        if (valid) {
#pragma unroll
                            for (int cb = 0; cb < D / 32; ++cb)
#pragma unroll
                                for (int v = 0; v < 8; ++v)
                                    po[(cb * 8 + v) * 256] = make_float4(
                                        __uint_as_float(r[cb][4 * v]) * svr, __uint_as_float(r[cb][4 * v + 1]) * svr,
                                        __uint_as_float(r[cb][4 * v + 2]) * svr, __uint_as_float(r[cb][4 * v + 3]) * svr);
                        }
                    } else if (valid) {                         // no keys in this split: zero partial
                        float4 *po = reinterpret_cast<float4 *>(p.part_o) + blk * (D / 4) * 256 + srow;
#pragma unroll
                        for (int c = 0; c < D / 4; ++c) po[c * 256] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    }
                    if (valid)
                        reinterpret_cast<float2 *>(p.part_ml)[blk * 256 + srow] =
                            make_float2(n_local > 0 ? m_run : -INFINITY, l_run);
                }
            }
        }
    }

    // Lane 0 of the producer and MMA warps arrives here long after the other lanes:
    // reconverge each warp first, so that the block barrier counts every warp only
    // once all its threads are done (TMEM is released right after it).
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of the KV-split partials: out = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s.
// Thread = (row, 4 float4 columns) of one (stream, head, query-tile pair) block:
// consecutive threads take consecutive rows, so every load of a split's column
// is coalesced.  The splits are merged four at a time with all their loads in
// flight (a split CTA without keys wrote zeros and a -inf maximum): the group's
// maximum updates the running one and rescales what was merged before, as in the
// online softmax; with up to four splits that is one group and no rescale.  The
// partials are read once (evict-first loads).
template <int D>
__global__ void __launch_bounds__(256, 3) attention_combine_kernel(const __grid_constant__ AttnParams p) {
    grid_dependency_wait();                         // the split CTAs' partials
    grid_launch_dependents();
    constexpr int kC16 = D / 16;                    // 16-column chunks per row
    constexpr int kGroup = 4;                       // splits whose loads are in flight together
    const int n_su = p.n_units - p.n_whole;         // split units
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int srow = static_cast<int>(idx & 255);
    const int64_t rest = idx >> 8;
    const int c16 = static_cast<int>(rest % kC16);
    const int su = static_cast<int>(rest / kC16);
    if (su >= n_su) return;
    const int unit = p.n_whole + su;
    const int qpair = unit % p.n_qpairs;
    const int h = (unit / p.n_qpairs) % p.heads;
    const int bg = p.b_offset + p.unit_stream[unit / (p.n_qpairs * p.heads)];
    const int token = qpair * 256 + srow;
    if (token >= p.lq) return;
    const int np = p.n_pieces;
    const float2 *ml_row = reinterpret_cast<const float2 *>(p.part_ml) + static_cast<int64_t>(su) * 256 + srow;
    const int64_t ml_split = static_cast<int64_t>(n_su) * 256;        // float2 stride between splits
    float m = -INFINITY;                            // running maximum over the splits merged so far
    float a[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = 0.0f;
    float l = 0.0f;
    for (int s0 = 0; s0 < np; s0 += kGroup) {
        // the group's (max, sum) first, then its columns split by split
        float2 ml[kGroup];
#pragma unroll
        for (int g = 0; g < kGroup; ++g)
            ml[g] = s0 + g < np ? __ldcs(ml_row + (s0 + g) * ml_split) : make_float2(-INFINITY, 0.0f);
        float mg = m;
#pragma unroll
        for (int g = 0; g < kGroup; ++g) mg = fmaxf(mg, ml[g].x);
        // rescale what was merged so far to the new maximum (nothing merged yet: factor 0)
        const float c = m == -INFINITY ? 0.0f : exp2f(m - mg);
        l *= c;
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] *= c;
#pragma unroll
        for (int g = 0; g < kGroup; ++g) {
            if (s0 + g < np) {                      // (the slots past the last split hold no data)
                const int64_t blk = static_cast<int64_t>(s0 + g) * n_su + su;
                const float4 *po = reinterpret_cast<const float4 *>(p.part_o) + blk * (D / 4) * 256 + (c16 * 4) * 256 + srow;
                const float w = ml[g].x == -INFINITY ? 0.0f : exp2f(ml[g].x - mg);
                l += w * ml[g].y;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 u = __ldcs(po + i * 256);
                    a[4 * i] += w * u.x;
                    a[4 * i + 1] += w * u.y;
                    a[4 * i + 2] += w * u.z;
                    a[4 * i + 3] += w * u.w;
                }
            }
        }
        m = mg;
    }
    const float inv = 1.0f / l;
    uint16_t *orow = p.out + ((static_cast<int64_t>(bg) * p.lq + token) * p.heads + h) * D + c16 * 16;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
        uint4 w;
        w.x = pack_bf16x2(a[8 * v + 0] * inv, a[8 * v + 1] * inv);
        w.y = pack_bf16x2(a[8 * v + 2] * inv, a[8 * v + 3] * inv);
        w.z = pack_bf16x2(a[8 * v + 4] * inv, a[8 * v + 5] * inv);
        w.w = pack_bf16x2(a[8 * v + 6] * inv, a[8 * v + 7] * inv);
        *reinterpret_cast<uint4 *>(orow + v * 8) = w;
    }
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing
// arrives on, with the given bound; the bounded wait gives up, records
// kStatusSelfTest in the status word and the kernel returns normally.
__global__ void bounded_wait_selftest_kernel(uint32_t *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&bar, 0)) {
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(status, kStatusSelfTest);
            return;
        }
    }
}

cudaError_t launch_wait_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t s) {
    bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

template <int D, bool F8, bool FUSE, bool PK, typename FP>
static cudaError_t launch_attention_d(const AttnParams &p, const FP &f, const CUtensorMap &tq, const CUtensorMap &tk,
                                      const CUtensorMap &tv, cudaStream_t s) {
    static bool configured = false;
    const int smem = AttnLayout<D, F8, FUSE>::kAlloc;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(chunk_attention_kernel<D, F8, FUSE, PK>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (p.n_units == 0) return cudaSuccess;
    // pair mode: one CTA per (stream, pair of heads); otherwise whole units, then pieces
    dim3 grid(static_cast<unsigned>(p.pair ? p.n_units / p.heads * ((p.heads + 1) / 2)
                                           : p.n_whole + (p.n_units - p.n_whole) * p.n_pieces));
    return launch_dependent(chunk_attention_kernel<D, F8, FUSE, PK>, grid, dim3(kAttnThreads), static_cast<size_t>(smem),
                            s, p, tq, tk, tv, f);
}

cudaError_t launch_attention(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, int head_dim, cudaStream_t s) {
    const FuseNone none{0};
    if (p.f8)
        return p.pack2 ? launch_attention_d<128, true, false, true>(p, none, tq, tk, tv, s)
                       : launch_attention_d<128, true, false, false>(p, none, tq, tk, tv, s);
    if (head_dim == 64) return launch_attention_d<64, false, false, false>(p, none, tq, tk, tv, s);
    return launch_attention_d<128, false, false, false>(p, none, tq, tk, tv, s);
}

cudaError_t launch_append_attention(const AttnParams &p, const FuseParams &f, const CUtensorMap &tq,
                                    const CUtensorMap &tk, const CUtensorMap &tv, int head_dim, cudaStream_t s) {
    if (head_dim == 64) return launch_attention_d<64, false, true, false>(p, f, tq, tk, tv, s);
    return launch_attention_d<128, false, true, false>(p, f, tq, tk, tv, s);
}

cudaError_t launch_combine(const AttnParams &p, int head_dim, cudaStream_t s) {
    if (p.n_units == p.n_whole) return cudaSuccess;
    const int64_t threads = static_cast<int64_t>(p.n_units - p.n_whole) * (head_dim / 16) * 256;
    const dim3 grid(static_cast<unsigned>((threads + 255) / 256));
    if (head_dim == 64) return launch_dependent(attention_combine_kernel<64>, grid, dim3(256), 0, s, p);
    return launch_dependent(attention_combine_kernel<128>, grid, dim3(256), 0, s, p);
}

}  // namespace sdv2

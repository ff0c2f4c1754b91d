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
// Q: rope_q_kernel rotates the chunk's queries once per call (fp32 RoPE,
// rounded to bf16) into a scratch buffer; the producer warp TMA-loads the
// rotated tiles straight into the 128-byte-swizzled K-major layout the MMA
// reads.
// fp8 (E4M3) cache (the F8 instantiation, head_dim 128): KV tiles are the
// 128-token blocks of each valid slot (tile g = block g % n_blk of slot
// g / n_blk, padding tokens masked), V tiles come from the slot's transposed
// codes, and Q, K, P and V enter kind::f8f6f4 MMAs (K = 32 per instruction).
// Each tile's K scale and the query row's scale fold into the softmax scale of
// that tile; each tile's V scale divided by the CTA's largest V scale
// multiplies P before its E4M3 coding, and the epilogue multiplies O back by
// that largest scale.  P takes columns [0, 32) of S_t.
// KV splits: each split CTA writes its unnormalised O, row max and row sum;
// attention_combine_kernel (a dependent launch) merges them over the whole
// GPU.
// Every wait is bounded (2 s), after which the CTA records an error in the
// device status word and unwinds; TMEM is always released.
#include <cmath>

#include "ptx.cuh"

namespace sdv2 {

template <int D, bool F8 = false>
struct AttnLayout {
    static constexpr int kElem = F8 ? 1 : 2;          // bytes per element of Q, K, V
    static constexpr int kQTile = kBlockM * D * kElem;    // bytes of one Q tile
    static constexpr int kKVTile = kBlockN * D * kElem;   // bytes of one K (or V) tile
    static constexpr int kSub = kBlockM * 128;        // one 64-column (128-byte) sub-tile
    static constexpr int kKStages = 2;                // K tile i is needed one half-iteration before V tile i,
    static constexpr int kVStages = 3;                // so V gets the deeper ring to hide its load latency
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQTilesPerCta * kQTile;
    static constexpr int kV = kK + kKStages * kKVTile;
    static constexpr int kBar = kV + kVStages * kKVTile;
    // barriers
    static constexpr int kQFull = 0;
    static constexpr int kKFull = 1;
    static constexpr int kKEmpty = kKFull + kKStages;
    static constexpr int kVFull = kKEmpty + kKStages;
    static constexpr int kVEmpty = kVFull + kVStages;
    static constexpr int kSFull = kVEmpty + kVStages;
    static constexpr int kPFull = kSFull + 2;
    static constexpr int kOFull = kPFull + 2;
    static constexpr int kDrain = kOFull + 2;
    static constexpr int kNumBars = kDrain + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;   // tmem base, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;      // room to align the base to 1024 bytes
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

// RoPE of the chunk's queries: q_rot = rotate(q) at (phase(frame), row, col),
// fp32 arithmetic, bf16 result.  Block = 64 (token, head) rows of one stream,
// 4 threads per row, every 4th 16-byte vector of the row per thread (loads
// first).  grid = (row blocks, streams of the launch).  The temporal angles
// phase * base^(-j / n_t) of the stream's chunk frames are evaluated in fp64
// by each block and rounded to fp32, like the row and column tables.
__global__ void __launch_bounds__(256) rope_q_kernel(const __grid_constant__ AttnParams p, int head_dim) {
    // Launched right behind the KV append, whose own wait already ordered it after
    // the producer of q: q can be read at once.  Completing only after the append
    // (wait at the end) lets the attention kernel wait on this kernel alone.
    grid_launch_dependents();
    const int bl = blockIdx.y;
    __shared__ float2 s_tab[kAttnTabEntries];        // temporal (cos, sin) of this stream's frames
    for (int e = threadIdx.x; e < p.chunk_frames * p.n_t; e += blockDim.x) {
        const int fi = e / p.n_t, j = e - fi * p.n_t;
        const int64_t f = p.f0[bl] + fi;
        const int64_t ph = p.rope_reset > 0 ? f % p.rope_reset : f;
        const double a = static_cast<double>(ph) * pow(p.rope_base, -static_cast<double>(j) / static_cast<double>(p.n_t));
        double sn, cs;
        sincos(a, &sn, &cs);
        s_tab[e] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
    __syncthreads();
    const int rows = p.lq * p.heads;
    const int row = blockIdx.x * 64 + (threadIdx.x >> 2);
    const int sub = threadIdx.x & 3;
    if (p.lk[bl] <= 0 || row >= rows) {
        grid_dependency_wait();
        return;
    }
    const int token = row / p.heads;
    const int fi = token / p.tokens_per_frame;
    const int n = token - fi * p.tokens_per_frame;
    const int prow = n / p.frame_w;
    const int pcol = n - prow * p.frame_w;
    const int64_t off = (static_cast<int64_t>(p.b_offset + bl) * rows + row) * head_dim;
    constexpr int kMaxVec = 4;
    const int nvec = head_dim / 32;
    uint4 x[kMaxVec];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i)
        if (i < nvec) x[i] = *reinterpret_cast<const uint4 *>(p.q + off + (sub + 4 * i) * 8);
    const float2 *tab_t = s_tab + fi * p.n_t;
    const float2 *tab_h = reinterpret_cast<const float2 *>(p.rope_h) + prow * p.n_h - p.n_t;
    const float2 *tab_w = reinterpret_cast<const float2 *>(p.rope_w) + pcol * p.n_w - p.n_t - p.n_h;
    float2 cs[kMaxVec][4];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        if (i >= nvec) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = (sub + 4 * i) * 4 + q;
            cs[i][q] = *(j < p.n_t ? tab_t + j : (j < p.n_t + p.n_h ? tab_h + j : tab_w + j));
        }
    }
    if (p.q_scale == nullptr) {
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
            if (i >= nvec) break;
            const uint32_t in[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x0 = bf16_lo(in[q]), x1 = bf16_hi(in[q]);
                o[q] = pack_bf16x2(x0 * cs[i][q].x - x1 * cs[i][q].y, x0 * cs[i][q].y + x1 * cs[i][q].x);
            }
            *reinterpret_cast<uint4 *>(p.q_rot + off + (sub + 4 * i) * 8) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
        // fp8 cache (head_dim 128): the rotated row is coded as E4M3 with its own scale
        // amax / 448, amax over the row's 128 channels (the row's 4 threads combine theirs).
        float r[kMaxVec][8];
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
            const uint32_t in[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x0 = bf16_lo(in[q]), x1 = bf16_hi(in[q]);
                r[i][2 * q] = x0 * cs[i][q].x - x1 * cs[i][q].y;
                r[i][2 * q + 1] = x0 * cs[i][q].y + x1 * cs[i][q].x;
                am = fmaxf(am, fmaxf(fabsf(r[i][2 * q]), fabsf(r[i][2 * q + 1])));
            }
        }
        const unsigned group = 0xFu << (threadIdx.x & 28u);
        am = fmaxf(am, __shfl_xor_sync(group, am, 1));
        am = fmaxf(am, __shfl_xor_sync(group, am, 2));
        float scale, inv;
        e4m3_scale_inv(am, scale, inv);
        uint8_t *q8 = reinterpret_cast<uint8_t *>(p.q_rot);
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
            uint32_t c[2];
#pragma unroll
            for (int k = 0; k < 2; ++k)
                c[k] = pack_e4m3x2(r[i][4 * k] * inv, r[i][4 * k + 1] * inv) |
                       (pack_e4m3x2(r[i][4 * k + 2] * inv, r[i][4 * k + 3] * inv) << 16);
            *reinterpret_cast<uint2 *>(q8 + off + (sub + 4 * i) * 8) = make_uint2(c[0], c[1]);
        }
        if (sub == 0) p.q_scale[static_cast<int64_t>(p.b_offset + bl) * rows + row] = scale;
    }
    grid_dependency_wait();
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
__device__ __forceinline__ float softmax_exp_store_f8(const uint32_t (&sr)[kBlockN / 32][32], float c, float neg_m,
                                                      float r, uint32_t s_tmem) {
    const uint64_t scale2 = f2_pack(c, c);
    const uint64_t negm2 = f2_pack(neg_m, neg_m);
    const uint64_t r2 = f2_pack(r, r);
    const uint64_t zero2 = f2_pack(0.0f, 0.0f);
    uint64_t acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0ull;
#pragma unroll
    for (int cb = 0; cb < kBlockN / 32; ++cb) {
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

template <int D, bool F8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    chunk_attention_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v) {
    using L = AttnLayout<D, F8>;
    static_assert(!F8 || D == 128, "the fp8 cache is built for head_dim 128");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // work unit of this CTA: whole units first, then the pieces of the split ones
    int unit, split, n_split;
    if (static_cast<int>(blockIdx.x) < p.n_whole) {
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
    // valid slot (fp8: tile g is block g % n_blk of slot g / n_blk)
    const int n_kv = F8 ? (lk / p.tokens_per_frame) * p.n_blk : (lk + kBlockN - 1) / kBlockN;
    const int per = (n_kv + n_split - 1) / n_split;
    const int kv_begin = split * per;
    const int kv_end = min(n_kv, kv_begin + per);
    const int n_local = kv_end > kv_begin ? kv_end - kv_begin : 0;
    const int q_row0 = qpair * (kBlockM * kQTilesPerCta);
    const int n_qt = (q_row0 + kBlockM < p.lq) ? 2 : 1;
    const bool dual = n_qt == 1;                // one query tile: the two accumulator sets split the KV tiles

    if (threadIdx.x == 0) {
        mbar_init(&bars[L::kQFull], 1);
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
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
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
    // Everything above overlaps the previous kernels (dependent launch); the
    // rotated queries, the cache and the split partials are only touched below.
    grid_dependency_wait();
    grid_launch_dependents();

    if (warp < 4) {
      regs_dec<80>();
      if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_local > 0) {
            // rotated query tiles of this CTA (rows past lq are filled with zeros)
            mbar_arrive_expect_tx(&bars[L::kQFull], n_qt * L::kQTile);
            for (int t = 0; t < n_qt; ++t) {
                if constexpr (F8) {
                    tma_load_4d(smem + L::kQ + t * L::kQTile, &tmap_q, &bars[L::kQFull], 0, h, q_row0 + t * kBlockM, bg);
                } else {
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_4d(smem + L::kQ + t * L::kQTile + kb * L::kSub, &tmap_q, &bars[L::kQFull], kb * 64,
                                    h, q_row0 + t * kBlockM, bg);
                }
            }
            // K tile `it` and V tile `it` are issued as soon as their own ring slot is free.
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            while (ok && v_issued < n_local) {
                if (k_issued < n_local && k_issued <= v_issued + 1) {
                    const int st = k_issued % L::kKStages;
                    const uint32_t ph = (k_issued / L::kKStages) & 1;
                    if (!mbar_wait(&bars[L::kKEmpty + st], ph ^ 1u, abort_flag, p.status, kStatusTmaWait)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[L::kKFull + st], L::kKVTile);
                    if constexpr (F8) {
                        const int g = kv_begin + k_issued, sl = g / p.n_blk;
                        tma_load_4d(smem + L::kK + st * L::kKVTile, &tmap_k, &bars[L::kKFull + st], 0, h,
                                    sl * p.np_tokens + (g - sl * p.n_blk) * kBlockN, bg);
                    } else {
#pragma unroll
                        for (int kb = 0; kb < D / 64; ++kb)
                            tma_load_4d(smem + L::kK + st * L::kKVTile + kb * L::kSub, &tmap_k, &bars[L::kKFull + st],
                                        kb * 64, h, (kv_begin + k_issued) * kBlockN, bg);
                    }
                    ++k_issued;
                }
                const int st = v_issued % L::kVStages;
                const uint32_t ph = (v_issued / L::kVStages) & 1;
                if (!mbar_wait(&bars[L::kVEmpty + st], ph ^ 1u, abort_flag, p.status, kStatusTmaWait)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars[L::kVFull + st], L::kKVTile);
                if constexpr (F8) {
                    const int g = kv_begin + v_issued, sl = g / p.n_blk;
                    tma_load_5d(smem + L::kV + st * L::kKVTile, &tmap_v, &bars[L::kVFull + st],
                                (g - sl * p.n_blk) * kBlockN, 0, h, sl, bg);
                } else {
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_4d(smem + L::kV + st * L::kKVTile + kb * L::kSub, &tmap_v, &bars[L::kVFull + st],
                                    kb * 64, h, (kv_begin + v_issued) * kBlockN, bg);
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
                const uint64_t a0 = dq + static_cast<uint64_t>((dual ? 0 : t) * (L::kQTile >> 4));
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
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 32; ++kk)
                        umma_ts_f8(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, b0 + kk * 2, idesc_pv,
                                   (acc || kk > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk)
                        umma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                                b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(&bars[L::kQFull], 0, abort_flag, p.status, kStatusMmaWait);
            if (dual) {
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
        if (t < n_qt || dual) {
            // in the single-tile mode, tile 1's warps take the odd KV tiles of tile 0's rows
            const int token = q_row0 + (dual ? 0 : t) * kBlockM + row;
            const bool valid = token < p.lq;
            const int n_mine = dual ? (n_local + 1 - t) / 2 : n_local;
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
                sq = valid ? p.q_scale[(static_cast<int64_t>(bg) * p.lq + token) * p.heads + h] : 0.0f;
                scale_base = static_cast<int64_t>(bg) * p.slots * p.scale_slot_stride + h * p.n_blk;
                sv_ref = 0.0f;
                for (int i = 0; i < n_local; ++i) {
                    const int g = kv_begin + i, sl = g / p.n_blk;
                    sv_ref = fmaxf(sv_ref, p.v_scale[scale_base + sl * (p.scale_slot_stride - p.n_blk) + g]);
                }
                sv_ref = fmaxf(sv_ref, 1e-30f);
            }
            for (int it = 0; it < n_mine; ++it) {
                const int g = kv_begin + (dual ? 2 * it + t : it);   // KV tile of this iteration
                float c_t = p.scale_log2, r_t = 1.0f;
                int valid_cols;
                if constexpr (F8) {
                    const int sl = g / p.n_blk;
                    const int64_t si = scale_base + sl * (p.scale_slot_stride - p.n_blk) + g;
                    c_t = fmaxf(p.scale_log2 * sq * p.k_scale[si], 1e-30f);
                    r_t = p.v_scale[si] / sv_ref;
                    valid_cols = p.tokens_per_frame - (g - sl * p.n_blk) * kBlockN;
                } else {
                    valid_cols = lk - g * kBlockN;
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
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                const float m_tile = mx * c_t;
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
                    l_run += softmax_exp_store_f8(sr, c_t, -m_run, r_t, s_tmem);
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

            if (dual) {
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
                        uint16_t *orow = p.out + ((static_cast<int64_t>(bg) * p.lq + token) * p.heads + h) * D;
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
// is coalesced.  Every split's (max, sum) and columns are loaded unconditionally
// (a split CTA without keys writes zeros), so all of a thread's loads are in
// flight at once; the partials are read once (evict-first loads).
template <int D>
__global__ void __launch_bounds__(256) attention_combine_kernel(const __grid_constant__ AttnParams p) {
    grid_dependency_wait();                         // the split CTAs' partials
    grid_launch_dependents();
    constexpr int kC16 = D / 16;                    // 16-column chunks per row
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
    float2 ml[kMaxSplits];
    float4 u[kMaxSplits][4];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
        ml[s] = make_float2(-INFINITY, 0.0f);
        if (s < p.n_pieces) {
            const int64_t blk = static_cast<int64_t>(s) * n_su + su;
            ml[s] = __ldcs(reinterpret_cast<const float2 *>(p.part_ml) + blk * 256 + srow);
            const float4 *po = reinterpret_cast<const float4 *>(p.part_o) + blk * (D / 4) * 256 + (c16 * 4) * 256 + srow;
#pragma unroll
            for (int i = 0; i < 4; ++i) u[s][i] = __ldcs(po + i * 256);
        }
    }
    float m = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) m = fmaxf(m, ml[s].x);
    float a[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = 0.0f;
    float l = 0.0f;
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
        if (s < p.n_pieces) {
            const float w = ml[s].x == -INFINITY ? 0.0f : exp2f(ml[s].x - m);
            l += w * ml[s].y;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[4 * i] += w * u[s][i].x;
                a[4 * i + 1] += w * u[s][i].y;
                a[4 * i + 2] += w * u[s][i].z;
                a[4 * i + 3] += w * u[s][i].w;
            }
        }
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

template <int D, bool F8>
static cudaError_t launch_attention_d(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                                      const CUtensorMap &tv, cudaStream_t s) {
    static bool configured = false;
    const int smem = AttnLayout<D, F8>::kAlloc;
    if (!configured) {
        cudaError_t e =
            cudaFuncSetAttribute(chunk_attention_kernel<D, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (p.n_units == 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>(p.n_whole + (p.n_units - p.n_whole) * p.n_pieces));
    return launch_dependent(chunk_attention_kernel<D, F8>, grid, dim3(kAttnThreads), static_cast<size_t>(smem), s, p,
                            tq, tk, tv);
}

cudaError_t launch_attention(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, int head_dim, cudaStream_t s) {
    if (p.q_scale != nullptr) return launch_attention_d<128, true>(p, tq, tk, tv, s);
    if (head_dim == 64) return launch_attention_d<64, false>(p, tq, tk, tv, s);
    return launch_attention_d<128, false>(p, tq, tk, tv, s);
}

cudaError_t launch_combine(const AttnParams &p, int head_dim, cudaStream_t s) {
    if (p.n_units == p.n_whole) return cudaSuccess;
    const int64_t threads = static_cast<int64_t>(p.n_units - p.n_whole) * (head_dim / 16) * 256;
    const dim3 grid(static_cast<unsigned>((threads + 255) / 256));
    if (head_dim == 64) return launch_dependent(attention_combine_kernel<64>, grid, dim3(256), 0, s, p);
    return launch_dependent(attention_combine_kernel<128>, grid, dim3(256), 0, s, p);
}

cudaError_t launch_rope_q(const AttnParams &p, int sm_count, cudaStream_t s) {
    (void)sm_count;
    int nb = 0;
    for (int i = 0; i < kMaxBatch; ++i)
        if (p.lk[i] > 0) nb = i + 1;
    if (nb == 0) return cudaSuccess;
    const int head_dim = static_cast<int>(p.n_t + p.n_h + p.n_w) * 2;
    const int rows = p.lq * p.heads;
    dim3 grid(static_cast<unsigned>((rows + 63) / 64), static_cast<unsigned>(nb));
    return launch_dependent(rope_q_kernel, grid, dim3(256), 0, s, p, head_dim);
}

}  // namespace sdv2

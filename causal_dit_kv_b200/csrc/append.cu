// KV ring-buffer append with per-frame 3D RoPE on K.
//
// Sources: admirer.cn article on StreamDiffusionV2, method item 1 (sink
// tokens + rolling KV cache); agentlens page "chenfengxu714/StreamDiffusionV2",
// component table (ring buffer for sliding-window attention); qq8o.cn
// walkthrough, "Adaptive sink and RoPE refresh" (periodic RoPE phase reset).
//
// Each frame of the chunk is a contiguous N*H*d block in both the input and
// its ring slot, so the kernel is a 16-byte-vector stream over (K frames,
// V frames).  K vectors are rotated pair by pair in fp64 with
// separately rounded products and sums (no FMA) and rounded once to bf16 by
// cvt.rn.bf16.f64; V vectors are copied.  The temporal cos/sin of each frame
// arrive in the kernel parameters (computed on the host per call); the row
// and column tables live in the cache buffer.
#include "ptx.cuh"

namespace sdv2 {

// K block = 32 (token, head) rows of one frame, 4 threads per row; each thread
// moves every 4th 16-byte vector of its row (4 vectors for d = 128), all loads
// issued before the rotations and stores.  V block = 64 rows, 2 threads per row
// (a copy needs no tables).  grid = (K row blocks, frames of the launch, {K, V});
// the V blocks past the last 64-row block return at once.
constexpr int kAppendRowsPerBlock = 32;

__global__ void __launch_bounds__(128) kv_append_kernel(const __grid_constant__ AppendParams p) {
    // The previous kernel in the stream may still be running (dependent launch):
    // wait for it, then let the next one (the attention kernel, whose set-up and query
    // rotation need nothing this kernel writes) start alongside.
    grid_dependency_wait();
    grid_launch_dependents();
    const int fi = blockIdx.y;
    const bool is_v = blockIdx.z != 0;
    __shared__ double2 s_tab[64];                    // temporal (cos, sin) of this block's frame
    if (!is_v) {
        if (threadIdx.x < p.n_t)
            s_tab[threadIdx.x] = make_double2(p.tab_t[p.tab_row[fi] * p.n_t + threadIdx.x][0],
                                              p.tab_t[p.tab_row[fi] * p.n_t + threadIdx.x][1]);
        __syncthreads();
    }
    const int rows = static_cast<int>(p.frame_elems / p.head_dim);     // N * H
    const int b = p.src_b[fi];
    if (is_v) {
        // V is copied: 2 threads per row, 8 (d = 128) or 4 (d = 64) 16-byte vectors each, all
        // loads in flight before the stores; twice the rows of a K block, so the V blocks
        // need half the threads and the whole launch fits one wave of the GPU
        const int vrow = blockIdx.x * (2 * kAppendRowsPerBlock) + (threadIdx.x >> 1);
        const int vsub = threadIdx.x & 1;
        if (vrow >= rows) return;
        const int64_t vsrc = static_cast<int64_t>(b) * p.chunk_tokens * p.heads * p.head_dim +
                             static_cast<int64_t>(p.src_i[fi]) * p.frame_elems + static_cast<int64_t>(vrow) * p.head_dim;
        const int64_t vdst = (static_cast<int64_t>(b) * p.slots + p.dst_slot[fi]) * p.frame_elems +
                             static_cast<int64_t>(vrow) * p.head_dim;
        constexpr int kMaxV = 8;
        const int nv = p.head_dim / 16;              // vectors per thread: 8 (d = 128) or 4 (d = 64)
        uint4 y[kMaxV];
#pragma unroll
        for (int i = 0; i < kMaxV; ++i)
            if (i < nv) y[i] = ld_nc_v4(p.v_in + vsrc + (vsub + 2 * i) * 8);
#pragma unroll
        for (int i = 0; i < kMaxV; ++i)
            if (i < nv) *reinterpret_cast<uint4 *>(p.v_layer + vdst + (vsub + 2 * i) * 8) = y[i];
        return;
    }
    const int row = blockIdx.x * kAppendRowsPerBlock + (threadIdx.x >> 2);
    const int sub = threadIdx.x & 3;
    if (row >= rows) return;
    const int64_t src = static_cast<int64_t>(b) * p.chunk_tokens * p.heads * p.head_dim +
                        static_cast<int64_t>(p.src_i[fi]) * p.frame_elems + static_cast<int64_t>(row) * p.head_dim;
    const int64_t dst = (static_cast<int64_t>(b) * p.slots + p.dst_slot[fi]) * p.frame_elems +
                        static_cast<int64_t>(row) * p.head_dim;
    constexpr int kMaxVec = 4;                       // d = 128: 16 vectors per row / 4 threads
    const int nvec = p.head_dim / 32;                // vectors per thread: 4 (d = 128) or 2 (d = 64)
    uint4 x[kMaxVec];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i)
        if (i < nvec) x[i] = ld_nc_v4(p.k_in + src + (sub + 4 * i) * 8);
    const int n = row / p.heads;                     // token in the frame
    const int prow = n / p.frame_w;
    const int pcol = n - prow * p.frame_w;
    // (cos, sin) of every pair of this thread's vectors: branch-free addresses so
    // all table loads issue together (the temporal entries come from shared memory)
    const double2 *tab_h = reinterpret_cast<const double2 *>(p.rope_h) + static_cast<int64_t>(prow) * p.n_h - p.n_t;
    const double2 *tab_w =
        reinterpret_cast<const double2 *>(p.rope_w) + static_cast<int64_t>(pcol) * p.n_w - p.n_t - p.n_h;
    double2 cs[kMaxVec][4];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        if (i >= nvec) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = (sub + 4 * i) * 4 + q;
            const double2 *t = j < p.n_t ? &s_tab[j] : (j < p.n_t + p.n_h ? tab_h + j : tab_w + j);
            cs[i][q] = *t;
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        if (i >= nvec) break;
        uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = rotate_pair(w[q], cs[i][q].x, cs[i][q].y);
        *reinterpret_cast<uint4 *>(p.k_layer + dst + (sub + 4 * i) * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// fp8 (E4M3) cache.  Block = one 128-token block of one frame and one head, K
// (blockIdx.z == 0) or V; thread t takes token t/4 of the block and channels
// [32 (t & 3), 32 (t & 3) + 32).  Keys are rotated exactly as above (so the
// quantised values are the bf16 cache's values), the block's largest magnitude
// is reduced over the block, and every value is coded as E4M3(x * 448/amax)
// (fp32 product, nearest even, saturating).  K codes go out token-major; V
// codes are transposed through shared memory into the slot's [H][d][Np] rows.
// Tokens past N in the last block get code 0 and take no part in the maximum.
constexpr int kF8AppendThreads = 512;

__global__ void __launch_bounds__(kF8AppendThreads, 2) kv_append_fp8_kernel(const __grid_constant__ AppendParams p) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int fi = blockIdx.y;
    const bool is_v = blockIdx.z != 0;
    const int h = static_cast<int>(blockIdx.x) % p.heads;
    const int blk = static_cast<int>(blockIdx.x) / p.heads;
    const int tid = threadIdx.x;
    const int tok = tid >> 2, sub = tid & 3;
    const int n = blk * kBlockN + tok;                // token in the frame
    const bool real = n < p.tokens;
    __shared__ double2 s_tab[64];                     // temporal (cos, sin) of this block's frame
    __shared__ float s_max[kF8AppendThreads / 32];
    __shared__ __align__(16) uint8_t s_vt[128][128 + 16];   // V codes, [channel][token]
    if (!is_v && tid < p.n_t)
        s_tab[tid] = make_double2(p.tab_t[p.tab_row[fi] * p.n_t + tid][0], p.tab_t[p.tab_row[fi] * p.n_t + tid][1]);
    __syncthreads();
    const int b = p.src_b[fi];
    const int slot = p.dst_slot[fi];
    uint32_t w[16];                                   // 32 bf16 values, packed pairs (dims 2j, 2j+1)
    if (real) {
        const uint16_t *in = (is_v ? p.v_in : p.k_in) + static_cast<int64_t>(b) * p.chunk_tokens * p.heads * 128 +
                             static_cast<int64_t>(p.src_i[fi]) * p.frame_elems +
                             (static_cast<int64_t>(n) * p.heads + h) * 128 + sub * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 x = ld_nc_v4(in + i * 8);
            w[4 * i] = x.x;
            w[4 * i + 1] = x.y;
            w[4 * i + 2] = x.z;
            w[4 * i + 3] = x.w;
        }
        if (!is_v) {
            const int prow = n / p.frame_w;
            const int pcol = n - prow * p.frame_w;
            const double2 *tab_h = reinterpret_cast<const double2 *>(p.rope_h) + static_cast<int64_t>(prow) * p.n_h - p.n_t;
            const double2 *tab_w =
                reinterpret_cast<const double2 *>(p.rope_w) + static_cast<int64_t>(pcol) * p.n_w - p.n_t - p.n_h;
#pragma unroll
            for (int q0 = 0; q0 < 16; q0 += 4) {             // table loads of 4 pairs in flight at a time
                double2 cs[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = sub * 16 + q0 + q;
                    cs[q] = j < p.n_t ? s_tab[j] : (j < p.n_t + p.n_h ? tab_h[j] : tab_w[j]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) w[q0 + q] = rotate_pair(w[q0 + q], cs[q].x, cs[q].y);
            }
        }
    } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) w[q] = 0u;
    }
    float am = 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q) am = fmaxf(am, fmaxf(fabsf(bf16_lo(w[q])), fabsf(bf16_hi(w[q]))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if ((tid & 31) == 0) s_max[tid >> 5] = am;
    __syncthreads();
    float amax = s_max[0];
#pragma unroll
    for (int i = 1; i < kF8AppendThreads / 32; ++i) amax = fmaxf(amax, s_max[i]);
    float scale, inv;
    e4m3_scale_inv(amax, scale, inv);
    uint32_t c4[8];                                   // 32 codes, 4 per word, channel order
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t lo = pack_e4m3x2(__fmul_rn(bf16_lo(w[2 * q]), inv), __fmul_rn(bf16_hi(w[2 * q]), inv));
        const uint32_t hi =
            pack_e4m3x2(__fmul_rn(bf16_lo(w[2 * q + 1]), inv), __fmul_rn(bf16_hi(w[2 * q + 1]), inv));
        c4[q] = lo | (hi << 16);
    }
    const int64_t bs = static_cast<int64_t>(b) * p.slots + slot;
    if (tid == 0)
        (is_v ? p.v_scale_layer : p.k_scale_layer)[bs * p.scale_slot_stride + h * p.n_blk + blk] = scale;
    if (!is_v) {
        uint8_t *dst = p.k8_layer + ((bs * p.np_tokens + n) * p.heads + h) * 128 + sub * 32;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(c4[0], c4[1], c4[2], c4[3]);
        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(c4[4], c4[5], c4[6], c4[7]);
        return;
    }
    // channel order rotated by sub, so the four channel groups of a warp hit different banks
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int q = (i + sub) & 31;
        s_vt[sub * 32 + q][tok] = static_cast<uint8_t>(c4[q >> 2] >> (8 * (q & 3)));
    }
    __syncthreads();
    uint8_t *dst = p.v8t_layer + (bs * p.heads + h) * 128 * p.np_tokens + blk * kBlockN;
    for (int i = tid; i < 128 * 8; i += kF8AppendThreads) {
        const int r = i >> 3, c = i & 7;
        *reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(r) * p.np_tokens + c * 16) =
            *reinterpret_cast<const uint4 *>(&s_vt[r][c * 16]);
    }
}

cudaError_t launch_append(const AppendParams &p, int sm_count, cudaStream_t s) {
    (void)sm_count;
    if (p.n_frames == 0) return cudaSuccess;
    if (p.k8_layer != nullptr) {
        dim3 grid(static_cast<unsigned>(p.n_blk * p.heads), static_cast<unsigned>(p.n_frames), 2u);
        return launch_dependent(kv_append_fp8_kernel, grid, dim3(kF8AppendThreads), 0, s, p);
    }
    const int rows = static_cast<int>(p.frame_elems / p.head_dim);
    dim3 grid(static_cast<unsigned>((rows + kAppendRowsPerBlock - 1) / kAppendRowsPerBlock),
              static_cast<unsigned>(p.n_frames), 2u);
    return launch_dependent(kv_append_kernel, grid, dim3(4 * kAppendRowsPerBlock), 0, s, p);
}

}  // namespace sdv2

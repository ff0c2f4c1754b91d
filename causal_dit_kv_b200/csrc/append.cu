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

__device__ __forceinline__ uint16_t bf16_from_f64_rn(double x) {
    uint16_t r;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
    return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const uint16_t *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ double bf16_to_f64(uint32_t bits16) {
    return static_cast<double>(__uint_as_float(bits16 << 16));
}

// Rotate one packed pair (lo = dim 2j, hi = dim 2j+1) by (c, s).
__device__ __forceinline__ uint32_t rotate_pair(uint32_t w, double c, double s) {
    const double x0 = bf16_to_f64(w & 0xFFFFu);
    const double x1 = bf16_to_f64(w >> 16);
    const double r0 = __dsub_rn(__dmul_rn(x0, c), __dmul_rn(x1, s));
    const double r1 = __dadd_rn(__dmul_rn(x0, s), __dmul_rn(x1, c));
    return static_cast<uint32_t>(bf16_from_f64_rn(r0)) | (static_cast<uint32_t>(bf16_from_f64_rn(r1)) << 16);
}

// Block = 32 (token, head) rows of one frame, 4 threads per row; each thread
// moves every 4th 16-byte vector of its row (4 vectors for d = 128), all
// loads issued before the rotations and stores.  grid = (row blocks, frames
// of the launch, {K, V}).
constexpr int kAppendRowsPerBlock = 32;

__global__ void __launch_bounds__(128) kv_append_kernel(const __grid_constant__ AppendParams p) {
    // The previous kernel in the stream may still be running (dependent launch):
    // wait for it, then let the next one (the queries' RoPE) start alongside.
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
    const int row = blockIdx.x * kAppendRowsPerBlock + (threadIdx.x >> 2);
    const int sub = threadIdx.x & 3;
    if (row >= rows) return;
    const int b = p.src_b[fi];
    const int64_t src = static_cast<int64_t>(b) * p.chunk_tokens * p.heads * p.head_dim +
                        static_cast<int64_t>(p.src_i[fi]) * p.frame_elems + static_cast<int64_t>(row) * p.head_dim;
    const int64_t dst = (static_cast<int64_t>(b) * p.slots + p.dst_slot[fi]) * p.frame_elems +
                        static_cast<int64_t>(row) * p.head_dim;
    constexpr int kMaxVec = 4;                       // d = 128: 16 vectors per row / 4 threads
    const int nvec = p.head_dim / 32;                // vectors per thread: 4 (d = 128) or 2 (d = 64)
    uint4 x[kMaxVec];
    const uint16_t *in = is_v ? p.v_in : p.k_in;
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i)
        if (i < nvec) x[i] = ld_nc_v4(in + src + (sub + 4 * i) * 8);
    if (is_v) {
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i)
            if (i < nvec) *reinterpret_cast<uint4 *>(p.v_layer + dst + (sub + 4 * i) * 8) = x[i];
        return;
    }
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

cudaError_t launch_append(const AppendParams &p, int sm_count, cudaStream_t s) {
    (void)sm_count;
    if (p.n_frames == 0) return cudaSuccess;
    const int rows = static_cast<int>(p.frame_elems / p.head_dim);
    dim3 grid(static_cast<unsigned>((rows + kAppendRowsPerBlock - 1) / kAppendRowsPerBlock),
              static_cast<unsigned>(p.n_frames), 2u);
    return launch_dependent(kv_append_kernel, grid, dim3(4 * kAppendRowsPerBlock), 0, s, p);
}

}  // namespace sdv2

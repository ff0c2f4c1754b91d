// KV ring-buffer append with per-frame 3D RoPE on K.
//
// Sources: admirer.cn article on StreamDiffusionV2, method item 1 (sink
// tokens + rolling KV cache); agentlens page "chenfengxu714/StreamDiffusionV2",
// component table (ring buffer for sliding-window attention); qq8o.cn
// walkthrough, "Adaptive sink and RoPE refresh" (periodic RoPE phase reset).
//
// Each frame of the chunk is a contiguous N*H*d block in both the input and
// its ring slot, so the kernel is a flat 16-byte-vector stream over
// (K frames, V frames).  K vectors are rotated pair by pair in fp64 with
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

__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams p) {
    const uint32_t vec_per_frame = static_cast<uint32_t>(p.frame_elems / 8);
    const uint32_t k_vectors = static_cast<uint32_t>(p.n_frames) * vec_per_frame;
    const uint32_t total = 2u * k_vectors;
    const uint32_t hd = static_cast<uint32_t>(p.heads * p.head_dim);
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < total; g += gridDim.x * blockDim.x) {
        const bool is_v = g >= k_vectors;
        const uint32_t r = is_v ? g - k_vectors : g;
        const uint32_t fi = r / vec_per_frame;
        const uint32_t vec = r - fi * vec_per_frame;
        const int b = p.src_b[fi];
        const int64_t src = static_cast<int64_t>(b) * p.chunk_tokens * hd +
                            static_cast<int64_t>(p.src_i[fi]) * p.frame_elems + static_cast<int64_t>(vec) * 8;
        const int64_t dst = (static_cast<int64_t>(b) * p.slots + p.dst_slot[fi]) * p.frame_elems +
                            static_cast<int64_t>(vec) * 8;
        if (is_v) {
            const uint4 x = ld_nc_v4(p.v_in + src);
            *reinterpret_cast<uint4 *>(p.v_layer + dst) = x;
            continue;
        }
        uint4 x = ld_nc_v4(p.k_in + src);
        const uint32_t e = vec * 8;
        const uint32_t n = e / hd;                       // token in the frame
        const uint32_t dd = e - n * hd;
        const uint32_t j0 = (dd % static_cast<uint32_t>(p.head_dim)) >> 1;   // first pair of the vector
        const uint32_t row = n / static_cast<uint32_t>(p.frame_w);
        const uint32_t col = n - row * static_cast<uint32_t>(p.frame_w);
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = static_cast<int>(j0) + q;
            double c, s;
            if (j < p.n_t) {
                c = p.tab_t[fi * p.n_t + j][0];
                s = p.tab_t[fi * p.n_t + j][1];
            } else if (j < p.n_t + p.n_h) {
                const double *t = p.rope_h + 2 * (static_cast<int64_t>(row) * p.n_h + (j - p.n_t));
                c = t[0];
                s = t[1];
            } else {
                const double *t = p.rope_w + 2 * (static_cast<int64_t>(col) * p.n_w + (j - p.n_t - p.n_h));
                c = t[0];
                s = t[1];
            }
            w[q] = rotate_pair(w[q], c, s);
        }
        *reinterpret_cast<uint4 *>(p.k_layer + dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

cudaError_t launch_append(const AppendParams &p, int sm_count, cudaStream_t s) {
    const uint64_t total = 2ull * static_cast<uint64_t>(p.n_frames) * static_cast<uint64_t>(p.frame_elems / 8);
    if (total == 0) return cudaSuccess;
    uint64_t blocks = (total + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(sm_count) * 8;
    if (blocks > cap) blocks = cap;
    kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace sdv2

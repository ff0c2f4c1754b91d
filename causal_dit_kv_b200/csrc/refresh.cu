// Adaptive sink refresh: chunk-mean embedding, cosine against the sink set,
// device-side decision, predicated copy of the chunk's last frame K/V.
//
// Source: qq8o.cn walkthrough of StreamDiffusionV2, "Adaptive sink and RoPE
// refresh" (compare the new chunk embedding with the sink set by cosine
// similarity; replace the least similar sink when the similarity falls
// below the threshold tau).
//
// Kernel 1, grid (column blocks, token chunks, B): block (x, r, b) sums 256
// columns of the hidden states over token chunk r in fp64 (warp w takes
// tokens w, w+8, ...; lane l takes columns 8l..8l+7 with one 16-byte load per
// token; fixed-order reduction across warps).  The number of token chunks is
// chosen per cache so the grid covers the GPU about twice.  The last block of stream b (atomic ticket) adds the chunk
// sums in chunk order, divides by the token count, computes the dot products
// and norms in fp64, takes the decision, updates the sink embedding and the
// sink-frame record, and writes out_slot[b].
// Kernel 2, two blocks per SM: for every stream b with out_slot[b] >= 0, copies
// slot last_slot[b] to slot out_slot[b] in every layer, K and V (for the fp8
// cache: K and V codes and their block scales), as 16-byte vectors spread over
// all blocks; streams without a refresh are skipped.
#include <cmath>

#include "ptx.cuh"

namespace sdv2 {

constexpr int kRefreshThreads = 256;
constexpr int kRefreshCols = 256;                 // 8 per lane

__device__ __forceinline__ uint4 ld_stream_v4(const uint16_t *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ double block_sum_fixed(double v, double *red) {
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < kRefreshThreads / 32; ++w) s += red[w];
    return s;
}

__global__ void __launch_bounds__(kRefreshThreads) refresh_decide_kernel(const __grid_constant__ RefreshParams p) {
    // Launched as a dependent of the last layer's attention: the column sums read only
    // the caller's hidden states and this call's scratch, so they start at once; the
    // kernel waits for its predecessor before it touches what later kernels read (the
    // decision), and lets the copy kernel launch early (it waits for this grid).
    grid_launch_dependents();
    const int b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!p.active[b]) {
        grid_dependency_wait();
        if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) p.out_slot[b] = -1;
        return;
    }
    __shared__ double part[kRefreshThreads / 32][kRefreshCols];
    __shared__ double red[kRefreshThreads / 32];
    __shared__ int is_last;

    // column sums of this block's 256 columns over its chunk of tokens
    const int col0 = blockIdx.x * kRefreshCols + 8 * lane;
    const int t_begin = static_cast<int>((static_cast<int64_t>(p.lq) * blockIdx.y) / p.row_chunks);
    const int t_end = static_cast<int>((static_cast<int64_t>(p.lq) * (blockIdx.y + 1)) / p.row_chunks);
    const uint16_t *hb = p.hidden + static_cast<int64_t>(b) * p.lq * p.dim;
    double a[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = 0.0;
    if (col0 < p.dim) {
        if ((p.dim & 7) == 0) {                      // rows are 16-byte aligned: one vector per token
#pragma unroll 4
            for (int t = t_begin + warp; t < t_end; t += kRefreshThreads / 32) {
                const uint4 w = ld_stream_v4(hb + static_cast<int64_t>(t) * p.dim + col0);
                const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    a[2 * q] += static_cast<double>(bf16_lo(v[q]));
                    a[2 * q + 1] += static_cast<double>(bf16_hi(v[q]));
                }
            }
        } else {
            for (int t = t_begin + warp; t < t_end; t += kRefreshThreads / 32)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (col0 + j < p.dim)
                        a[j] += static_cast<double>(
                            __uint_as_float(static_cast<uint32_t>(hb[static_cast<int64_t>(t) * p.dim + col0 + j]) << 16));
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) part[warp][8 * lane + j] = a[j];
    __syncthreads();
    {
        const int c = blockIdx.x * kRefreshCols + tid;
        if (c < p.dim) {
            double sum = 0.0;
            for (int w = 0; w < kRefreshThreads / 32; ++w) sum += part[w][tid];
            p.partial[(static_cast<int64_t>(b) * p.row_chunks + blockIdx.y) * p.dim + c] = sum;
        }
    }
    // Two-level merge.  The last block of each column block adds that block's 256
    // column sums over the token chunks (in chunk order) and leaves the chunk mean
    // in place of token chunk 0's sums; the last column block of the stream then
    // takes the decision.
    uint32_t *col_counter = p.counter + kMaxBatch + static_cast<int64_t>(b) * kRefreshMaxColBlocks + blockIdx.x;
    grid_dependency_wait();
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(col_counter, 1u) == gridDim.y - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    double *pb = p.partial + static_cast<int64_t>(b) * p.row_chunks * p.dim;
    {
        const int c = blockIdx.x * kRefreshCols + tid;
        if (c < p.dim) {
            // all chunk sums of the column in flight at once, then added in chunk order
            double v[kRefreshMaxChunks];
#pragma unroll
            for (int r = 0; r < kRefreshMaxChunks; ++r)
                v[r] = r < p.row_chunks ? __ldcg(pb + static_cast<int64_t>(r) * p.dim + c) : 0.0;
            double sum = 0.0;
#pragma unroll
            for (int r = 0; r < kRefreshMaxChunks; ++r) sum += v[r];
            pb[c] = sum / static_cast<double>(p.lq);
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        *col_counter = 0u;
        is_last = atomicAdd(p.counter + b, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // last column block of stream b: the chunk mean h is in pb[0 .. D), then the decision
    auto mean_at = [&](int c) { return __ldcg(pb + c); };
    double *emb = p.sink_embed + static_cast<int64_t>(b) * p.sinks * p.dim;
    if (p.fill_count[b] > 0) {
        // The chunk fills sink slots itself: record their embedding only.
        for (int c = tid; c < p.dim; c += kRefreshThreads) {
            const double h = mean_at(c);
            for (int j = p.fill_first[b]; j < p.fill_first[b] + p.fill_count[b]; ++j)
                emb[static_cast<int64_t>(j) * p.dim + c] = h;
        }
        if (tid == 0) {
            for (int j = p.fill_first[b]; j < p.fill_first[b] + p.fill_count[b]; ++j)
                p.sink_frame[static_cast<int64_t>(b) * p.sinks + j] = j;
            p.out_slot[b] = -1;
            p.counter[b] = 0u;
        }
        return;
    }
    // h is consumed column by column; each thread keeps its columns' values
    constexpr int kMaxColsPerThread = 64;          // embed_dim <= 16384
    double hv[kMaxColsPerThread];
    double hh = 0.0;
    int k = 0;
    for (int c = tid; c < p.dim && k < kMaxColsPerThread; c += kRefreshThreads, ++k) {
        hv[k] = mean_at(c);
        hh += hv[k] * hv[k];
    }
    hh = block_sum_fixed(hh, red);
    double best = 0.0;
    int best_j = -1;
    for (int j = 0; j < p.sinks; ++j) {
        double he = 0.0, ee = 0.0;
        k = 0;
        for (int c = tid; c < p.dim && k < kMaxColsPerThread; c += kRefreshThreads, ++k) {
            const double e = emb[static_cast<int64_t>(j) * p.dim + c];
            he += hv[k] * e;
            ee += e * e;
        }
        he = block_sum_fixed(he, red);
        ee = block_sum_fixed(ee, red);
        const double cj = (hh == 0.0 || ee == 0.0) ? 1.0 : he / (sqrt(hh) * sqrt(ee));
        if (best_j < 0 || cj < best) {   // strict: the lowest index wins ties
            best = cj;
            best_j = j;
        }
    }
    const bool fire = best < p.tau;
    __syncthreads();
    if (fire) {
        k = 0;
        for (int c = tid; c < p.dim && k < kMaxColsPerThread; c += kRefreshThreads, ++k)
            emb[static_cast<int64_t>(best_j) * p.dim + c] = hv[k];
    }
    if (tid == 0) {
        if (fire) p.sink_frame[static_cast<int64_t>(b) * p.sinks + best_j] = p.last_frame[b];
        p.out_slot[b] = fire ? best_j : -1;
        p.counter[b] = 0u;
    }
}

__global__ void __launch_bounds__(256) refresh_copy_kernel(const __grid_constant__ RefreshParams p) {
    grid_dependency_wait();                     // the decision, and every earlier kernel's reads of the slots
    grid_launch_dependents();
    // Every block takes a share of every refreshed stream's copy (streams whose decision
    // was "no refresh" cost one load of out_slot), four 16-byte vectors in flight per thread.
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int b = 0; b < p.batch; ++b) {
        if (!p.active[b] || p.fill_count[b] > 0) continue;
        const int dst_slot = *reinterpret_cast<volatile const int32_t *>(p.out_slot + b);
        if (dst_slot < 0) continue;
        const int src_slot = p.last_slot[b];
        for (int r = 0; r < p.n_copy; ++r) {
            const int64_t vec_per_slot = p.copy_slot_bytes[r] / 16;
            const int64_t total = static_cast<int64_t>(p.layers) * vec_per_slot;
            for (int64_t g0 = gid; g0 < total; g0 += 4 * nthreads) {
                uint4 x[4];
                uint4 *dst[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t g = g0 + u * nthreads;
                    if (g < total) {
                        const int64_t layer = g / vec_per_slot;
                        const int64_t vec = g - layer * vec_per_slot;
                        uint8_t *lb = p.copy_base[r] + layer * p.copy_layer_bytes[r] +
                                      static_cast<int64_t>(b) * p.slots * p.copy_slot_bytes[r];
                        x[u] = *reinterpret_cast<const uint4 *>(lb + src_slot * p.copy_slot_bytes[r] + vec * 16);
                        dst[u] = reinterpret_cast<uint4 *>(lb + dst_slot * p.copy_slot_bytes[r] + vec * 16);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (g0 + u * nthreads < total) *dst[u] = x[u];
            }
        }
    }
}

cudaError_t launch_refresh(const RefreshParams &p, int sm_count, cudaStream_t s, int *launches) {
    dim3 g1(static_cast<unsigned>((p.dim + kRefreshCols - 1) / kRefreshCols), static_cast<unsigned>(p.row_chunks),
            static_cast<unsigned>(p.batch));
    cudaError_t e = launch_dependent(refresh_decide_kernel, g1, dim3(kRefreshThreads), 0, s, p);
    if (e != cudaSuccess) return e;
    dim3 g2(static_cast<unsigned>(sm_count > 0 ? 2 * sm_count : 296));
    *launches = 2;
    return launch_dependent(refresh_copy_kernel, g2, dim3(256), 0, s, p);
}

}  // namespace sdv2

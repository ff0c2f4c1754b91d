// Motion-aware noise rate: frame-difference RMS, k-frame maximum, clip and EMA.
//
// Sources: admirer.cn article on StreamDiffusionV2, method item 2 (motion
// strength from the L2 distance of adjacent frames; more motion -> less
// noise); qq8o.cn walkthrough, "Motion-aware noise scheduler" (normalise by
// a statistical scale over a short k-frame window, clip to [0, 1], EMA with
// 0 < lambda < 1 between s_min and s_max).
//
// One launch per call.  Block (x, b) owns a contiguous slice of the latent
// frame of stream b (2048 elements, read as 16-byte vectors when the frame
// size and the latents allow it): it sums squared differences of that slice
// for every frame of the chunk in fp64 (warp-shuffle, then fixed-order
// reduction across warps), writes one partial per frame, then overwrites
// the slice of the stored previous frame with the chunk's last frame (only
// this block touches that slice, so no ordering across blocks is needed).
// The last block of a stream to finish (counted with an atomic ticket) sums
// the partials (one warp, lanes over blocks, then a fixed butterfly) and runs
// the recurrence in fp64.
#include <cmath>

#include "ptx.cuh"

namespace sdv2 {

__global__ void __launch_bounds__(kMotionThreads) motion_kernel(const __grid_constant__ MotionParams p) {
    // Launched as a dependent of the step's last kernel: the motion state is written only
    // by this kernel (whose previous launch completed before this step's first kernel), so
    // the work needs nothing from the kernel before it.  Every thread still waits for that
    // kernel before it exits, so that this grid completes only after it (later kernels of
    // the stream rely on that order).
    grid_launch_dependents();
    const int b = blockIdx.y;
    const int blk = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t n = p.frame_elems;
    const int64_t begin = static_cast<int64_t>(blk) * kMotionBlockElems;
    const int64_t end = begin + kMotionBlockElems < n ? begin + kMotionBlockElems : n;
    const float *x = p.latents + static_cast<int64_t>(b) * p.chunk_frames * n;
    float *prev = p.prev + static_cast<int64_t>(b) * n;
    const bool had_prev = p.has_prev[b] != 0;

    __shared__ double red[kMotionThreads / 32];
    __shared__ int is_last;
    // 16-byte vectors when every frame starts on a 16-byte boundary (block slices are
    // multiples of 2048 elements, so they do too)
    const bool vec = (n & 3) == 0 && (reinterpret_cast<uintptr_t>(p.latents) & 15u) == 0;

    for (int t = 0; t < p.chunk_frames; ++t) {
        double acc = 0.0;
        if (t > 0 || had_prev) {
            const float *cur = x + static_cast<int64_t>(t) * n;
            const float *before = t == 0 ? prev : x + static_cast<int64_t>(t - 1) * n;
            if (vec) {
                const float4 *c4 = reinterpret_cast<const float4 *>(cur);
                const float4 *b4 = reinterpret_cast<const float4 *>(before);
#pragma unroll 2
                for (int64_t e = begin / 4 + tid; e < end / 4; e += kMotionThreads) {
                    const float4 u = __ldcs(c4 + e), v = __ldcg(b4 + e);
                    const double d0 = static_cast<double>(u.x) - static_cast<double>(v.x);
                    const double d1 = static_cast<double>(u.y) - static_cast<double>(v.y);
                    const double d2 = static_cast<double>(u.z) - static_cast<double>(v.z);
                    const double d3 = static_cast<double>(u.w) - static_cast<double>(v.w);
                    acc += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
                }
            } else {
                for (int64_t e = begin + tid; e < end; e += kMotionThreads) {
                    const double dlt = static_cast<double>(cur[e]) - static_cast<double>(before[e]);
                    acc += dlt * dlt;
                }
            }
        }
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if ((tid & 31) == 0) red[tid >> 5] = acc;
        __syncthreads();
        if (tid == 0) {
            double s = 0.0;
            for (int w = 0; w < kMotionThreads / 32; ++w) s += red[w];
            p.partial[(static_cast<int64_t>(b) * p.chunk_frames + t) * p.n_blocks + blk] = s;
        }
        __syncthreads();
    }
    // This block's slice of the previous frame is no longer needed: replace it.
    const float *last = x + static_cast<int64_t>(p.chunk_frames - 1) * n;
    if (vec) {
        const float4 *l4 = reinterpret_cast<const float4 *>(last);
        float4 *p4 = reinterpret_cast<float4 *>(prev);
        for (int64_t e = begin / 4 + tid; e < end / 4; e += kMotionThreads) p4[e] = __ldcg(l4 + e);
    } else {
        for (int64_t e = begin + tid; e < end; e += kMotionThreads) prev[e] = last[e];
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned ticket = atomicAdd(p.counter + b, 1u);
        is_last = ticket == static_cast<unsigned>(p.n_blocks - 1);
    }
    __syncthreads();
    if (!is_last || tid >= 32) {
        grid_dependency_wait();
        return;
    }
    __threadfence();

    // The last block's first warp: every lane sums the partials i = lane, lane + 32, ...
    // of each frame (all loads in flight at once), then a fixed butterfly adds the lanes.
    double ss_frame[kMotionMaxFrames];
    for (int t = 0; t < p.chunk_frames; ++t) {
        const double *part = p.partial + (static_cast<int64_t>(b) * p.chunk_frames + t) * p.n_blocks;
        double ss = 0.0;
        for (int i = tid; i < p.n_blocks; i += 32) ss += __ldcg(part + i);
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (t < kMotionMaxFrames) ss_frame[t] = ss;
    }
    if (tid != 0) {
        grid_dependency_wait();
        return;
    }
    double rate = p.rate[b];
    int len = p.hist_len[b];
    int pos = p.hist_pos[b];
    double *hist = p.hist + static_cast<int64_t>(b) * p.window;
    bool have = had_prev;
    for (int t = 0; t < p.chunk_frames; ++t) {
        float d_out = -1.0f;
        if (have) {
            const double d = sqrt(ss_frame[t] / static_cast<double>(n));
            hist[pos] = d;
            pos = (pos + 1) % p.window;
            if (len < p.window) ++len;
            double dbar = hist[0];
            for (int i = 1; i < len; ++i) dbar = fmax(dbar, hist[i]);
            double dhat = dbar / p.sigma;
            dhat = dhat < 0.0 ? 0.0 : (dhat > 1.0 ? 1.0 : dhat);
            const double target = p.s_max - (p.s_max - p.s_min) * dhat;
            rate = p.lambda * target + (1.0 - p.lambda) * rate;
            d_out = static_cast<float>(d);
        }
        have = true;
        if (p.out_d) p.out_d[static_cast<int64_t>(b) * p.chunk_frames + t] = d_out;
    }
    p.rate[b] = rate;
    p.hist_len[b] = len;
    p.hist_pos[b] = pos;
    p.has_prev[b] = 1;
    p.out_rate[b] = static_cast<float>(rate);
    p.counter[b] = 0u;
    grid_dependency_wait();
}

cudaError_t launch_motion(const MotionParams &p, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(p.n_blocks), static_cast<unsigned>(p.batch));
    return launch_dependent(motion_kernel, grid, dim3(kMotionThreads), 0, s, p);
}

}  // namespace sdv2

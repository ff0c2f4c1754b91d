// Allocation-free variant of the motion noise-rate launch.
//
// sdv2_motion_noise_rate keeps its per-call scratch (one fp64 partial sum per
// block and frame, one ticket counter per stream) inside the caller's motion
// buffer.  This variant keeps that scratch in a fixed device array owned by
// the library instead, so a caller that cannot allocate device memory at the
// point of the call never has to provide it.  The array is created when the
// library is loaded and every GPU that loads the library holds it until the
// process exits.
#include <mutex>

#include "ptx.cuh"
#include "sdv2_internal.h"

namespace sdv2 {

// Capacity: kNoAllocPartials fp64 partial sums (batch * chunk_frames * blocks
// per frame) followed by kMaxBatch ticket counters.  128 KB + 256 B.
constexpr int kNoAllocPartials = 16384;
constexpr size_t kNoAllocCounterOffset = static_cast<size_t>(kNoAllocPartials) * sizeof(double);
constexpr size_t kNoAllocBytes = kNoAllocCounterOffset + kMaxBatch * sizeof(uint32_t);

static __device__ __align__(256) unsigned char g_motion_scratch[kNoAllocBytes];

// Device address of g_motion_scratch for the current device, looked up once
// per device (host code cannot use the symbol itself as a device pointer).
static cudaError_t scratch_address(void **out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_motion_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

int motion_noalloc_max_partials() { return kNoAllocPartials; }

cudaError_t launch_motion_noalloc(MotionParams p, cudaStream_t s) {
    void *base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) return e;
    p.partial = static_cast<double *>(base);
    p.counter = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(base) + kNoAllocCounterOffset);
    // The tickets must start at zero; the array keeps whatever the last call left.
    e = cudaMemsetAsync(p.counter, 0, sizeof(uint32_t) * static_cast<size_t>(p.batch), s);
    if (e != cudaSuccess) return e;
    return launch_motion(p, s);
}

}  // namespace sdv2

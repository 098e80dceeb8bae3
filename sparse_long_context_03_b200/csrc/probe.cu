// probe.cu -- a streaming read kernel used only to measure the memory
// system's read bandwidth (the roofline denominators): reading a buffer that
// fits in L2 over and over gives the L2 read bandwidth, one pass over a
// buffer much larger than L2 gives the HBM read bandwidth.  Not part of the
// DSA layer.
//
// Loads are 16-byte ld.global.cg (cached in L2 only, not in L1), the access
// pattern of the attention's cp.async.cg gathers, eight in flight per thread.
#include "kernels.h"

namespace dsa {

namespace {

__device__ __forceinline__ uint4 ld_cg_16(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kProbeThreads = 512;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(kProbeThreads) read_probe_kernel(const uint4 *__restrict__ buf, size_t n16, int reps,
                                                                  uint32_t *__restrict__ sink) {
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * kProbeThreads;
    for (int r = 0; r < reps; ++r) {
        size_t i = (size_t)blockIdx.x * kProbeThreads + threadIdx.x;
        for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) v[u] = ld_cg_16(buf + i + u * stride);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
        }
        for (; i < n16; i += stride) {
            const uint4 v = ld_cg_16(buf + i);
            acc ^= v.x ^ v.y ^ v.z ^ v.w;
        }
    }
    // every load feeds acc, and acc is stored when it takes one particular
    // value, so the compiler cannot drop the loads
    if (acc == 0xFFFFFFFFu) sink[0] = acc;
}

}  // namespace

cudaError_t launch_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink, cudaStream_t stream) {
    const size_t n16 = bytes / 16;
    if (n16 == 0 || reps <= 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (sms > 0 ? sms : 148) * 4;  // four 512-thread CTAs per SM
    read_probe_kernel<<<grid, kProbeThreads, 0, stream>>>(static_cast<const uint4 *>(buf), n16, reps, sink);
    return cudaGetLastError();
}

}  // namespace dsa

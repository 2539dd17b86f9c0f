// Read-bandwidth probe: streams a buffer with 16-byte loads from every SM and
// folds it into a checksum.  A measurement utility for the roofline
// denominators of the scan: run over page-locked host memory it measures the
// host link as the scan uses it (SM loads over the link, no copy engine);
// over device memory, HBM read bandwidth.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads)
probe_kernel(const uint4* __restrict__ src, size_t n16, unsigned long long* sink) {
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * kThreads;
    size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
        uint4 v = __ldcs(src + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0 && acc) atomicXor(sink, (unsigned long long)acc);
}

}  // namespace

cudaError_t launch_probe(const void* src, size_t bytes, unsigned long long* sink, int ctas, cudaStream_t stream) {
    probe_kernel<<<ctas, kThreads, 0, stream>>>(static_cast<const uint4*>(src), bytes / 16, sink);
    return cudaGetLastError();
}

}  // namespace fathom

// stream_probe.cu — a plain read-only stream over device memory.
//
// The select reads about five hundred bytes for every byte it writes, so the
// copy bandwidth (a read and a write of every byte) understates what it can
// reach; this stream is the read-only figure to set beside it.  Every thread
// keeps eight 16-byte loads in flight (evict-first), four blocks per SM; the
// words read are XOR-ed into one word, which keeps every load live and lets a
// test check that the whole buffer was read.
#include "wc_common.cuh"
#include "wc_internal.h"

namespace wc {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeUnroll = 8;

__global__ void __launch_bounds__(kProbeThreads) read_stream_kernel(const uint4* __restrict__ p, int64_t n16,
                                                                   uint32_t* sink) {
    uint32_t acc = 0;
    const int64_t stride = (int64_t)gridDim.x * kProbeThreads;
    int64_t i = (int64_t)blockIdx.x * kProbeThreads + threadIdx.x;
    for (; i + (kProbeUnroll - 1) * stride < n16; i += kProbeUnroll * stride) {
        uint4 v[kProbeUnroll];
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) v[u] = __ldcs(p + i + u * stride);
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
        const uint4 v = __ldcs(p + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace

wc_status launch_read_probe(const void* buf, int64_t bytes, uint32_t* sink, cudaStream_t st) {
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WC_ERR_CUDA;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return WC_ERR_CUDA;
    if (cudaMemsetAsync(sink, 0, sizeof(uint32_t), st) != cudaSuccess) return WC_ERR_CUDA;
    read_stream_kernel<<<nsm * 4, kProbeThreads, 0, st>>>(static_cast<const uint4*>(buf), bytes / 16, sink);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace wc

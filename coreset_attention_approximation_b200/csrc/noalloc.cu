// noalloc.cu — coreset attention for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// running under an allocator that must not be re-entered, a host process
// whose memory budget is fixed before the first call, or a plugin that only
// receives its input and output tensors.  wc_attend_noalloc serves them: the
// attention step's scratch lives in a fixed array in device memory that
// belongs to the library, so the call allocates nothing.
//
// The array below is a file-scope __device__ symbol.  Host code cannot use
// its name as a device address (in host code it names a host-side stand-in),
// so the first call on each device looks its address up with
// cudaGetSymbolAddress, with that device current, and hands the address to
// the kernels.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "wc_common.cuh"
#include "wc_expmm.cuh"
#include "wc_internal.h"

namespace wc {
namespace {

constexpr size_t kNoAllocScratch = size_t(16) << 20;  // 16 MiB per device, held until exit

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratch];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
std::atomic<unsigned char*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (set up once per device).
wc_status scratch_on_current_device(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WC_ERR_CUDA;
    unsigned char* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return WC_ERR_CUDA;
            p = static_cast<unsigned char*>(addr);
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return WC_OK;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace wc

using namespace wc;

extern "C" wc_status wc_attend_noalloc(const wc_shape* shape, const void* Q, const void* Ks, const float* W,
                                       const int32_t* rank, float* out, void* stream) {
    Shape s;
    wc_status e = make_shape(shape, &s);
    if (e != WC_OK) return e;
    if (s.nq == 0) return WC_OK;
    if (!Q || !Ks || !W || !rank || !out) return WC_ERR_INVALID;
    auto a16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
    if (!a16(Q) || !a16(Ks) || !a16(W) || !a16(out)) return WC_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!tc_supported(s)) {
        // the CUDA-core kernel needs no scratch at all
        return launch_attend(s, Q, Ks, W, rank, out, nullptr, st);
    }
    // scratch: status word | fp16 weights | column scales | normaliser column
    const size_t o_w16 = 256;
    const size_t o_sigma = o_w16 + up256((size_t)2 * s.units * s.r * s.dv);
    const size_t o_wn = o_sigma + up256(sizeof(float) * (size_t)s.units * s.dv);
    const size_t need = o_wn + up256(sizeof(float) * (size_t)s.units * s.r_pad);
    if (need > kNoAllocScratch) return WC_ERR_WORKSPACE;
    unsigned char* base = nullptr;
    if ((e = scratch_on_current_device(&base)) != WC_OK) return e;
    int* status = reinterpret_cast<int*>(base);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return WC_ERR_CUDA;
    return launch_attend_tc_at(s, Q, Ks, W, rank, out, status, reinterpret_cast<__half*>(base + o_w16),
                               reinterpret_cast<float*>(base + o_sigma), reinterpret_cast<float*>(base + o_wn), st);
}

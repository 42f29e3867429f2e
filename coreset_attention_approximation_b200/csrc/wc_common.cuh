// wc_common.cuh — device helpers shared by the WildCat kernels (sm_100a).
//
// Status word, the debug build's bounds checks, bounded waits, the
// Philox4x32-10 counter generator (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC'11) and element loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wildcat.h"

namespace wc {

// ------------------------------------------------------------------ status

// First error recorded on the device wins; later ones are dropped.
__device__ __forceinline__ void record_status(int* status, int code) {
    atomicCAS(status, 0, code);
}

// Bounds checks of data-dependent indices (pivots, ranks), compiled in with
// -DWC_DEBUG_BOUNDS=1 (libwildcat_debug.so): a failed check records
// WC_ERR_BOUNDS and the caller skips the access.  In the release build every
// check is `true` and costs nothing.
#ifndef WC_DEBUG_BOUNDS
#define WC_DEBUG_BOUNDS 0
#endif
__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
#if WC_DEBUG_BOUNDS
    if (!ok && status) record_status(status, WC_ERR_BOUNDS);
    return ok;
#else
    (void)ok;
    (void)status;
    return true;
#endif
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_volatile_i32(const int* p) {
    return *(const volatile int*)p;
}

// Spin until *ctr >= target.  Gives up when `timeout_ns` has passed since the
// wait began (records WC_ERR_TIMEOUT) or when another block already recorded
// an error.  Returns true when the target was reached.  One thread calls it.
__device__ __forceinline__ bool wait_geq(const uint32_t* ctr, uint32_t target, uint64_t timeout_ns,
                                         int* status) {
    const uint64_t t0 = global_ns();
    uint32_t backoff = 32;
    for (uint64_t it = 0;; ++it) {
        if (ld_acquire_u32(ctr) >= target) return true;
        if (ld_volatile_i32(status) != 0) return false;
        if ((it & 15) == 15 && global_ns() - t0 > timeout_ns) {
            record_status(status, WC_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(backoff);
        if (backoff < 1024) backoff <<= 1;
    }
}

// Barrier among the `nblocks` thread blocks of one unit.  `ctr` counts
// arrivals over the whole launch; the e-th barrier (e = 1, 2, ...) waits for
// nblocks * e.  All threads of the block call it; the block's global writes
// before the call are visible to the unit's other blocks after it.
__device__ __forceinline__ bool unit_barrier(uint32_t* ctr, uint32_t nblocks, uint32_t epoch,
                                             uint64_t timeout_ns, int* status, int* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        *s_ok = wait_geq(ctr, nblocks * epoch, timeout_ns, status) ? 1 : 0;
        __threadfence();
    }
    __syncthreads();
    return *s_ok != 0;
}

// ------------------------------------------------------------------ Philox

// Philox4x32-10: ten rounds of two 32x32 -> 64-bit products whose high halves
// are xored into the other two words together with the round key; the key
// advances by the Weyl constants (golden ratio, sqrt(3) - 1) between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

// u_j in [0, 1): first output word of counter (j, unit, 0, 0) over 2^32.
__device__ __forceinline__ double pivot_uniform(uint64_t seed, uint32_t j, uint32_t unit) {
    const uint4 o = philox4x32_10(make_uint4(j, unit, 0u, 0u),
                                  make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
    return (double)o.x * 0x1p-32;
}

// ------------------------------------------------------------------ loads

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Load that bypasses L1 (data another block wrote during this launch).
__device__ __forceinline__ float ld_cg_f32(const float* p) { return __ldcg(p); }

}  // namespace wc

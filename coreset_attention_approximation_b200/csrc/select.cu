// select.cu — randomly pivoted Cholesky on H = exp(beta K K^T), one persistent
// launch per wave of units.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gist.science
// technical summary, "Methodik" item 1): a partial Cholesky factorisation of
// the exponential kernel matrix whose pivot at every step is drawn from the
// diagonal of the current residual matrix.
//
// The factorisation runs on exp(beta K K^T - M), M = max_i beta |k_i|^2 over
// the unit: the kernel times a positive constant, so the pivot draws (ratios of
// the residual diagonal) and the stop rule (relative to the diagonal's
// maximum, now 1) are unchanged, every entry is at most 1 and the fp32 factor
// cannot overflow; F is the unshifted factor times exp(-M / 2).
//
// Design (B200): each (batch, kv-head) unit owns C thread blocks; block c owns
// a contiguous slice of rows (keys).  The residual diagonal of the slice stays
// in shared memory in fp64 for the whole run.  A step is
//   1. every block reads the C slice sums of the residual diagonal (fp64,
//      written at the end of the previous step), draws t = u_j * sum with
//      Philox4x32-10 and finds the block whose slice holds the crossing;
//   2. that block scans its slice (inverse CDF, strict ">") and publishes the
//      pivot s_j and its residual through the unit's sync slot;
//   3. every block streams, for its rows i, the transposed keys Kt[:, i] and
//      the factor columns F[0..j), i (both laid out with i contiguous, so a
//      warp reads 256 contiguous bytes of each F column) and computes
//        F[j, i] = (exp(beta <k_i, k_s> - M) - sum_c F[c, i] F[c, s]) / sqrt(d_s)
//      with fp32 products summed in chunks of eight into fp64, then downdates
//      its residual diagonal and publishes its new slice sum;
//   4. a bounded barrier among the unit's blocks closes the step.
// Blocks of one unit wait on each other, so a wave with C > 1 is launched
// cooperatively (all blocks co-resident); every wait gives up after the
// shape's timeout and records WC_ERR_TIMEOUT.
//
// Three forms of the same steps serve shorter units (launch_select_t picks,
// in this order):
//   * resident: few units, each one's keys and factor within the shared
//     memory of a cluster of up to 8 blocks, all units on the GPU at once;
//     nothing streams, the blocks meet at the cluster barrier;
//   * cluster: units of 2 to 8 blocks; the blocks of a unit form a cluster
//     and hand the step over through distributed shared memory instead of
//     global-memory flags and barriers; keys and factor stream as above;
//   * unit: many units (at least one per SM) of at most 1024 keys; one block
//     per unit keeps the unit's keys in shared memory and streams the factor.
// All forms do every row's arithmetic in the same order as the streaming
// kernel, so the factor agrees with it wherever the slice boundaries do.
#include <cooperative_groups.h>
#include <type_traits>

#include "wc_common.cuh"
#include "wc_exp2.cuh"
#include "wc_internal.h"

namespace wc {
namespace {

// threads per block: 256 (2 blocks per SM), or 128 (4 per SM) where the units
// are too many for 2 blocks per SM to give each enough of them (binned
// selections); shared memory is planned for the larger
constexpr int kThreads = 256;
// rows per thread per pass (one float2 of F): with about 14 rows of a block's
// slice per thread, 2-row groups keep the threads of a block evenly loaded
// (8-row groups left a seventh of a step idle), and the streams go as 8-byte
// loads, 32 of them in flight per thread
constexpr int kGroup = 2;
// Rows per block are a multiple of 128, so every block's slice of F (fp32) and
// of the transposed keys (bf16) starts on a 256-byte boundary: blocks whose
// slices did not streamed their share about 6 % slower, and every step waits
// for the slowest block of the unit.
constexpr int kRowAlign = 128;

struct SelectArgs {
    const void* K;
    int32_t* piv;
    float* F;
    int32_t* rank;
    void* Kt;
    UnitSync* sync;
    double* partials;
    int* status;
    int64_t ldf;
    int32_t n, d, r;
    int32_t C;      // blocks per unit
    int32_t m;      // rows per block (multiple of kRowAlign)
    int32_t unit0;  // first unit of this wave
    double beta, eps;
    uint64_t seed;
    uint64_t timeout_ns;
    int32_t bins;      // key bins per caller unit: unit u is bin u % bins of its unit
    int32_t bin_keys;  // keys per bin (pivot indices are reported within the caller's unit)
    const double* kbar;  // centring: mean key of each caller unit ([units / bins][d]), else null
    uint32_t unit_base;  // Philox unit index of unit 0 (a larger problem's units split across calls)
};

// Shared-memory plan (bytes) for m rows, r pivots, d dims.
__host__ __device__ inline size_t select_smem_bytes(int m, int r, int d) {
    return (size_t)m * 8          // residual diagonal (fp64)
           + (size_t)kThreads * 8 // per-thread inclusive scan
           + (size_t)kMaxBlocksPerUnit * 8  // the unit's block sums of a step
           + (size_t)d * 8        // pivot key
           + (size_t)d * 8        // pivot key as fp32 pairs
           + (size_t)r * 8        // F[s, 0..j) as pairs
           + (size_t)m            // pivot flags
           + 64;                  // broadcast scalars
}

struct Bcast {
    double base, tau, d_s;
    int owner, stop, s, ok, tstar, pad;
};

// Inclusive scan over the block of one double per thread (fixed order,
// deterministic); writes each thread's inclusive value to scan[tid] and
// returns the block total.
template <int NT>
__device__ double block_scan(double v, double* scan) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    __shared__ double wtot[NT / 32];
    if (lane == 31) wtot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        double w = lane < NT / 32 ? wtot[lane] : 0.0;
#pragma unroll
        for (int o = 1; o < NT / 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NT / 32) wtot[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += wtot[warp - 1];
    scan[threadIdx.x] = v;
    const double total = wtot[NT / 32 - 1];
    __syncthreads();
    return total;
}

// Contiguous chunk of the slice that thread `t` sums for the scans.
template <int NT>
__device__ __forceinline__ void chunk_of(int t, int mlen, int* lo, int* hi) {
    const int q = (mlen + NT - 1) / NT;
    *lo = min(mlen, t * q);
    *hi = min(mlen, *lo + q);
}

__device__ __forceinline__ float2 ld_stream_f2(const float* p) {
    float2 v;
    asm volatile("ld.global.L1::no_allocate.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// The two-row sums below run the two rows' fp32 products as packed pairs
// (fma.rn.f32x2: per lane the rounding of fmaf), against the pivot's values
// held twice over in shared memory ({v, v} pairs, read four floats at a time).

// <k_i, k_s> for the 2 rows at Kt + i0 (column stride ldf): products of 8
// consecutive dimensions summed in fp32, the chunks summed in fp64.  ks2: the
// pivot key as fp32 pairs (exact: it holds bf16 values); ks: in fp64.
template <typename T>
__device__ __forceinline__ void key_dots(const T* Kt, int64_t ldf, int d, const float2* ks2, const double* ks,
                                         double dot[2]);

__device__ __forceinline__ float2 bf16_pair(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <>
__device__ __forceinline__ void key_dots<__nv_bfloat16>(const __nv_bfloat16* Kt, int64_t ldf, int d,
                                                       const float2* ks2, const double*, double dot[2]) {
    dot[0] = dot[1] = 0.0;
#pragma unroll 4
    for (int c0 = 0; c0 < d; c0 += 8) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float4 kk = *reinterpret_cast<const float4*>(ks2 + c0 + c);
            const uint32_t w0 = ld_stream_u32(Kt + (int64_t)(c0 + c) * ldf);
            const uint32_t w1 = ld_stream_u32(Kt + (int64_t)(c0 + c + 1) * ldf);
            acc = fma2(bf16_pair(w0), make_float2(kk.x, kk.y), acc);
            acc = fma2(bf16_pair(w1), make_float2(kk.z, kk.w), acc);
        }
        dot[0] += (double)acc.x;
        dot[1] += (double)acc.y;
    }
}

template <>
__device__ __forceinline__ void key_dots<float>(const float* Kt, int64_t ldf, int d, const float2*,
                                               const double* ks, double dot[2]) {
    // fp32 (or centred) keys: products and sums in fp64
    dot[0] = dot[1] = 0.0;
#pragma unroll 8
    for (int c = 0; c < d; ++c) {
        const float2 v = ld_stream_f2(Kt + (int64_t)c * ldf);
        const double kc = ks[c];
        dot[0] += (double)v.x * kc;
        dot[1] += (double)v.y * kc;
    }
}

// The same two-row dots with the keys in shared memory (column stride m).
__device__ __forceinline__ void key_dots_shared(const __nv_bfloat16* Kt, int m, int d, const float2* ks2,
                                                const double*, double dot[2]) {
    dot[0] = dot[1] = 0.0;
#pragma unroll 4
    for (int c0 = 0; c0 < d; c0 += 8) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float4 kk = *reinterpret_cast<const float4*>(ks2 + c0 + c);
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(Kt + (size_t)(c0 + c) * m);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(Kt + (size_t)(c0 + c + 1) * m);
            acc = fma2(bf16_pair(w0), make_float2(kk.x, kk.y), acc);
            acc = fma2(bf16_pair(w1), make_float2(kk.z, kk.w), acc);
        }
        dot[0] += (double)acc.x;
        dot[1] += (double)acc.y;
    }
}

__device__ __forceinline__ void key_dots_shared(const float* Kt, int m, int d, const float2*, const double* ks,
                                                double dot[2]) {
    dot[0] = dot[1] = 0.0;
#pragma unroll 8
    for (int c = 0; c < d; ++c) {
        const float2 v = *reinterpret_cast<const float2*>(Kt + (size_t)c * m);
        const double kc = ks[c];
        dot[0] += (double)v.x * kc;
        dot[1] += (double)v.y * kc;
    }
}

// sum_{c<j} F[c, i] F[c, s] for the 2 rows at Fi (column stride ldf): products
// of 8 consecutive columns summed in fp32, the chunks summed in fp64.  32
// columns are loaded before any is used.  fs2: F[s, c] as pairs.
__device__ __forceinline__ void correction(const float* Fi, int64_t ldf, int j, const float2* fs2, double cor[2]) {
    cor[0] = cor[1] = 0.0;
    int c0 = 0;
    for (; c0 + 32 <= j; c0 += 32) {
        float2 v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = ld_stream_f2(Fi + (int64_t)(c0 + c) * ldf);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float4 ff = *reinterpret_cast<const float4*>(fs2 + c0 + 8 * q + c);
                acc = fma2(v[8 * q + c], make_float2(ff.x, ff.y), acc);
                acc = fma2(v[8 * q + c + 1], make_float2(ff.z, ff.w), acc);
            }
            cor[0] += (double)acc.x;
            cor[1] += (double)acc.y;
        }
    }
    for (; c0 + 8 <= j; c0 += 8) {
        float2 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = ld_stream_f2(Fi + (int64_t)(c0 + c) * ldf);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float4 ff = *reinterpret_cast<const float4*>(fs2 + c0 + c);
            acc = fma2(v[c], make_float2(ff.x, ff.y), acc);
            acc = fma2(v[c + 1], make_float2(ff.z, ff.w), acc);
        }
        cor[0] += (double)acc.x;
        cor[1] += (double)acc.y;
    }
    if (c0 < j) {
        float2 acc = make_float2(0.f, 0.f);
        for (int c = c0; c < j; ++c) acc = fma2(ld_stream_f2(Fi + (int64_t)c * ldf), fs2[c], acc);
        cor[0] += (double)acc.x;
        cor[1] += (double)acc.y;
    }
}

// One row's <k_i, k_s> and correction, from shared memory (the resident
// variant with a row per thread): the same sums, in the same order, as the
// two-row forms above.
__device__ __forceinline__ double key_dot1(const __nv_bfloat16* Kt, int m, int d, const float* ksf) {
    double dot = 0.0;
#pragma unroll 4
    for (int c0 = 0; c0 < d; c0 += 8) {
        const float4 k0 = *reinterpret_cast<const float4*>(ksf + c0);
        const float4 k1 = *reinterpret_cast<const float4*>(ksf + c0 + 4);
        const float kc[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        float a0 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t w = (uint32_t)*reinterpret_cast<const unsigned short*>(Kt + (size_t)(c0 + c) * m) << 16;
            a0 = fmaf(__uint_as_float(w), kc[c], a0);
        }
        dot += (double)a0;
    }
    return dot;
}

__device__ __forceinline__ double key_dot1(const float* Kt, int m, int d, const double* ks) {
    double dot = 0.0;
#pragma unroll 8
    for (int c = 0; c < d; ++c) dot += (double)Kt[(size_t)c * m] * ks[c];
    return dot;
}

__device__ __forceinline__ double correction1(const float* Fi, int m, int j, const float* fs) {
    double cor = 0.0;
    int c0 = 0;
    for (; c0 + 32 <= j; c0 += 32) {
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = Fi[(size_t)(c0 + c) * m];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f0 = *reinterpret_cast<const float4*>(fs + c0 + 8 * q);
            const float4 f1 = *reinterpret_cast<const float4*>(fs + c0 + 8 * q + 4);
            const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            float a0 = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) a0 = fmaf(v[8 * q + c], f[c], a0);
            cor += (double)a0;
        }
    }
    for (; c0 + 8 <= j; c0 += 8) {
        float a0 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) a0 = fmaf(Fi[(size_t)(c0 + c) * m], fs[c0 + c], a0);
        cor += (double)a0;
    }
    if (c0 < j) {
        float a0 = 0.f;
        for (int c = c0; c < j; ++c) a0 = fmaf(Fi[(size_t)c * m], fs[c], a0);
        cor += (double)a0;
    }
    return cor;
}

// T: element type of K; TK: of the transposed copy that every step streams
// (T, or fp32 when the keys are centred).
template <typename T, typename TK, int NT>
__global__ void __launch_bounds__(NT, 512 / NT) rpcholesky_kernel(const SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x;
    const int unit = a.unit0 + blockIdx.x / a.C;
    const int blk = blockIdx.x % a.C;
    const int n = a.n, d = a.d, r = a.r;
    const int64_t ldf = a.ldf;
    const int r0 = min(n, blk * a.m);
    const int r1 = min(n, r0 + a.m);
    const int mlen = r1 - r0;
    // groups this block computes: its rows, and for the last block the padding
    // up to the row stride ldf as well (F is zero there)
    const int ng = r1 == n ? (int)((ldf - r0 + kGroup - 1) / kGroup) : (mlen + kGroup - 1) / kGroup;

    double* dg = reinterpret_cast<double*>(smem);
    double* scan = dg + a.m;
    double* bsum = scan + kThreads;  // the scan array is planned for the larger block
    double* ks = bsum + kMaxBlocksPerUnit;
    float2* ks2 = reinterpret_cast<float2*>(ks + d);
    float2* fs2 = ks2 + d;
    unsigned char* ispiv = reinterpret_cast<unsigned char*>(fs2 + r);
    __shared__ Bcast bc;

    const T* K = static_cast<const T*>(a.K) + (size_t)unit * n * d;
    TK* Kt = static_cast<TK*>(a.Kt) + (size_t)unit * d * ldf;
    const double* kb = a.kbar ? a.kbar + (size_t)(unit / a.bins) * d : nullptr;
    float* F = a.F + (size_t)unit * r * ldf;
    UnitSync* us = a.sync + unit;
    double* part = a.partials + (size_t)unit * 2 * kMaxBlocksPerUnit;
    int* status = a.status;

    // ---- initial residual in the log domain, beta |k_i|^2 (centred: k_i - kbar, in
    // fp64, the transposed copy stored as fp32); transpose the slice
    double lmax = 0.0;
    for (int il = tid; il < ng * kGroup; il += NT) {
        const int i = r0 + il;
        if (il < mlen) {
            const T* krow = K + (size_t)i * d;
            double ss = 0.0;
            for (int c = 0; c < d; ++c) {
                const T v = krow[c];
                double x = (double)to_f32(v);
                if (kb) x -= kb[c];
                ss += x * x;
                if constexpr (std::is_same<T, TK>::value) Kt[(int64_t)c * ldf + i] = kb ? TK((float)x) : v;
                else Kt[(int64_t)c * ldf + i] = (TK)(float)x;
            }
            dg[il] = a.beta * ss;
            lmax = fmax(lmax, dg[il]);
        } else {
            for (int c = 0; c < d; ++c) Kt[(int64_t)c * ldf + i] = TK(0.f);
            if (il < a.m) dg[il] = 0.0;
        }
        if (il < a.m) ispiv[il] = 0;
    }
    // block max of beta |k_i|^2 -> unit max M (non-negative doubles order like their bits)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if ((tid & 31) == 0 && lmax > 0.0) atomicMax(&us->hmax_bits, (unsigned long long)__double_as_longlong(lmax));
    // the unit's blocks meet; a unit of one block only needs its own threads
    auto unit_sync = [&](uint32_t epoch) -> bool {
        if (a.C == 1) {
            __syncthreads();
            return true;
        }
        return unit_barrier(&us->bar, a.C, epoch, a.timeout_ns, status, &bc.ok);
    };
    bool alive = unit_sync(1);
    // The factor is taken of the shifted kernel H' = exp(beta K K^T - M): every
    // entry is at most 1 (Cauchy-Schwarz), the diagonal's maximum is 1, and the
    // pivots, the stop rule (relative to the diagonal's maximum) and the weights
    // do not change; F is H's factor times exp(-M / 2).
    double shift = 0.0;
    if (alive) {
        shift = __longlong_as_double((long long)__ldcg(&us->hmax_bits));
        if (!isfinite(shift)) {
            if (tid == 0) record_status(status, WC_ERR_NUMERIC);
            alive = false;
        }
    }
    for (int il = tid; il < mlen; il += NT) dg[il] = exp(dg[il] - shift);
    __syncthreads();  // the scan chunks below span rows that other threads initialised
    {
        int lo, hi;
        chunk_of<NT>(tid, mlen, &lo, &hi);
        double sum = 0.0;
        for (int il = lo; il < hi; ++il) sum += dg[il];
        const double tot = block_scan<NT>(sum, scan);
        if (tid == 0) part[blk] = tot;
    }
    if (alive) alive = unit_sync(2);
    const double hmax = 1.0;  // the shifted diagonal's maximum

    int final_rank = alive ? r : 0;
    for (int j = 0; alive && j < r; ++j) {
        const double* pj = part + (size_t)(j & 1) * kMaxBlocksPerUnit;
        // 1. which block's slice holds t = u_j * sum(d): the unit's block sums
        // come into shared memory in parallel, then one thread adds them in
        // block order
        for (int c = tid; c < a.C; c += NT) bsum[c] = __ldcg(pj + c);
        __syncthreads();
        if (tid == 0) {
            double total = 0.0;
            for (int c = 0; c < a.C; ++c) total += bsum[c];
            bc.stop = 0;
            bc.owner = -1;
            if (!(total > 0.0)) {
                if (isnan(total)) record_status(status, WC_ERR_NUMERIC);
                bc.stop = 1;
            } else {
                const double tau = pivot_uniform(a.seed, (uint32_t)j, a.unit_base + (uint32_t)unit) * total;
                double run = 0.0;
                for (int c = 0; c < a.C; ++c) {
                    const double nxt = run + bsum[c];
                    if (nxt > tau) { bc.owner = c; bc.base = run; break; }
                    run = nxt;
                }
                if (bc.owner < 0) {  // rounding left tau at the top: last block with mass
                    run = 0.0;
                    for (int c = 0; c < a.C; ++c) {
                        const double p = bsum[c];
                        if (p > 0.0) { bc.owner = c; bc.base = run; }
                        run += p;
                    }
                }
                bc.tau = tau;
            }
            bc.tstar = NT;
        }
        __syncthreads();
        if (bc.stop) { final_rank = j; break; }

        // 2. the owner block finds the pivot in its slice and publishes it
        if (blk == bc.owner) {
            const double base = bc.base, tau = bc.tau;
            if (base + scan[tid] > tau) atomicMin(&bc.tstar, tid);
            __syncthreads();
            if (tid == 0 && bc.tstar == NT) bc.tstar = NT - 1;  // rounding guard
            __syncthreads();
            if (tid == bc.tstar) {
                int lo, hi;
                chunk_of<NT>(tid, mlen, &lo, &hi);
                double run = tid == 0 ? base : base + scan[tid - 1];
                int sl = -1;
                for (int il = lo; il < hi; ++il) {
                    run += dg[il];
                    if (run > tau) { sl = il; break; }
                }
                if (sl < 0) {  // rounding: last positive entry of the chunk, else of the slice
                    for (int il = hi - 1; il >= lo && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                    for (int il = mlen - 1; il >= 0 && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                }
                const double ds = sl >= 0 ? dg[sl] : 0.0;
                const int stop = !(ds > a.eps * hmax);
                us->s = r0 + sl;
                us->d_s = ds;
                us->stop = stop;
                if (!stop) a.piv[(size_t)unit * r + j] = r0 + sl + (unit % a.bins) * a.bin_keys;
                if (a.C > 1) {  // the unit's other blocks wait for it
                    __threadfence();
                    st_release_u32(&us->pivflag, (uint32_t)j + 1u);
                }
                bc.s = r0 + sl;
                bc.d_s = ds;
                bc.stop = stop;
            }
            __syncthreads();
        } else {
            if (tid == 0) {
                if (wait_geq(&us->pivflag, (uint32_t)j + 1u, a.timeout_ns, status)) {
                    bc.s = *(volatile int32_t*)&us->s;
                    bc.d_s = *(volatile double*)&us->d_s;
                    bc.stop = *(volatile int32_t*)&us->stop;
                    bc.ok = 1;
                } else {
                    bc.ok = 0;
                }
            }
            __syncthreads();
            if (!bc.ok) { final_rank = j; alive = false; break; }
        }
        if (bc.stop) { final_rank = j; break; }
        const int s = bc.s;
        const double ds = bc.d_s;
        if (!in_bounds(s >= 0 && s < n, status)) {  // every block reads the same s: all stop here
            final_rank = j;
            break;
        }

        // 3. pivot key and F[s, 0..j) into shared memory
        for (int c = tid; c < d; c += NT) {
            const double kv = (double)to_f32(K[(size_t)s * d + c]) - (kb ? kb[c] : 0.0);
            ks[c] = kv;
            ks2[c] = make_float2((float)kv, (float)kv);
        }
        for (int c0 = tid; c0 < j; c0 += 8 * NT) {  // 8 loads in flight before the stores
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int c = c0 + q * NT;
                v[q] = c < j ? ld_cg_f32(F + (int64_t)c * ldf + s) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (c0 + q * NT < j) fs2[c0 + q * NT] = make_float2(v[q], v[q]);
        }
        __syncthreads();

        // 4. column j over this block's rows, and the residual downdate
        const double root = sqrt(ds);
        float* Fj = F + (int64_t)j * ldf;
        for (int g = tid; g < ng; g += NT) {
            const int il0 = g * kGroup;
            const int i0 = r0 + il0;
            if (!in_bounds(i0 + kGroup <= ldf, status)) continue;
            double dot[kGroup], cor[kGroup];
            key_dots<TK>(Kt + i0, ldf, d, ks2, ks, dot);
            correction(F + i0, ldf, j, fs2, cor);
            float out[kGroup];
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                const int il = il0 + k;
                double f = 0.0;
                if (il < mlen && !ispiv[il]) f = (exp(a.beta * dot[k] - shift) - cor[k]) / root;
                out[k] = (float)f;
                if (il < mlen) {
                    const double nd = dg[il] - f * f;
                    dg[il] = nd > 0.0 ? nd : 0.0;
                }
            }
            *reinterpret_cast<float2*>(Fj + i0) = make_float2(out[0], out[1]);
        }
        __syncthreads();
        if (s >= r0 && s < r1 && tid == 0) {
            dg[s - r0] = 0.0;
            ispiv[s - r0] = 1;
        }
        __syncthreads();

        // 5. new slice sum, then close the step
        {
            int lo, hi;
            chunk_of<NT>(tid, mlen, &lo, &hi);
            double sum = 0.0;
            for (int il = lo; il < hi; ++il) sum += dg[il];
            const double tot = block_scan<NT>(sum, scan);
            if (tid == 0) part[(size_t)((j + 1) & 1) * kMaxBlocksPerUnit + blk] = tot;
        }
        if (!unit_sync((uint32_t)j + 3u)) {
            final_rank = j + 1;
            alive = false;
            break;
        }
    }

    // ---- columns >= rank are zero; piv beyond rank is -1
    for (int jj = final_rank; jj < r; ++jj) {
        float* Fj = F + (int64_t)jj * ldf;
        for (int g = tid; g < ng; g += NT) {
            const int i0 = r0 + g * kGroup;
            *reinterpret_cast<float2*>(Fj + i0) = make_float2(0.f, 0.f);
        }
    }
    if (blk == 0) {
        for (int jj = final_rank + tid; jj < r; jj += NT) a.piv[(size_t)unit * r + jj] = -1;
        if (tid == 0) a.rank[unit] = final_rank;
    }
}

// ---- resident variant: a unit's keys and factor held in shared memory ----
//
// When a unit's transposed keys and factor columns fit in the shared memory of
// a cluster of at most kMaxCluster blocks (short heads: n r fp32 plus n d key
// elements) and all units fit on the GPU at once (few units: the factor in
// shared memory allows far fewer units at a time than streaming it), each block
// keeps its slice of Kt and of F for the whole run: a step reads no global
// memory but the pivot's key when centred, writes none (F and the pivots go
// out after the last step), and the unit's blocks meet at the cluster barrier,
// the slice sums, the pivot, its key and its factor row travelling through
// distributed shared memory.  Every row's arithmetic is that of
// rpcholesky_kernel (same dot and correction order, same scans and draw), so
// results agree with it wherever the slice boundaries do.
constexpr int kMaxCluster = 8;
// threads per resident block, a row each per pass (measured against 256
// threads with two rows each: about 5 % faster on one 512-key unit)
constexpr int kResThreads = 512;

struct PivMsg {
    double d_s;
    int s, stop;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) / 16 * 16; }

// Shared-memory plan of a resident block: m rows, r pivots, d dims, key copy
// elements of tk bytes.  Offsets in the order the kernel carves them.
struct ResidentSmem {
    size_t dg, scan, bsum, bmax, uj, ks, ksf, fs, msg, pv, f, kt, ispiv, total;
    __host__ __device__ ResidentSmem(int m, int r, int d, int tk, int nt) {
        size_t o = 0;
        dg = o;    o = align16(o + (size_t)m * 8);
        scan = o;  o = align16(o + (size_t)nt * 8);
        bsum = o;  o = align16(o + (size_t)kMaxCluster * 8);
        bmax = o;  o = align16(o + (size_t)kMaxCluster * 8);
        uj = o;    o = align16(o + (size_t)r * 8);
        ks = o;    o = align16(o + (size_t)d * 8);
        ksf = o;   o = align16(o + (size_t)d * 4);
        fs = o;    o = align16(o + (size_t)r * 4);
        msg = o;   o = align16(o + sizeof(PivMsg));
        pv = o;    o = align16(o + (size_t)r * 4);
        f = o;     o = align16(o + (size_t)r * m * 4);
        kt = o;    o = align16(o + (size_t)d * m * tk);
        ispiv = o; o = align16(o + (size_t)m);
        total = o;
    }
};

namespace cg = cooperative_groups;

template <typename T, typename TK, int NT>
__global__ void __launch_bounds__(NT, 1) rpcholesky_resident_kernel(const SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int blk = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31;
    const int unit = blockIdx.x / CL;
    const int n = a.n, d = a.d, r = a.r, m = a.m;
    const int64_t ldf = a.ldf;
    const int r0 = min(n, blk * m);
    const int r1 = min(n, r0 + m);
    const int mlen = r1 - r0;
    // rows this block writes to F: its slice, and for the last block the
    // padding up to ldf (F is zero there); m is a multiple of 64 and at least
    // ldf - r0 for the last block
    const int64_t tail = ldf - r0;
    const int rows = tail < m ? (tail > 0 ? (int)tail : 0) : m;

    const ResidentSmem L(m, r, d, (int)sizeof(TK), NT);
    double* dg = reinterpret_cast<double*>(smem + L.dg);
    double* scan = reinterpret_cast<double*>(smem + L.scan);
    double* bsum = reinterpret_cast<double*>(smem + L.bsum);
    double* bmax = reinterpret_cast<double*>(smem + L.bmax);
    double* uj = reinterpret_cast<double*>(smem + L.uj);
    double* ks = reinterpret_cast<double*>(smem + L.ks);
    float* ksf = reinterpret_cast<float*>(smem + L.ksf);
    float* fs = reinterpret_cast<float*>(smem + L.fs);
    PivMsg* msg = reinterpret_cast<PivMsg*>(smem + L.msg);
    int* pv = reinterpret_cast<int*>(smem + L.pv);     // the pivots, written out at the end
    float* Fs = reinterpret_cast<float*>(smem + L.f);   // [r][m]
    TK* Kts = reinterpret_cast<TK*>(smem + L.kt);      // [d][m]
    unsigned char* ispiv = smem + L.ispiv;
    __shared__ unsigned long long lmax_bits;

    const T* K = static_cast<const T*>(a.K) + (size_t)unit * n * d;
    const double* kb = a.kbar ? a.kbar + (size_t)(unit / a.bins) * d : nullptr;
    float* F = a.F + (size_t)unit * r * ldf;
    int* status = a.status;

    // ---- the unit's pivot draws (they depend on nothing the steps compute);
    // the slice's keys, transposed into shared memory; beta |k_i|^2
    for (int jj = tid; jj < r; jj += NT) uj[jj] = pivot_uniform(a.seed, (uint32_t)jj, a.unit_base + (uint32_t)unit);
    if (tid == 0) lmax_bits = 0ull;
    __syncthreads();
    double lmax = 0.0;
    for (int il = tid; il < m; il += NT) {
        double v = 0.0;
        if (il < mlen) {
            const T* krow = K + (size_t)(r0 + il) * d;
            double ss = 0.0;
            for (int c = 0; c < d; ++c) {
                const T kv = krow[c];
                double x = (double)to_f32(kv);
                if (kb) x -= kb[c];
                ss += x * x;
                if constexpr (std::is_same<T, TK>::value) Kts[(size_t)c * m + il] = kb ? TK((float)x) : kv;
                else Kts[(size_t)c * m + il] = (TK)(float)x;
            }
            v = a.beta * ss;
        } else {
            for (int c = 0; c < d; ++c) Kts[(size_t)c * m + il] = TK(0.f);
        }
        dg[il] = v;
        ispiv[il] = 0;
        lmax = fmax(lmax, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if (lane == 0 && lmax > 0.0) atomicMax(&lmax_bits, (unsigned long long)__double_as_longlong(lmax));
    __syncthreads();
    if (tid < CL) cluster.map_shared_rank(bmax, tid)[blk] = __longlong_as_double((long long)lmax_bits);
    cluster.sync();
    double shift = 0.0;
    for (int c = 0; c < CL; ++c) shift = fmax(shift, bmax[c]);
    bool alive = isfinite(shift);
    if (!alive && blk == 0 && tid == 0) record_status(status, WC_ERR_NUMERIC);
    const double hmax = 1.0;  // the shifted diagonal's maximum

    if (alive) {
        for (int il = tid; il < mlen; il += NT) dg[il] = exp(dg[il] - shift);
        __syncthreads();
        int lo, hi;
        chunk_of<NT>(tid, mlen, &lo, &hi);
        double sum = 0.0;
        for (int il = lo; il < hi; ++il) sum += dg[il];
        const double tot = block_scan<NT>(sum, scan);
        if (tid < CL) cluster.map_shared_rank(bsum, tid)[blk] = tot;
        cluster.sync();
    }

    int final_rank = alive ? r : 0;
    for (int j = 0; alive && j < r; ++j) {
        // 1. the block whose slice holds t = u_j * sum(d), from the slice sums:
        // every thread of every block of the unit takes the same decision
        double total = 0.0;
        for (int c = 0; c < CL; ++c) total += bsum[c];
        if (!(total > 0.0)) {
            if (isnan(total) && blk == 0 && tid == 0) record_status(status, WC_ERR_NUMERIC);
            final_rank = j;
            break;
        }
        const double tau = uj[j] * total;
        int owner = -1;
        double base = 0.0;
        {
            double run = 0.0;
            for (int c = 0; c < CL; ++c) {
                const double nxt = run + bsum[c];
                if (nxt > tau) { owner = c; base = run; break; }
                run = nxt;
            }
            if (owner < 0) {  // rounding left tau at the top: last block with mass
                run = 0.0;
                for (int c = 0; c < CL; ++c) {
                    const double p = bsum[c];
                    if (p > 0.0) { owner = c; base = run; }
                    run += p;
                }
            }
        }

        // 2. in the owner, the first thread whose inclusive slice prefix passes
        // tau (prefixes of non-negative terms do not decrease), else the last
        // thread, scans its chunk; its warp sends the pivot, its key and its
        // factor row to every block of the unit
        if (blk == owner) {
            const bool past = base + scan[tid] > tau;
            const bool prev = tid > 0 && base + scan[tid - 1] > tau;
            const bool mine = (past && !prev) || (tid == NT - 1 && !past);
            const unsigned bal = __ballot_sync(0xffffffffu, mine);
            if (bal) {
                int sl = -1, stop = 1;
                double ds = 0.0;
                if (mine) {
                    int lo, hi;
                    chunk_of<NT>(tid, mlen, &lo, &hi);
                    double run = tid == 0 ? base : base + scan[tid - 1];
                    for (int il = lo; il < hi; ++il) {
                        run += dg[il];
                        if (run > tau) { sl = il; break; }
                    }
                    if (sl < 0) {  // rounding: last positive entry of the chunk, else of the slice
                        for (int il = hi - 1; il >= lo && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                        for (int il = mlen - 1; il >= 0 && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                    }
                    ds = sl >= 0 ? dg[sl] : 0.0;
                    stop = !(ds > a.eps * hmax);
                }
                const int src = __ffs(bal) - 1;
                sl = __shfl_sync(0xffffffffu, sl, src);
                stop = __shfl_sync(0xffffffffu, stop, src);
                ds = __shfl_sync(0xffffffffu, ds, src);
                for (int p = 0; p < CL; ++p) {
                    if (sl >= 0) {
                        double* ksp = cluster.map_shared_rank(ks, p);
                        float* ksfp = cluster.map_shared_rank(ksf, p);
                        float* fsp = cluster.map_shared_rank(fs, p);
                        for (int c = lane; c < d; c += 32) {
                            const double kv = kb ? (double)to_f32(K[(size_t)(r0 + sl) * d + c]) - kb[c]
                                                 : (double)to_f32(Kts[(size_t)c * m + sl]);
                            ksp[c] = kv;
                            ksfp[c] = (float)kv;
                        }
                        for (int c = lane; c < j; c += 32) fsp[c] = Fs[(size_t)c * m + sl];
                    }
                    if (lane == 0) {
                        PivMsg* mp = cluster.map_shared_rank(msg, p);
                        mp->s = r0 + sl;
                        mp->d_s = ds;
                        mp->stop = stop;
                    }
                }
            }
        }
        cluster.sync();
        if (msg->stop) { final_rank = j; break; }
        const int s = msg->s;
        const double ds = msg->d_s;
        if (!in_bounds(s >= 0 && s < n, status)) {  // every block reads the same s: all stop here
            final_rank = j;
            break;
        }
        if (tid == 0) pv[j] = s;

        // 3. column j over this block's rows, and the residual downdate (the
        // pivot's own row leaves the residual here); the factor goes out to
        // global memory after the last step, so that no step's barrier waits
        // for global stores
        const double root = sqrt(ds);
        const int spl = s - r0;
        float* Fsj = Fs + (size_t)j * m;
        for (int il = tid; il < rows; il += NT) {
            double dot;
            if constexpr (std::is_same<TK, float>::value) dot = key_dot1(Kts + il, m, d, ks);
            else dot = key_dot1(Kts + il, m, d, ksf);
            const double cor = correction1(Fs + il, m, j, fs);
            double f = 0.0;
            if (il < mlen && !ispiv[il]) f = (exp(a.beta * dot - shift) - cor) / root;
            Fsj[il] = (float)f;
            if (il < mlen) {
                const double nd = dg[il] - f * f;
                dg[il] = il == spl ? 0.0 : (nd > 0.0 ? nd : 0.0);
                if (il == spl) ispiv[il] = 1;
            }
        }
        __syncthreads();

        // 4. new slice sum to every block, then close the step
        {
            int lo, hi;
            chunk_of<NT>(tid, mlen, &lo, &hi);
            double sum = 0.0;
            for (int il = lo; il < hi; ++il) sum += dg[il];
            const double tot = block_scan<NT>(sum, scan);
            if (tid < CL) cluster.map_shared_rank(bsum, tid)[blk] = tot;
        }
        cluster.sync();
    }

    // ---- the factor's columns (zero from the rank on) and the pivots (-1 from
    // the rank on) out to global memory
    __syncthreads();
    for (int jj = 0; jj < r; ++jj) {
        float* Fj = F + (int64_t)jj * ldf + r0;
        const float* Fsj = Fs + (size_t)jj * m;
        for (int g = tid; g < rows / 2; g += NT)
            *reinterpret_cast<float2*>(Fj + 2 * g) =
                jj < final_rank ? *reinterpret_cast<const float2*>(Fsj + 2 * g) : make_float2(0.f, 0.f);
    }
    if (blk == 0) {
        const int off = (unit % a.bins) * a.bin_keys;
        for (int jj = tid; jj < r; jj += NT) a.piv[(size_t)unit * r + jj] = jj < final_rank ? pv[jj] + off : -1;
        if (tid == 0) a.rank[unit] = final_rank;
    }
    cluster.sync();  // no block leaves while a peer may still write to its shared memory
}

// ---- one block per unit: keys in shared memory, factor streamed ----
//
// Many short units (at least one per SM, at most 2 kUnitThreads keys each) take
// a block of kUnitThreads threads per unit, a pair of rows per thread.  The
// block keeps the unit's transposed keys in shared memory and streams only the
// factor columns (from L2: a wave's factors are a few tens of MB).  With one
// block per unit no step waits on another block: the slice sum is the block's
// own scan total, the pivot draws are taken before the first step, the pivot is
// found by the one thread whose inclusive prefix first passes tau, and the
// pivot's factor row is in flight while the key dots run.  Same per-row
// arithmetic as rpcholesky_kernel.
constexpr int kUnitThreads = 512;

struct UnitSmem {
    size_t dg, scan, uj, ks, ks2, fs2, ispiv, kt, total;
    __host__ __device__ UnitSmem(int m, int r, int d, int tk) {
        size_t o = 0;
        dg = o;    o = align16(o + (size_t)m * 8);
        scan = o;  o = align16(o + (size_t)kUnitThreads * 8);
        uj = o;    o = align16(o + (size_t)r * 8);
        ks = o;    o = align16(o + (size_t)d * 8);
        ks2 = o;   o = align16(o + (size_t)d * 8);
        fs2 = o;   o = align16(o + (size_t)r * 8);
        ispiv = o; o = align16(o + (size_t)m);
        kt = o;    o = align16(o + (size_t)d * m * tk);
        total = o;
    }
};

template <typename T, typename TK>
__global__ void __launch_bounds__(kUnitThreads, 1) rpcholesky_unit_kernel(const SelectArgs a) {
    constexpr int NT = kUnitThreads;
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x;
    const int unit = blockIdx.x;
    const int n = a.n, d = a.d, r = a.r, m = a.m;  // m = ldf <= 2 NT
    const int64_t ldf = a.ldf;
    const UnitSmem L(m, r, d, (int)sizeof(TK));
    double* dg = reinterpret_cast<double*>(smem + L.dg);
    double* scan = reinterpret_cast<double*>(smem + L.scan);
    double* uj = reinterpret_cast<double*>(smem + L.uj);
    double* ks = reinterpret_cast<double*>(smem + L.ks);
    float2* ks2 = reinterpret_cast<float2*>(smem + L.ks2);
    float2* fs2 = reinterpret_cast<float2*>(smem + L.fs2);
    unsigned char* ispiv = smem + L.ispiv;
    TK* Kts = reinterpret_cast<TK*>(smem + L.kt);  // [d][m]
    __shared__ double piv_ds;
    __shared__ int piv_s, piv_stop;
    __shared__ unsigned long long lmax_bits;

    const T* K = static_cast<const T*>(a.K) + (size_t)unit * n * d;
    const double* kb = a.kbar ? a.kbar + (size_t)(unit / a.bins) * d : nullptr;
    float* F = a.F + (size_t)unit * r * ldf;
    int* status = a.status;
    // this thread's rows: il0 and il0 + 1 (rows >= n up to ldf are padding, F zero there)
    const int il0 = 2 * tid;
    const bool has = il0 < ldf;
    const int lo = min(n, il0), hi = min(n, il0 + 2);

    // ---- the pivot draws; the keys, transposed into shared memory; beta |k_i|^2
    for (int jj = tid; jj < r; jj += NT) uj[jj] = pivot_uniform(a.seed, (uint32_t)jj, a.unit_base + (uint32_t)unit);
    if (tid == 0) lmax_bits = 0ull;
    __syncthreads();
    double lmax = 0.0;
    for (int il = il0; il < il0 + 2 && il < m; ++il) {
        double v = 0.0;
        if (il < n) {
            const T* krow = K + (size_t)il * d;
            double ss = 0.0;
            for (int c = 0; c < d; ++c) {
                const T kv = krow[c];
                double x = (double)to_f32(kv);
                if (kb) x -= kb[c];
                ss += x * x;
                if constexpr (std::is_same<T, TK>::value) Kts[(size_t)c * m + il] = kb ? TK((float)x) : kv;
                else Kts[(size_t)c * m + il] = (TK)(float)x;
            }
            v = a.beta * ss;
        } else {
            for (int c = 0; c < d; ++c) Kts[(size_t)c * m + il] = TK(0.f);
        }
        dg[il] = v;
        ispiv[il] = 0;
        lmax = fmax(lmax, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if ((tid & 31) == 0 && lmax > 0.0) atomicMax(&lmax_bits, (unsigned long long)__double_as_longlong(lmax));
    __syncthreads();
    const double shift = __longlong_as_double((long long)lmax_bits);
    bool alive = isfinite(shift);
    if (!alive && tid == 0) record_status(status, WC_ERR_NUMERIC);
    const double hmax = 1.0;  // the shifted diagonal's maximum

    double total = 0.0;
    if (alive) {
        double sum = 0.0;
        for (int il = lo; il < hi; ++il) {
            dg[il] = exp(dg[il] - shift);
            sum += dg[il];
        }
        total = block_scan<NT>(sum, scan);
    }

    int final_rank = alive ? r : 0;
    for (int j = 0; alive && j < r; ++j) {
        // 1. the pivot: the thread whose inclusive prefix first passes
        // t = u_j * total (else the last thread) scans its two rows
        if (!(total > 0.0)) {
            if (isnan(total) && tid == 0) record_status(status, WC_ERR_NUMERIC);
            final_rank = j;
            break;
        }
        const double tau = uj[j] * total;
        const bool past = scan[tid] > tau;
        const bool prev = tid > 0 && scan[tid - 1] > tau;
        if ((past && !prev) || (tid == NT - 1 && !past)) {
            double run = tid == 0 ? 0.0 : scan[tid - 1];
            int sl = -1;
            for (int il = lo; il < hi; ++il) {
                run += dg[il];
                if (run > tau) { sl = il; break; }
            }
            if (sl < 0) {  // rounding: last positive entry of the pair, else of the unit
                for (int il = hi - 1; il >= lo && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                for (int il = n - 1; il >= 0 && sl < 0; --il) if (dg[il] > 0.0) sl = il;
            }
            const double ds = sl >= 0 ? dg[sl] : 0.0;
            const int stop = !(ds > a.eps * hmax);
            if (!stop) a.piv[(size_t)unit * r + j] = sl + (unit % a.bins) * a.bin_keys;
            piv_s = sl;
            piv_ds = ds;
            piv_stop = stop;
        }
        __syncthreads();
        if (piv_stop) { final_rank = j; break; }
        const int s = piv_s;
        const double ds = piv_ds;
        if (!in_bounds(s >= 0 && s < n, status)) {  // every thread reads the same s: all stop here
            final_rank = j;
            break;
        }

        // 2. the pivot key into shared memory; its factor row's loads issued
        for (int c = tid; c < d; c += NT) {
            const double kv = kb ? (double)to_f32(K[(size_t)s * d + c]) - kb[c] : (double)to_f32(Kts[(size_t)c * m + s]);
            ks[c] = kv;
            ks2[c] = make_float2((float)kv, (float)kv);
        }
        const float fv0 = tid < j ? ld_cg_f32(F + (int64_t)tid * ldf + s) : 0.f;
        const float fv1 = tid + NT < j ? ld_cg_f32(F + (int64_t)(tid + NT) * ldf + s) : 0.f;
        __syncthreads();

        // 3. key dots while the factor row arrives, then the correction, the
        // column and the downdate (the pivot's own row leaves the residual)
        double dot[2] = {0.0, 0.0}, cor[2] = {0.0, 0.0};
        if (has) key_dots_shared(Kts + il0, m, d, ks2, ks, dot);
        if (tid < j) fs2[tid] = make_float2(fv0, fv0);
        if (tid + NT < j) fs2[tid + NT] = make_float2(fv1, fv1);
        __syncthreads();
        if (has) {
            correction(F + il0, ldf, j, fs2, cor);
            const double root = sqrt(ds);
            float out[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int il = il0 + k;
                double f = 0.0;
                if (il < n && !ispiv[il]) f = (exp(a.beta * dot[k] - shift) - cor[k]) / root;
                out[k] = (float)f;
                if (il < n) {
                    const double nd = dg[il] - f * f;
                    dg[il] = il == s ? 0.0 : (nd > 0.0 ? nd : 0.0);
                    if (il == s) ispiv[il] = 1;
                }
            }
            *reinterpret_cast<float2*>(F + (int64_t)j * ldf + il0) = make_float2(out[0], out[1]);
        }

        // 4. the new inclusive prefixes and total (each thread sums its own rows)
        double sum = 0.0;
        for (int il = lo; il < hi; ++il) sum += dg[il];
        total = block_scan<NT>(sum, scan);
    }

    // ---- columns >= rank are zero; piv beyond rank is -1
    if (has)
        for (int jj = final_rank; jj < r; ++jj)
            *reinterpret_cast<float2*>(F + (int64_t)jj * ldf + il0) = make_float2(0.f, 0.f);
    for (int jj = final_rank + tid; jj < r; jj += NT) a.piv[(size_t)unit * r + jj] = -1;
    if (tid == 0) a.rank[unit] = final_rank;
}

// ---- a cluster per unit, keys and factor streamed ----
//
// Units of 2 to kMaxCluster blocks (moderate key counts, tens of units) take the
// streaming kernel's steps with the hand-off through distributed shared memory:
// the blocks of a unit form a thread-block cluster; the slice sums go to every
// block, the owner block finds the pivot and sends it, the pivot key and the
// pivot's factor row (its own rows, so its own writes) to every block, and the
// blocks meet at the cluster barrier.  A step then waits on no global-memory
// flag or barrier, and each block reads and writes only its own rows of Kt and
// F.  The pivot draws are taken before the first step; the pivots go out after
// the last.  Same per-row arithmetic as rpcholesky_kernel.
struct ClusterSmem {
    size_t dg, scan, bsum, bmax, uj, ks, ks2, fs2, msg, pv, ispiv, total;
    __host__ __device__ ClusterSmem(int m, int r, int d) {
        size_t o = 0;
        dg = o;    o = align16(o + (size_t)m * 8);
        scan = o;  o = align16(o + (size_t)kThreads * 8);
        bsum = o;  o = align16(o + (size_t)kMaxCluster * 8);
        bmax = o;  o = align16(o + (size_t)kMaxCluster * 8);
        uj = o;    o = align16(o + (size_t)r * 8);
        ks = o;    o = align16(o + (size_t)d * 8);
        ks2 = o;   o = align16(o + (size_t)d * 8);
        fs2 = o;   o = align16(o + (size_t)r * 8);
        msg = o;   o = align16(o + sizeof(PivMsg));
        pv = o;    o = align16(o + (size_t)r * 4);
        ispiv = o; o = align16(o + (size_t)m);
        total = o;
    }
};

template <typename T, typename TK>
__global__ void __launch_bounds__(kThreads, 2) rpcholesky_cluster_kernel(const SelectArgs a) {
    constexpr int NT = kThreads;
    extern __shared__ __align__(16) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int blk = (int)cluster.block_rank();
    const int tid = threadIdx.x;
    const int unit = blockIdx.x / CL;
    const int n = a.n, d = a.d, r = a.r, m = a.m;
    const int64_t ldf = a.ldf;
    const int r0 = min(n, blk * m);
    const int r1 = min(n, r0 + m);
    const int mlen = r1 - r0;
    // groups this block computes: its rows, and for the last block the padding
    // up to the row stride ldf as well (F is zero there)
    const int ng = r1 == n ? (int)((ldf - r0 + kGroup - 1) / kGroup) : (mlen + kGroup - 1) / kGroup;

    const ClusterSmem L(m, r, d);
    double* dg = reinterpret_cast<double*>(smem + L.dg);
    double* scan = reinterpret_cast<double*>(smem + L.scan);
    double* bsum = reinterpret_cast<double*>(smem + L.bsum);
    double* bmax = reinterpret_cast<double*>(smem + L.bmax);
    double* uj = reinterpret_cast<double*>(smem + L.uj);
    double* ks = reinterpret_cast<double*>(smem + L.ks);
    float2* ks2 = reinterpret_cast<float2*>(smem + L.ks2);
    float2* fs2 = reinterpret_cast<float2*>(smem + L.fs2);
    PivMsg* msg = reinterpret_cast<PivMsg*>(smem + L.msg);
    int* pv = reinterpret_cast<int*>(smem + L.pv);
    unsigned char* ispiv = smem + L.ispiv;
    __shared__ int own_sl, own_stop;
    __shared__ double own_ds;
    __shared__ unsigned long long lmax_bits;

    const T* K = static_cast<const T*>(a.K) + (size_t)unit * n * d;
    TK* Kt = static_cast<TK*>(a.Kt) + (size_t)unit * d * ldf;
    const double* kb = a.kbar ? a.kbar + (size_t)(unit / a.bins) * d : nullptr;
    float* F = a.F + (size_t)unit * r * ldf;
    int* status = a.status;

    // ---- the pivot draws; the slice's keys transposed (this block's rows of
    // the unit's copy); beta |k_i|^2
    for (int jj = tid; jj < r; jj += NT) uj[jj] = pivot_uniform(a.seed, (uint32_t)jj, a.unit_base + (uint32_t)unit);
    if (tid == 0) lmax_bits = 0ull;
    __syncthreads();
    double lmax = 0.0;
    for (int il = tid; il < ng * kGroup; il += NT) {
        const int i = r0 + il;
        if (il < mlen) {
            const T* krow = K + (size_t)i * d;
            double ss = 0.0;
            for (int c = 0; c < d; ++c) {
                const T v = krow[c];
                double x = (double)to_f32(v);
                if (kb) x -= kb[c];
                ss += x * x;
                if constexpr (std::is_same<T, TK>::value) Kt[(int64_t)c * ldf + i] = kb ? TK((float)x) : v;
                else Kt[(int64_t)c * ldf + i] = (TK)(float)x;
            }
            dg[il] = a.beta * ss;
            lmax = fmax(lmax, dg[il]);
        } else {
            for (int c = 0; c < d; ++c) Kt[(int64_t)c * ldf + i] = TK(0.f);
            if (il < m) dg[il] = 0.0;
        }
        if (il < m) ispiv[il] = 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if ((tid & 31) == 0 && lmax > 0.0) atomicMax(&lmax_bits, (unsigned long long)__double_as_longlong(lmax));
    __syncthreads();
    if (tid < CL) cluster.map_shared_rank(bmax, tid)[blk] = __longlong_as_double((long long)lmax_bits);
    cluster.sync();
    double shift = 0.0;
    for (int c = 0; c < CL; ++c) shift = fmax(shift, bmax[c]);
    bool alive = isfinite(shift);
    if (!alive && blk == 0 && tid == 0) record_status(status, WC_ERR_NUMERIC);
    const double hmax = 1.0;  // the shifted diagonal's maximum

    if (alive) {
        for (int il = tid; il < mlen; il += NT) dg[il] = exp(dg[il] - shift);
        __syncthreads();
        int lo, hi;
        chunk_of<NT>(tid, mlen, &lo, &hi);
        double sum = 0.0;
        for (int il = lo; il < hi; ++il) sum += dg[il];
        const double tot = block_scan<NT>(sum, scan);
        if (tid < CL) cluster.map_shared_rank(bsum, tid)[blk] = tot;
        cluster.sync();
    }

    int final_rank = alive ? r : 0;
    for (int j = 0; alive && j < r; ++j) {
        // 1. the block whose slice holds t = u_j * sum(d), from the slice sums:
        // every thread of every block of the unit takes the same decision
        double total = 0.0;
        for (int c = 0; c < CL; ++c) total += bsum[c];
        if (!(total > 0.0)) {
            if (isnan(total) && blk == 0 && tid == 0) record_status(status, WC_ERR_NUMERIC);
            final_rank = j;
            break;
        }
        const double tau = uj[j] * total;
        int owner = -1;
        double base = 0.0;
        {
            double run = 0.0;
            for (int c = 0; c < CL; ++c) {
                const double nxt = run + bsum[c];
                if (nxt > tau) { owner = c; base = run; break; }
                run = nxt;
            }
            if (owner < 0) {  // rounding left tau at the top: last block with mass
                run = 0.0;
                for (int c = 0; c < CL; ++c) {
                    const double p = bsum[c];
                    if (p > 0.0) { owner = c; base = run; }
                    run += p;
                }
            }
        }

        // 2. the owner: the first thread whose inclusive prefix passes tau (else
        // the last) scans its chunk; then the block sends the pivot, its key
        // and its factor row (rows of this block: written by this block) to
        // every block of the unit
        if (blk == owner) {
            const bool past = base + scan[tid] > tau;
            const bool prev = tid > 0 && base + scan[tid - 1] > tau;
            if ((past && !prev) || (tid == NT - 1 && !past)) {
                int lo, hi;
                chunk_of<NT>(tid, mlen, &lo, &hi);
                double run = tid == 0 ? base : base + scan[tid - 1];
                int sl = -1;
                for (int il = lo; il < hi; ++il) {
                    run += dg[il];
                    if (run > tau) { sl = il; break; }
                }
                if (sl < 0) {  // rounding: last positive entry of the chunk, else of the slice
                    for (int il = hi - 1; il >= lo && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                    for (int il = mlen - 1; il >= 0 && sl < 0; --il) if (dg[il] > 0.0) sl = il;
                }
                own_sl = sl;
                own_ds = sl >= 0 ? dg[sl] : 0.0;
                own_stop = !(own_ds > a.eps * hmax);
            }
            __syncthreads();
            const int sl = own_sl;
            if (!own_stop) {
                const int sg = r0 + sl;
                for (int c = tid; c < d; c += NT) {
                    const double kv = (double)to_f32(K[(size_t)sg * d + c]) - (kb ? kb[c] : 0.0);
                    const float2 kv2 = make_float2((float)kv, (float)kv);
                    for (int p = 0; p < CL; ++p) {
                        cluster.map_shared_rank(ks, p)[c] = kv;
                        cluster.map_shared_rank(ks2, p)[c] = kv2;
                    }
                }
                for (int c = tid; c < j; c += NT) {
                    const float v = ld_cg_f32(F + (int64_t)c * ldf + sg);
                    for (int p = 0; p < CL; ++p) cluster.map_shared_rank(fs2, p)[c] = make_float2(v, v);
                }
            }
            if (tid < CL) {
                PivMsg* mp = cluster.map_shared_rank(msg, tid);
                mp->s = r0 + sl;
                mp->d_s = own_ds;
                mp->stop = own_stop;
            }
        }
        cluster.sync();
        if (msg->stop) { final_rank = j; break; }
        const int s = msg->s;
        const double ds = msg->d_s;
        if (!in_bounds(s >= 0 && s < n, status)) {  // every block reads the same s: all stop here
            final_rank = j;
            break;
        }
        if (tid == 0) pv[j] = s;

        // 3. column j over this block's rows, and the residual downdate (the
        // pivot's own row leaves the residual here)
        const double root = sqrt(ds);
        const int spl = s - r0;
        float* Fj = F + (int64_t)j * ldf;
        for (int g = tid; g < ng; g += NT) {
            const int il0 = g * kGroup;
            const int i0 = r0 + il0;
            if (!in_bounds(i0 + kGroup <= ldf, status)) continue;
            double dot[kGroup], cor[kGroup] = {0.0, 0.0};
            key_dots<TK>(Kt + i0, ldf, d, ks2, ks, dot);
            correction(F + i0, ldf, j, fs2, cor);
            float out[kGroup];
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                const int il = il0 + k;
                double f = 0.0;
                if (il < mlen && !ispiv[il]) f = (exp(a.beta * dot[k] - shift) - cor[k]) / root;
                out[k] = (float)f;
                if (il < mlen) {
                    const double nd = dg[il] - f * f;
                    dg[il] = il == spl ? 0.0 : (nd > 0.0 ? nd : 0.0);
                    if (il == spl) ispiv[il] = 1;
                }
            }
            *reinterpret_cast<float2*>(Fj + i0) = make_float2(out[0], out[1]);
        }
        __syncthreads();

        // 4. new slice sum to every block, then close the step
        {
            int lo, hi;
            chunk_of<NT>(tid, mlen, &lo, &hi);
            double sum = 0.0;
            for (int il = lo; il < hi; ++il) sum += dg[il];
            const double tot = block_scan<NT>(sum, scan);
            if (tid < CL) cluster.map_shared_rank(bsum, tid)[blk] = tot;
        }
        cluster.sync();
    }

    // ---- columns >= rank are zero; piv beyond rank is -1
    for (int jj = final_rank; jj < r; ++jj) {
        float* Fj = F + (int64_t)jj * ldf;
        for (int g = tid; g < ng; g += NT) *reinterpret_cast<float2*>(Fj + r0 + g * kGroup) = make_float2(0.f, 0.f);
    }
    if (blk == 0) {
        const int off = (unit % a.bins) * a.bin_keys;
        for (int jj = tid; jj < r; jj += NT) a.piv[(size_t)unit * r + jj] = jj < final_rank ? pv[jj] + off : -1;
        if (tid == 0) a.rank[unit] = final_rank;
    }
    cluster.sync();  // no block leaves while a peer may still write to its shared memory
}

struct SelectPlan {
    int C = 0, m = 0;   // blocks per unit, rows per block
    long cap = 0;       // blocks the GPU holds at once with m rows each
    int per_sm = 0;     // of those, a SM's
};

// Most blocks per unit such that every block of the launch is co-resident
// (they wait on each other), at >= 256 rows per block; else the fewest blocks
// the shared memory allows, in co-resident waves.
template <typename T, typename TK, int NT>
wc_status plan_select(const Shape& s, int nsm, int max_smem, int m_max, SelectPlan* p) {
    auto kern = rpcholesky_kernel<T, TK, NT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem - 1024) != cudaSuccess)
        return WC_ERR_CUDA;
    auto blocks_per_sm = [&](int m) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, NT, select_smem_bytes(m, s.r, s.d)) != cudaSuccess)
            return 0;
        return b;
    };
    auto rows_for = [&](int C) { return ((s.n + C - 1) / C + kRowAlign - 1) / kRowAlign * kRowAlign; };
    const int c_min = (s.n + m_max - 1) / m_max;
    int c_hi = (s.n + 255) / 256;
    if (c_hi > kMaxBlocksPerUnit) c_hi = kMaxBlocksPerUnit;
    if (c_hi < c_min) c_hi = c_min;
    int m = rows_for(c_min);
    int bps = blocks_per_sm(m);
    for (int c = c_hi; c > c_min; --c) {
        const int mc = rows_for(c);
        const int ce = (s.n + mc - 1) / mc;
        const int bc = blocks_per_sm(mc);
        if ((long)s.units * ce <= (long)nsm * bc) {
            m = mc;
            bps = bc;
            break;
        }
    }
    p->m = m;
    p->C = (s.n + m - 1) / m;
    p->per_sm = bps;
    p->cap = (long)nsm * bps;
    return WC_OK;
}

template <typename T, typename TK, int NT>
wc_status run_select(const Shape& s, const SelectPlan& p, SelectArgs a, char* ws, cudaStream_t st) {
    auto kern = rpcholesky_kernel<T, TK, NT>;
    const size_t smem = select_smem_bytes(p.m, s.r, s.d);
    if (p.C == 1) {
        a.unit0 = 0;
        kern<<<s.units, NT, smem, st>>>(a);
        return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
    }
    // blocks of a unit wait on each other: co-resident waves, cooperative launch
    // (the launch attribute form, which stream capture into a CUDA graph takes)
    const int per_wave = (int)(p.cap / p.C);
    if (per_wave < 1) return WC_ERR_UNSUPPORTED;
    for (int u0 = 0; u0 < s.units; u0 += per_wave) {
        a.unit0 = u0;
        const int nu = s.units - u0 < per_wave ? s.units - u0 : per_wave;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(nu * p.C);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

// Cluster size and rows per block of the resident variant, or false where a
// unit does not fit in the shared memory of kMaxCluster blocks or the units
// do not all fit on the GPU at once.  The fewest blocks per unit that hold
// it, doubled while the launch would leave more than half of the SMs idle and
// blocks keep at least 128 rows.
template <typename T, typename TK, int NT>
bool plan_resident(const Shape& s, int nsm, int max_smem, int* cl_out, int* m_out, size_t* smem_out) {
    auto rows_for = [&](int cl) { return ((s.n + cl - 1) / cl + 63) / 64 * 64; };
    const size_t avail = (size_t)max_smem - 1024;
    int cl = 1;
    while (cl <= kMaxCluster && ResidentSmem(rows_for(cl), s.r, s.d, (int)sizeof(TK), NT).total > avail) cl *= 2;
    if (cl > kMaxCluster) return false;
    while (cl < kMaxCluster && (long)s.units * cl * 2 <= nsm && (s.n + 2 * cl - 1) / (2 * cl) >= 128) cl *= 2;
    const int m = rows_for(cl);
    if ((long)(cl - 1) * m >= s.n) return false;  // every block of a unit holds rows
    const size_t smem = ResidentSmem(m, s.r, s.d, (int)sizeof(TK), NT).total;
    auto kern = rpcholesky_resident_kernel<T, TK, NT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.units * cl));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
        cudaGetLastError();
        return false;
    }
    // A resident unit holds its whole factor in shared memory, so far fewer
    // units run at once than in the streaming kernel (ViT-sized heads: about 80
    // against about 300).  Its step is shorter, which pays only while every
    // unit runs at once.
    if (s.units > clusters) return false;
    *cl_out = cl;
    *m_out = m;
    *smem_out = smem;
    return true;
}

template <typename T, typename TK, int NT>
wc_status run_resident(const Shape& s, int cl, size_t smem, const SelectArgs& a, cudaStream_t st) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.units * cl));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rpcholesky_resident_kernel<T, TK, NT>, a) == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

template <typename T, typename TK>
wc_status launch_select_t(const Shape& s, const void* K, int32_t* piv, float* F, int32_t* rank, char* ws,
                          cudaStream_t st) {
    const WsLayout L = make_layout(s);
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WC_ERR_CUDA;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return WC_ERR_CUDA;
    int max_smem = 0;
    cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);

    // rows per block bounded by shared memory (fp64 diagonal + flags)
    const size_t fixed = select_smem_bytes(0, s.r, s.d) + 1024;
    if ((size_t)max_smem <= fixed) return WC_ERR_UNSUPPORTED;
    int m_max = (int)(((size_t)max_smem - fixed) / 9) / kRowAlign * kRowAlign;
    m_max = m_max > (1 << 20) ? (1 << 20) : m_max;

    SelectArgs a;
    a.K = K; a.piv = piv; a.F = F; a.rank = rank;
    a.bins = s.bins;
    a.bin_keys = s.n;
    a.unit_base = (uint32_t)s.unit_base * (uint32_t)s.bins;   // bin view: unit u * bins + bin
    a.kbar = s.center ? reinterpret_cast<const double*>(ws + L.kbar) : nullptr;
    a.Kt = ws + L.kt;
    a.sync = reinterpret_cast<UnitSync*>(ws + L.sync);
    a.partials = reinterpret_cast<double*>(ws + L.partials);
    a.status = reinterpret_cast<int*>(ws + L.status);
    a.ldf = s.ldf; a.n = s.n; a.d = s.d; a.r = s.r;
    a.beta = s.beta; a.eps = s.eps; a.seed = s.seed; a.timeout_ns = s.timeout_ns;
    a.unit0 = 0;

    // short units: keys and factor resident in the shared memory of a cluster
    {
        int cl = 0, m = 0;
        size_t smem = 0;
        if (plan_resident<T, TK, kResThreads>(s, nsm, max_smem, &cl, &m, &smem)) {
            a.C = cl;
            a.m = m;
            return run_resident<T, TK, kResThreads>(s, cl, smem, a, st);
        }
    }

    // 256-thread blocks, unless the launch is one co-resident wave either way
    // and 128-thread blocks leave the busiest SM fewer rows: with 2 blocks per
    // SM, units that are many and short (bins) leave SMs idle
    SelectPlan p256, p128;
    wc_status e = plan_select<T, TK, 256>(s, nsm, max_smem, m_max, &p256);
    if (e != WC_OK) return e;
    if ((e = plan_select<T, TK, 128>(s, nsm, max_smem, m_max, &p128)) != WC_OK) return e;
    auto one_wave = [&](const SelectPlan& p) { return p.C > 1 && (long)s.units * p.C <= p.cap; };
    auto sm_rows = [&](const SelectPlan& p) {
        const long blocks = (long)s.units * p.C;
        const long per_sm = (blocks + nsm - 1) / nsm;
        return (long)p.m * (per_sm < p.per_sm ? per_sm : p.per_sm);
    };
    const bool use128 = one_wave(p256) && one_wave(p128) && sm_rows(p128) * 100 < sm_rows(p256) * 97;
    const SelectPlan& p = use128 ? p128 : p256;
    if (p.cap < 1) return WC_ERR_CUDA;
    if (p.C > kMaxBlocksPerUnit) return WC_ERR_UNSUPPORTED;

    a.C = p.C; a.m = p.m;

    // units of 2 to kMaxCluster blocks: a cluster per unit
    if (!use128 && p.C >= 2 && p.C <= kMaxCluster) {
        auto kern = rpcholesky_cluster_kernel<T, TK>;
        const size_t csmem = ClusterSmem(p.m, s.r, s.d).total;
        if (csmem + 1024 <= (size_t)max_smem &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem) == cudaSuccess) {
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)p.C;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(s.units * p.C));
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = csmem;
            cfg.stream = st;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters >= 1) {
                a.unit0 = 0;
                return cudaLaunchKernelEx(&cfg, kern, a) == cudaSuccess ? WC_OK : WC_ERR_CUDA;
            }
        }
        cudaGetLastError();
    }

    // many short units: one block per unit, keys in shared memory
    if (s.units >= nsm && s.ldf <= 2 * kUnitThreads) {
        const size_t usmem = UnitSmem((int)s.ldf, s.r, s.d, (int)sizeof(TK)).total;
        if (usmem + 1024 <= (size_t)max_smem) {
            auto kern = rpcholesky_unit_kernel<T, TK>;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)usmem) != cudaSuccess)
                return WC_ERR_CUDA;
            a.C = 1;
            a.m = (int)s.ldf;
            kern<<<s.units, kUnitThreads, usmem, st>>>(a);
            return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
        }
    }

    if (cudaMemsetAsync(ws + L.sync, 0, sizeof(UnitSync) * (size_t)s.units, st) != cudaSuccess) return WC_ERR_CUDA;
    return use128 ? run_select<T, TK, 128>(s, p, a, ws, st) : run_select<T, TK, 256>(s, p, a, ws, st);
}

// Two blocks meet at a unit barrier that block 1 never reaches: block 0's
// bounded wait runs out and records WC_ERR_TIMEOUT.
__global__ void wait_selftest_kernel(UnitSync* sync, int* status, uint64_t timeout_ns) {
    __shared__ int ok;
    if (blockIdx.x == 1) return;
    unit_barrier(&sync->bar, 2, 1, timeout_ns, status, &ok);
}

}  // namespace

wc_status launch_select(const Shape& s, const void* K, int32_t* piv, float* F, int32_t* rank, char* ws,
                        cudaStream_t st) {
    if (s.dtype == WC_BF16) {
        if (s.center) return launch_select_t<__nv_bfloat16, float>(s, K, piv, F, rank, ws, st);
        return launch_select_t<__nv_bfloat16, __nv_bfloat16>(s, K, piv, F, rank, ws, st);
    }
    return launch_select_t<float, float>(s, K, piv, F, rank, ws, st);
}

wc_status launch_wait_selftest(char* ws, uint64_t timeout_ns, cudaStream_t st) {
    UnitSync* sync = reinterpret_cast<UnitSync*>(ws + 256);
    int* status = reinterpret_cast<int*>(ws);
    if (cudaMemsetAsync(sync, 0, sizeof(UnitSync), st) != cudaSuccess) return WC_ERR_CUDA;
    wait_selftest_kernel<<<2, 32, 0, st>>>(sync, status, timeout_ns);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace wc

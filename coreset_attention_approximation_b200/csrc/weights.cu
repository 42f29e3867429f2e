// weights.cu — Nystrom weights on the coreset.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gist.science
// technical summary, "Methodik" item 2): W = h(K_S,K_S)^+ h(K_S,K), values
// compressed as V_S = W V.  Here the weights act on [V | 1], so the softmax
// normaliser is compressed with the values:
//   C1 = exp(beta K_S K^T) [V | 1]           (gather + exp-GEMM, split over keys)
//   W  = L^-T (L^-1 C1),  L = F[piv, :rank]  (fp64 triangular solves, a warp per 4 columns)
// L L^T = h(K_S, K_S) because the pivot rows of the RPCholesky factor are the
// Cholesky factor of the kernel matrix on the coreset (in pivot order).
#include "wc_common.cuh"
#include "wc_internal.h"
#include "wc_expmm.cuh"

namespace wc {
namespace {

// Ks[u, a, :] = K[u, piv[a], :] and Lg[u, a, b] = F[u, b, piv[a]] (b <= a),
// zero beyond rank.  One block per (a, u).
template <typename T>
__global__ void gather_kernel(const T* __restrict__ K, const int32_t* __restrict__ piv,
                              const float* __restrict__ F, const int32_t* __restrict__ rank, T* Ks,
                              float* Lg, int n, int d, int r, int64_t ldf) {
    const int a = blockIdx.x, u = blockIdx.y;
    const int k = rank[u];
    const int p = a < k ? piv[(size_t)u * r + a] : -1;
    T* ks = Ks + ((size_t)u * r + a) * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x)
        ks[c] = p >= 0 ? K[((size_t)u * n + p) * d + c] : T(0.f);
    float* lrow = Lg + ((size_t)u * r + a) * r;
    const float* Fu = F + (size_t)u * r * ldf;
    for (int b = threadIdx.x; b < r; b += blockDim.x)
        lrow[b] = (p >= 0 && b <= a) ? Fu[(int64_t)b * ldf + p] : 0.f;
}

constexpr int kCols = 4;  // right-hand-side columns per solving warp

// C1 from the partial sums of the key splits, in fp64:
//   C1[a, c] = e^M sum_s e^{m_s - M} O_s[a, c],  M = max_s m_s
// written column-major, Ct[u, c, a], for the solves.  One block per (a, u).
__global__ void merge_c1_kernel(const float* __restrict__ c1part, const int32_t* __restrict__ rank, double* Ct,
                                int nsplit, int r, int dv) {
    const int a = blockIdx.x, u = blockIdx.y;
    if (a >= rank[u]) return;
    const int w = dv + 2, wcols = dv + 1;
    const float* part = c1part + (size_t)u * nsplit * r * w;
    double mx = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) mx = fmax(mx, (double)part[((size_t)sp * r + a) * w + dv + 1]);
    for (int c = threadIdx.x; c < wcols; c += blockDim.x) {
        double acc = 0.0;
        if (mx > -INFINITY) {
            for (int sp = 0; sp < nsplit; ++sp) {
                const float* row = part + ((size_t)sp * r + a) * w;
                const double ms = (double)row[dv + 1];
                if (ms > -INFINITY) acc += exp(ms - mx) * (double)row[c];
            }
            acc *= exp(mx);
        }
        Ct[((size_t)u * wcols + c) * r + a] = acc;
    }
}

// W = L^-T (L^-1 C1) for kCols right-hand sides of one unit, one warp, fp64,
// in blocks of 32 rows.  Forward, block [a0, a0+32): lane i owns row a0+i,
// subtracts L[a0+i, :a0] y[:a0] (its own row of L, independent loads), then the
// 32 x 32 diagonal block is solved through shuffles.  Backward, blocks from the
// last: lane i owns entry a0+i, subtracts sum_{b >= a0+32} L[b, a0+i] x_b (row
// segments of L, coalesced across the warp), then the diagonal block.
// y / x live in shared memory, [kCols][r].
__global__ void __launch_bounds__(32) trsv_kernel(const float* __restrict__ Lg, const int32_t* __restrict__ rank,
                                                  const double* __restrict__ Ct, float* W, int r, int dv) {
    extern __shared__ double ys[];
    const int u = blockIdx.y;
    const int wcols = dv + 1;
    const int c0 = blockIdx.x * kCols;
    const int nc = min(kCols, wcols - c0);
    const int k = rank[u];
    const float* L = Lg + (size_t)u * r * r;
    const double* C = Ct + (size_t)u * wcols * r;
    float* Wu = W + (size_t)u * r * wcols;
    const int lane = threadIdx.x;

    // ---- forward: L y = c
    for (int a0 = 0; a0 < k; a0 += 32) {
        const int a = a0 + lane;
        const bool live = a < k;
        double acc[kCols];
#pragma unroll
        for (int q = 0; q < kCols; ++q) acc[q] = (live && q < nc) ? C[(size_t)(c0 + q) * r + a] : 0.0;
        float lb[32];  // this row's entries in the diagonal block
        if (live) {
            const float* La = L + (size_t)a * r;
#pragma unroll 8
            for (int b = 0; b < a0; ++b) {
                const double l = (double)La[b];
#pragma unroll
                for (int q = 0; q < kCols; ++q) acc[q] -= l * ys[q * r + b];
            }
#pragma unroll
            for (int t = 0; t < 32; ++t) lb[t] = (a0 + t < k) ? La[a0 + t] : 0.f;
        } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) lb[t] = 0.f;
        }
        const int rows = min(32, k - a0);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i < rows) {
                double yi[kCols];
#pragma unroll
                for (int q = 0; q < kCols; ++q) {
                    const double v = (lane == i) ? acc[q] / (double)lb[i] : 0.0;
                    yi[q] = __shfl_sync(0xffffffffu, v, i);
                }
                if (lane == i) {
#pragma unroll
                    for (int q = 0; q < kCols; ++q) ys[q * r + a] = yi[q];
                }
                if (lane > i) {
                    const double l = (double)lb[i];
#pragma unroll
                    for (int q = 0; q < kCols; ++q) acc[q] -= l * yi[q];
                }
            }
        }
        __syncwarp();
    }

    // ---- backward: L^T x = y
    for (int a0 = (k - 1) / 32 * 32; k > 0 && a0 >= 0; a0 -= 32) {
        const int a = a0 + lane;
        const bool live = a < k;
        double acc[kCols];
#pragma unroll
        for (int q = 0; q < kCols; ++q) acc[q] = live ? ys[q * r + a] : 0.0;
#pragma unroll 8
        for (int b = a0 + 32; b < k; ++b) {
            const double l = live ? (double)L[(size_t)b * r + a] : 0.0;
#pragma unroll
            for (int q = 0; q < kCols; ++q) acc[q] -= l * ys[q * r + b];
        }
        float lt[32];  // lt[i] = L[a0 + i, a]: this entry's column of the diagonal block
#pragma unroll
        for (int i = 0; i < 32; ++i) lt[i] = (live && a0 + i < k) ? L[(size_t)(a0 + i) * r + a] : 0.f;
        const int rows = min(32, k - a0);
#pragma unroll
        for (int i = 31; i >= 0; --i) {
            if (i < rows) {
                double xi[kCols];
#pragma unroll
                for (int q = 0; q < kCols; ++q) {
                    const double v = (lane == i) ? acc[q] / (double)lt[i] : 0.0;
                    xi[q] = __shfl_sync(0xffffffffu, v, i);
                }
                if (lane == i) {
#pragma unroll
                    for (int q = 0; q < kCols; ++q) ys[q * r + a] = xi[q];
                }
                if (lane < i) {
                    const double l = (double)lt[i];
#pragma unroll
                    for (int q = 0; q < kCols; ++q) acc[q] -= l * xi[q];
                }
            }
        }
        __syncwarp();
    }
    for (int q = 0; q < nc; ++q)
        for (int a = lane; a < r; a += 32) Wu[(size_t)a * wcols + c0 + q] = a < k ? (float)ys[q * r + a] : 0.f;
}

}  // namespace

wc_status launch_gather(const Shape& s, const void* K, const int32_t* piv, const float* F, const int32_t* rank,
                        void* Ks, char* ws, cudaStream_t st) {
    const WsLayout L = make_layout(s);
    float* Lg = reinterpret_cast<float*>(ws + L.lg);
    dim3 grid(s.r, s.units);
    if (s.dtype == WC_BF16)
        gather_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(K), piv, F, rank,
                                                           static_cast<__nv_bfloat16*>(Ks), Lg, s.n, s.d, s.r,
                                                           s.ldf);
    else
        gather_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(K), piv, F, rank,
                                                   static_cast<float*>(Ks), Lg, s.n, s.d, s.r, s.ldf);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

wc_status launch_coreset_values(const Shape& s, const void* Ks, const void* K, const void* V, const int32_t* rank,
                                char* ws, cudaStream_t st) {
    if (tc_supported(s)) return launch_coreset_values_tc(s, Ks, K, V, rank, ws, st);
    const WsLayout L = make_layout(s);
    ExpmmArgs e{};
    e.A = Ks; e.a_stride = (int64_t)s.r * s.d; e.a_rows = s.r;
    e.B = K; e.b_stride = (int64_t)s.n * s.d; e.b_rows = s.n;
    e.C = V; e.c_stride = (int64_t)s.n * s.dv; e.ldc = s.dv;
    e.wcol = nullptr;
    e.rank = rank;
    e.out = ws + L.c1part;
    e.d = s.d; e.dv = s.dv; e.r = s.r;
    e.nsplit = s.nsplit; e.split_len = kSplitKeys;
    e.beta = (float)s.beta;
    e.group = 1; e.hq = s.hkv;
    e.mode = kExpmmPartial;
    return launch_expmm_simt(e, s.dtype, s.units, st);
}

wc_status launch_solve(const Shape& s, const int32_t* rank, float* W, char* ws, cudaStream_t st) {
    const WsLayout L = make_layout(s);
    double* Ct = reinterpret_cast<double*>(ws + L.y);
    merge_c1_kernel<<<dim3(s.r, s.units), 160, 0, st>>>(reinterpret_cast<const float*>(ws + L.c1part), rank, Ct,
                                                        s.nsplit, s.r, s.dv);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
    const size_t smem = sizeof(double) * kCols * (size_t)s.r;
    if (cudaFuncSetAttribute(trsv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return WC_ERR_CUDA;
    trsv_kernel<<<dim3((s.dv + 1 + kCols - 1) / kCols, s.units), 32, smem, st>>>(
        reinterpret_cast<const float*>(ws + L.lg), rank, Ct, W, s.r, s.dv);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace wc

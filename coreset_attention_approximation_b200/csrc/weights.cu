// weights.cu — Nystrom weights on the coreset.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gist.science
// technical summary, "Methodik" item 2): W = h(K_S,K_S)^+ h(K_S,K), values
// compressed as V_S = W V.  Here the weights act on [V | 1], so the softmax
// normaliser is compressed with the values:
//   C1 = exp(beta K_S K^T) [V | 1]           (gather + exp-GEMM, split over keys)
//   W  = L^-T (L^-1 C1),  L = F[piv, :rank]  (blocked fp64 triangular solves)
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

constexpr int kTile = 32;      // rows per solve block / columns per solve CTA
constexpr int kSolveThreads = 256;

// Merge the C1 partials of row a, column c (fp64): sum_s e^{m_s} O_s.
__device__ __forceinline__ double merged_c1(const float* part, int nsplit, int r, int dv, int a, int c) {
    const int w = dv + 2;
    double mx = -INFINITY;
    for (int s = 0; s < nsplit; ++s) mx = fmax(mx, (double)part[((size_t)s * r + a) * w + dv + 1]);
    if (!(mx > -INFINITY)) return 0.0;
    double acc = 0.0;
    for (int s = 0; s < nsplit; ++s) {
        const float* row = part + ((size_t)s * r + a) * w;
        const double ms = (double)row[dv + 1];
        if (ms > -INFINITY) acc += exp(ms - mx) * (double)row[c];
    }
    return acc * exp(mx);
}

// One block per (column tile, unit): forward then backward substitution on
// kTile columns of C1, in kTile x kTile blocks, fp64 throughout.
__global__ void __launch_bounds__(kSolveThreads) solve_kernel(const float* __restrict__ c1part,
                                                              const float* __restrict__ Lg,
                                                              const int32_t* __restrict__ rank, double* Y,
                                                              float* W, int nsplit, int r, int dv) {
    const int u = blockIdx.y;
    const int c0 = blockIdx.x * kTile;
    const int wcols = dv + 1;
    const int ncol = min(kTile, wcols - c0);
    const int k = rank[u];
    const float* L = Lg + (size_t)u * r * r;
    const float* part = c1part + (size_t)u * nsplit * r * (dv + 2);
    double* Yu = Y + (size_t)u * r * wcols;
    float* Wu = W + (size_t)u * r * wcols;
    const int tid = threadIdx.x;

    __shared__ double Ls[kTile][kTile + 1];
    __shared__ double Ys[kTile][kTile + 1];
    __shared__ double Yd[kTile][kTile + 1];  // the diagonal block being solved

    // thread -> (row ra, columns ca + 8q)
    const int ra = tid / 8, ca = tid % 8;

    // ---- forward: L Y = C1
    for (int a0 = 0; a0 < k; a0 += kTile) {
        const int rows = min(kTile, k - a0);
        double acc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = ca + 8 * q;
            acc[q] = (ra < rows && c < ncol) ? merged_c1(part, nsplit, r, dv, a0 + ra, c0 + c) : 0.0;
        }
        for (int b0 = 0; b0 < a0; b0 += kTile) {
            for (int e = tid; e < kTile * kTile; e += kSolveThreads) {
                const int i = e / kTile, jj = e % kTile;
                Ls[i][jj] = (i < rows) ? (double)L[(size_t)(a0 + i) * r + b0 + jj] : 0.0;
                Ys[i][jj] = (jj < ncol) ? Yu[(size_t)(b0 + i) * wcols + c0 + jj] : 0.0;
            }
            __syncthreads();
#pragma unroll 4
            for (int b = 0; b < kTile; ++b) {
                const double l = Ls[ra][b];
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] -= l * Ys[b][ca + 8 * q];
            }
            __syncthreads();
        }
        // diagonal block
        for (int e = tid; e < kTile * kTile; e += kSolveThreads) {
            const int i = e / kTile, jj = e % kTile;
            Ls[i][jj] = (i < rows && jj < rows) ? (double)L[(size_t)(a0 + i) * r + a0 + jj] : 0.0;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) Yd[ra][ca + 8 * q] = acc[q];
        __syncthreads();
        if (tid < ncol) {
            for (int i = 0; i < rows; ++i) {
                double v = Yd[i][tid];
                for (int b = 0; b < i; ++b) v -= Ls[i][b] * Yd[b][tid];
                Yd[i][tid] = v / Ls[i][i];
            }
        }
        __syncthreads();
        for (int e = tid; e < rows * ncol; e += kSolveThreads) {
            const int i = e / ncol, c = e % ncol;
            Yu[(size_t)(a0 + i) * wcols + c0 + c] = Yd[i][c];
        }
        __syncthreads();
    }

    // ---- backward: L^T W = Y, blocks from the last
    const int nblk = (k + kTile - 1) / kTile;
    for (int bi = nblk - 1; bi >= 0; --bi) {
        const int a0 = bi * kTile;
        const int rows = min(kTile, k - a0);
        double acc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = ca + 8 * q;
            acc[q] = (ra < rows && c < ncol) ? Yu[(size_t)(a0 + ra) * wcols + c0 + c] : 0.0;
        }
        for (int b0 = a0 + kTile; b0 < k; b0 += kTile) {
            const int brows = min(kTile, k - b0);
            for (int e = tid; e < kTile * kTile; e += kSolveThreads) {
                const int i = e / kTile, jj = e % kTile;
                // Ls[i][jj] = L[b0 + jj][a0 + i]  (transposed block)
                Ls[i][jj] = (i < rows && jj < brows) ? (double)L[(size_t)(b0 + jj) * r + a0 + i] : 0.0;
                Ys[i][jj] = (i < brows && jj < ncol) ? Yu[(size_t)(b0 + i) * wcols + c0 + jj] : 0.0;
            }
            __syncthreads();
#pragma unroll 4
            for (int b = 0; b < kTile; ++b) {
                const double l = Ls[ra][b];
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] -= l * Ys[b][ca + 8 * q];
            }
            __syncthreads();
        }
        for (int e = tid; e < kTile * kTile; e += kSolveThreads) {
            const int i = e / kTile, jj = e % kTile;
            Ls[i][jj] = (i < rows && jj < rows) ? (double)L[(size_t)(a0 + i) * r + a0 + jj] : 0.0;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) Yd[ra][ca + 8 * q] = acc[q];
        __syncthreads();
        if (tid < ncol) {
            for (int i = rows - 1; i >= 0; --i) {
                double v = Yd[i][tid];
                for (int b = i + 1; b < rows; ++b) v -= Ls[b][i] * Yd[b][tid];
                Yd[i][tid] = v / Ls[i][i];
            }
        }
        __syncthreads();
        for (int e = tid; e < rows * ncol; e += kSolveThreads) {
            const int i = e / ncol, c = e % ncol;
            Yu[(size_t)(a0 + i) * wcols + c0 + c] = Yd[i][c];
            Wu[(size_t)(a0 + i) * wcols + c0 + c] = (float)Yd[i][c];
        }
        __syncthreads();
    }
    // rows >= rank are zero
    for (int e = tid; e < (r - k) * ncol; e += kSolveThreads) {
        const int i = k + e / ncol, c = e % ncol;
        Wu[(size_t)i * wcols + c0 + c] = 0.f;
    }
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
    dim3 grid((s.dv + 1 + kTile - 1) / kTile, s.units);
    solve_kernel<<<grid, kSolveThreads, 0, st>>>(reinterpret_cast<const float*>(ws + L.c1part),
                                                 reinterpret_cast<const float*>(ws + L.lg), rank,
                                                 reinterpret_cast<double*>(ws + L.y), W, s.nsplit, s.r, s.dv);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace wc

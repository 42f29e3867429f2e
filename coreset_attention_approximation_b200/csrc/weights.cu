// weights.cu — Nystrom weights on the coreset.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gist.science
// technical summary, "Methodik" item 2): W = h(K_S,K_S)^+ h(K_S,K), values
// compressed as V_S = W V.  Here the weights act on [V | 1], so the softmax
// normaliser is compressed with the values:
//   C1 = exp(beta K_S K^T) [V | 1]           (gather + exp-GEMM, split over keys)
//   W  = L^-T (L^-1 C1),  L = F[piv, :rank]  (blocked fp64 triangular solves, 2-8 columns a block)
// L L^T = h(K_S, K_S) because the pivot rows of the RPCholesky factor are the
// Cholesky factor of the kernel matrix on the coreset (in pivot order).
#include "wc_common.cuh"
#include "wc_internal.h"
#include "wc_expmm.cuh"

namespace wc {
namespace {

// Ks[u, a, :] = K[u, piv[a], :] and Lg[u, a, b] = F[u, b, piv[a]] (b <= a),
// zero beyond rank.  One block per (a, u).  With bins, u is bin u % bins of its
// caller unit: pivot indices count from the caller unit's first key, and Ks rows
// beyond the bin's rank repeat the bin's first pivot key (their weights are
// zero, and a real key's logit leaves the row maxima of the attention intact).
template <typename T>
__global__ void gather_kernel(const T* __restrict__ K, const int32_t* __restrict__ piv,
                              const float* __restrict__ F, const int32_t* __restrict__ rank, T* Ks,
                              float* Lg, int n, int d, int r, int64_t ldf, int bins, int tpr, int* status) {
    // tpr threads a row, blockDim.x / tpr rows a block
    const int a = blockIdx.x * (blockDim.x / tpr) + threadIdx.x / tpr, u = blockIdx.y, t = threadIdx.x % tpr;
    if (a >= r) return;
    int k = rank[u];
    if (!in_bounds(k >= 0 && k <= r, status)) k = 0;
    const int base = (u % bins) * n;  // the bin's first key within the caller's unit
    int p = a < k ? piv[(size_t)u * r + a] - base : -1;
    int pk = p >= 0 ? p : (bins > 1 && k > 0 ? piv[(size_t)u * r] - base : -1);
    if (!in_bounds(a >= k || (p >= 0 && p < n), status)) p = -1;
    if (!in_bounds(pk < n && (pk >= 0 || a >= k), status)) pk = -1;
    T* ks = Ks + ((size_t)u * r + a) * d;
    for (int c = t; c < d; c += tpr) ks[c] = pk >= 0 ? K[((size_t)u * n + pk) * d + c] : T(0.f);
    float* lrow = Lg + ((size_t)u * r + a) * r;
    const float* Fu = F + (size_t)u * r * ldf;
    for (int b = t; b < r; b += tpr) lrow[b] = (p >= 0 && b <= a) ? Fu[(int64_t)b * ldf + p] : 0.f;
}

// C1 from the partial sums of the key splits, in fp64:
//   C1[a, c] = e^(M + rho_a) sum_s e^{m_s - M} O_s[a, c],  M = max_s m_s
// written column-major, Ct[u, c, a], for the solves.  rho_a = -shift_u (the
// factor's shift, so that C1 is taken of the same shifted kernel as L), plus,
// with centred keys, beta (|kbar|^2 - <k_s, kbar>) for the pivot s of row a (the
// per-row factor of the centred kernel).  One block per (a, u).
__global__ void merge_c1_kernel(const float* __restrict__ c1part, const int32_t* __restrict__ rank, double* Ct,
                                int nsplit, int r, int dv, const int32_t* __restrict__ piv,
                                const double* __restrict__ cdot, const double* __restrict__ kk, int bins, int n_all,
                                double beta, const double* __restrict__ shift, int tpr, int* status) {
    // tpr threads a coreset row, blockDim.x / tpr rows a block
    const int a = blockIdx.x * (blockDim.x / tpr) + threadIdx.x / tpr, u = blockIdx.y, t = threadIdx.x % tpr;
    if (a >= r) return;
    if (a >= rank[u] || !in_bounds(rank[u] <= r, status)) return;
    double rho = -shift[u];
    if (cdot) {
        const int uc = u / bins;  // the caller's unit
        const int p = piv[(size_t)u * r + a];
        if (!in_bounds(p >= 0 && p < n_all, status)) return;
        rho += beta * (kk[uc] - cdot[(size_t)uc * n_all + p]);
    }
    const int w = c1_row(dv), wcols = dv + 1;
    const float* part = c1part + (size_t)u * nsplit * r * w;
    double mx = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) mx = fmax(mx, (double)part[((size_t)sp * r + a) * w + dv + 1]);
    for (int c = t; c < wcols; c += tpr) {
        double acc = 0.0;
        if (mx > -INFINITY) {
            for (int sp = 0; sp < nsplit; ++sp) {
                const float* row = part + ((size_t)sp * r + a) * w;
                const double ms = (double)row[dv + 1];
                if (ms > -INFINITY) acc += exp(ms - mx) * (double)row[c];
            }
            acc *= exp(mx + rho);
        }
        Ct[((size_t)u * wcols + c) * r + a] = acc;
    }
}

// W = L^-T (L^-1 C1) for NC right-hand-side columns of one unit, fp64, blocked
// by 64 rows (right-looking).  The NC columns live in shared memory (Y, row
// major [r][NC]) for the whole solve.
//   forward, block K = [kb, kb + 64):  Y_K <- L_KK^-1 Y_K (one warp per column,
//     lanes own rows kb + lane and kb + lane + 32, the diagonal block staged in
//     shared memory), then every later row i: Y_i -= L[i, K] Y_K (one thread
//     per row; a thread reads its row segment of L).
//   backward, blocks from the last:  Y_K <- L_KK^-T Y_K, then every earlier row
//     i: Y_i -= L[K, i]^T Y_K (threads over i read rows of L: coalesced).
// Rows at and beyond the rank are left out; W rows there are written as zero.
constexpr int kTB = 64;           // rows per diagonal block
constexpr int kTrsmThreads = 256;

// One 16-entry chunk c of row i's panel segment against the block K = [kb, kb + 64):
// forward L[i, kb + 16 c + e] (row major; float4 loads when rows start on 16
// bytes), backward L[kb + 16 c + e, i] (coalesced across the threads' rows).
template <bool kForward>
__device__ __forceinline__ void load_chunk(const float* L, int r, int i, int kb, int c, bool vec, float (&v)[16]) {
    if (kForward) {
        const float* p = L + (size_t)i * r + kb + 16 * c;
        if (vec) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 x = __ldg(reinterpret_cast<const float4*>(p + e));
                v[e] = x.x; v[e + 1] = x.y; v[e + 2] = x.z; v[e + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __ldg(p + e);
        }
    } else {
        const float* p = L + (size_t)(kb + 16 * c) * r + i;
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = __ldg(p + (size_t)e * r);
    }
}

template <int NC>
__device__ __forceinline__ void apply_chunk(double (&acc)[NC], const double* Y, int kb, int c, const float (&v)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const double l = (double)v[e];
        const double* yb = Y + (kb + 16 * c + e) * NC;
#pragma unroll
        for (int q = 0; q < NC; ++q) acc[q] = fma(-l, yb[q], acc[q]);
    }
}

// acc0 / acc1 (rows i0, i1) -= chunk c of their panel segments times Y_K: each
// Y_K entry read from shared memory serves both rows.
template <int NC>
__device__ __forceinline__ void apply_chunk2(double (&acc0)[NC], double (&acc1)[NC], const double* Y, int kb, int c,
                                             const float (&v0)[16], const float (&v1)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const double l0 = (double)v0[e], l1 = (double)v1[e];
        const double* yb = Y + (kb + 16 * c + e) * NC;
#pragma unroll
        for (int q = 0; q < NC; ++q) {
            const double y = yb[q];
            acc0[q] = fma(-l0, y, acc0[q]);
            acc1[q] = fma(-l1, y, acc1[q]);
        }
    }
}

// Rows i = first, first + stride, ... < end:  Y_i -= L-panel(i) Y_K for a whole
// 64-row block K.  The update is bound by load latency and shared-memory
// reads, not by the fp64 pipe: each thread keeps the next 16-entry chunk of
// its panel segments in flight while it applies the current one, and with
// ROWS = 2 takes two rows at a time (i, i + stride), so each Y_K entry it
// reads from shared memory feeds two fused multiply-adds (twice the registers:
// one block per SM; worth it when the panels are long, large r).
template <int NC, bool kForward, int ROWS>
__device__ void panel_update(double* Y, const float* L, int r, int kb, int first, int end, int stride, bool vec) {
    if constexpr (ROWS == 1) {
        if (first >= end) return;
        float P[16], Q[16];
        load_chunk<kForward>(L, r, first, kb, 0, vec, P);
        for (int i = first; i < end; i += stride) {
            double acc[NC];
#pragma unroll
            for (int q = 0; q < NC; ++q) acc[q] = Y[i * NC + q];
            load_chunk<kForward>(L, r, i, kb, 1, vec, Q);
            apply_chunk<NC>(acc, Y, kb, 0, P);
            load_chunk<kForward>(L, r, i, kb, 2, vec, P);
            apply_chunk<NC>(acc, Y, kb, 1, Q);
            load_chunk<kForward>(L, r, i, kb, 3, vec, Q);
            apply_chunk<NC>(acc, Y, kb, 2, P);
            if (i + stride < end) load_chunk<kForward>(L, r, i + stride, kb, 0, vec, P);
            apply_chunk<NC>(acc, Y, kb, 3, Q);
#pragma unroll
            for (int q = 0; q < NC; ++q) Y[i * NC + q] = acc[q];
        }
    } else {
    for (int i0 = first; i0 < end; i0 += 2 * stride) {
        const int i1 = i0 + stride;
        const bool two = i1 < end;
        double acc0[NC], acc1[NC];
#pragma unroll
        for (int q = 0; q < NC; ++q) {
            acc0[q] = Y[i0 * NC + q];
            acc1[q] = two ? Y[i1 * NC + q] : 0.0;
        }
        float P0[16], P1[16], Q0[16], Q1[16];
        load_chunk<kForward>(L, r, i0, kb, 0, vec, P0);
        if (two) load_chunk<kForward>(L, r, i1, kb, 0, vec, P1);
        else
#pragma unroll
            for (int e = 0; e < 16; ++e) P1[e] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
            load_chunk<kForward>(L, r, i0, kb, c + 1, vec, Q0);
            if (two) load_chunk<kForward>(L, r, i1, kb, c + 1, vec, Q1);
            else
#pragma unroll
                for (int e = 0; e < 16; ++e) Q1[e] = 0.f;
            apply_chunk2<NC>(acc0, acc1, Y, kb, c, P0, P1);
            if (c + 2 < 4) {
                load_chunk<kForward>(L, r, i0, kb, c + 2, vec, P0);
                if (two) load_chunk<kForward>(L, r, i1, kb, c + 2, vec, P1);
            }
            apply_chunk2<NC>(acc0, acc1, Y, kb, c + 1, Q0, Q1);
        }
#pragma unroll
        for (int q = 0; q < NC; ++q) {
            Y[i0 * NC + q] = acc0[q];
            if (two) Y[i1 * NC + q] = acc1[q];
        }
    }
    }
}

// The same for a block of bs < 64 rows (the last one), one entry at a time.
template <int NC, bool kForward>
__device__ void panel_update_short(double* Y, const float* L, int r, int kb, int bs, int first, int end, int stride) {
    for (int i = first; i < end; i += stride) {
        double acc[NC];
#pragma unroll
        for (int q = 0; q < NC; ++q) acc[q] = Y[i * NC + q];
        for (int b = 0; b < bs; ++b) {
            const double l = (double)__ldg(kForward ? L + (size_t)i * r + kb + b : L + (size_t)(kb + b) * r + i);
            const double* yb = Y + (kb + b) * NC;
#pragma unroll
            for (int q = 0; q < NC; ++q) acc[q] = fma(-l, yb[q], acc[q]);
        }
#pragma unroll
        for (int q = 0; q < NC; ++q) Y[i * NC + q] = acc[q];
    }
}

// The 64-row diagonal block solved for the right-hand sides q0, q0 + 8, ...
// (CPW of them) by one warp: lanes own rows kb + lane and kb + lane + 32, and
// the columns' shuffle and FMA chains interleave, so one serial pass of 64
// steps serves CPW columns.  kForward: L y = c; else L^T x = y.
template <int NC, int CPW, bool kForward>
__device__ __forceinline__ void diag_solve(double* Y, const float* Ld, const double* rinv, int kb, int bs, int q0,
                                           int lane) {
    double y0[CPW], y1[CPW];
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
        const int q = q0 + 8 * c;
        y0[c] = (q < NC && lane < bs) ? Y[(kb + lane) * NC + q] : 0.0;
        y1[c] = (q < NC && lane + 32 < bs) ? Y[(kb + lane + 32) * NC + q] : 0.0;
    }
    for (int s = 0; s < bs; ++s) {
        const int i = kForward ? s : bs - 1 - s;
        const double ri = rinv[i];
        const float l0 = kForward ? Ld[lane * (kTB + 1) + i] : Ld[i * (kTB + 1) + lane];
        const float l1 = kForward ? Ld[(lane + 32) * (kTB + 1) + i] : Ld[i * (kTB + 1) + lane + 32];
        const bool u0 = kForward ? lane > i : lane < i, u1 = kForward ? lane + 32 > i : lane + 32 < i;
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
            const double own = (i < 32) ? y0[c] : y1[c];
            const double yi = __shfl_sync(0xffffffffu, own * ri, i & 31);
            if (lane == (i & 31)) {
                if (i < 32) y0[c] = yi;
                else y1[c] = yi;
            }
            if (u0) y0[c] -= (double)l0 * yi;
            if (u1) y1[c] -= (double)l1 * yi;
        }
    }
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
        const int q = q0 + 8 * c;
        if (q < NC && lane < bs) Y[(kb + lane) * NC + q] = y0[c];
        if (q < NC && lane + 32 < bs) Y[(kb + lane + 32) * NC + q] = y1[c];
    }
}

template <int NC, int ROWS>
__global__ void __launch_bounds__(kTrsmThreads) trsm_kernel(const float* __restrict__ Lg,
                                                           const int32_t* __restrict__ rank,
                                                           const double* __restrict__ Ct, float* W, int r, int dv,
                                                           int* status) {
    extern __shared__ double sm_d[];
    double* Y = sm_d;                                        // [r][NC]
    double* rinv = Y + (size_t)r * NC;                       // [kTB] 1 / L_ii of the diagonal block
    float* Ld = reinterpret_cast<float*>(rinv + kTB);        // [kTB][kTB + 1] diagonal block
    const int u = blockIdx.y;
    const int wcols = dv + 1;
    const int c0 = blockIdx.x * NC;
    const int nc = min(NC, wcols - c0);
    int k = rank[u];
    if (!in_bounds(k >= 0 && k <= r, status)) k = 0;
    const float* L = Lg + (size_t)u * r * r;
    const double* C = Ct + (size_t)u * wcols * r;
    float* Wu = W + (size_t)u * r * wcols;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool rows16 = (r & 3) == 0;  // rows of L start on 16-byte boundaries
    // right-hand sides per solving warp; more than 8 columns a block only for a single
    // diagonal block (r <= 64: no trailing panels, checked by the launcher)
    constexpr int kCpw = (NC + 7) / 8;
    static_assert(NC <= 8 || NC % 8 == 0, "columns split evenly over the 8 warps");

    for (int e = tid; e < NC * k; e += kTrsmThreads) {
        const int q = e / k, a = e - q * k;
        Y[a * NC + q] = q < nc ? C[(size_t)(c0 + q) * r + a] : 0.0;
    }

    // The diagonal block [kb, kb + bs) of L into shared memory, with 1 / L_ii.
    auto stage_diag = [&](int kb, int bs) {
        __syncthreads();
        for (int e = tid; e < kTB * kTB; e += kTrsmThreads) {
            const int i = e / kTB, j = e % kTB;
            Ld[i * (kTB + 1) + j] = (i < bs && j <= i) ? L[(size_t)(kb + i) * r + kb + j] : 0.f;
        }
        if (tid < kTB) rinv[tid] = tid < bs ? 1.0 / (double)L[(size_t)(kb + tid) * r + kb + tid] : 0.0;
        __syncthreads();
    };

    // ---- forward: L y = c
    for (int kb = 0; kb < k; kb += kTB) {
        const int bs = min(kTB, k - kb);
        stage_diag(kb, bs);
        if (warp < (NC < 8 ? NC : 8)) diag_solve<NC, kCpw, true>(Y, Ld, rinv, kb, bs, warp, lane);
        __syncthreads();
        // every later row i: Y_i -= L[i, kb .. kb + bs) Y[kb .. kb + bs)
        if constexpr (NC <= 8) {
            if (bs == kTB)
                panel_update<NC, true, ROWS>(Y, L, r, kb, kb + bs + tid, k, kTrsmThreads, rows16);
            else
                panel_update_short<NC, true>(Y, L, r, kb, bs, kb + bs + tid, k, kTrsmThreads);
        }
    }

    // ---- backward: L^T x = y
    for (int kb = (k - 1) / kTB * kTB; k > 0 && kb >= 0; kb -= kTB) {
        const int bs = min(kTB, k - kb);
        stage_diag(kb, bs);
        if (warp < (NC < 8 ? NC : 8)) diag_solve<NC, kCpw, false>(Y, Ld, rinv, kb, bs, warp, lane);
        __syncthreads();
        // every earlier row i: Y_i -= L[kb .. kb + bs, i]^T Y[kb .. kb + bs) (loads coalesced across i)
        if constexpr (NC <= 8) {
            if (bs == kTB)
                panel_update<NC, false, ROWS>(Y, L, r, kb, tid, kb, kTrsmThreads, false);
            else
                panel_update_short<NC, false>(Y, L, r, kb, bs, tid, kb, kTrsmThreads);
        }
    }
    __syncthreads();
    for (int e = tid; e < r * nc; e += kTrsmThreads) {
        const int a = e / nc, q = e - a * nc;
        Wu[(size_t)a * wcols + c0 + q] = a < k ? (float)Y[a * NC + q] : 0.f;
    }
}

// W = L^-T (L^-1 C1) for a coreset of at most 64 rows (one diagonal block),
// one block per unit and one thread per right-hand side: thread q substitutes
// column q row by row (L read from shared memory as a broadcast, the columns
// interleaved in shared memory so a warp's reads are contiguous), so no lane
// idles on a triangular mask and no shuffle chain serialises the columns.
constexpr int kSmallR = 64;
__global__ void trsm_small_kernel(const float* __restrict__ Lg, const int32_t* __restrict__ rank,
                                  const double* __restrict__ Ct, float* W, int r, int dv, int* status) {
    __shared__ float Ls[kSmallR][kSmallR + 1];
    __shared__ double rinv[kSmallR];
    extern __shared__ double Ys[];                          // [k][wcols]
    const int u = blockIdx.x, wcols = dv + 1, tid = threadIdx.x;
    int k = rank[u];
    if (!in_bounds(k >= 0 && k <= r && r <= kSmallR, status)) k = 0;
    const float* L = Lg + (size_t)u * r * r;
    const double* C = Ct + (size_t)u * wcols * r;
    for (int e = tid; e < k * k; e += blockDim.x) {
        const int i = e / k, j = e - i * k;
        Ls[i][j] = j <= i ? L[(size_t)i * r + j] : 0.f;
    }
    for (int i = tid; i < k; i += blockDim.x) rinv[i] = 1.0 / (double)L[(size_t)i * r + i];
    for (int e = tid; e < k * wcols; e += blockDim.x) {
        const int q = e / k, a = e - q * k;
        Ys[a * wcols + q] = C[(size_t)q * r + a];
    }
    __syncthreads();
    if (tid < wcols) {
        const int q = tid;
        // forward: L y = c
        for (int i = 0; i < k; ++i) {
            double a0 = Ys[i * wcols + q], a1 = 0.0;
            int j = 0;
            for (; j + 1 < i; j += 2) {
                a0 = fma(-(double)Ls[i][j], Ys[j * wcols + q], a0);
                a1 = fma(-(double)Ls[i][j + 1], Ys[(j + 1) * wcols + q], a1);
            }
            if (j < i) a0 = fma(-(double)Ls[i][j], Ys[j * wcols + q], a0);
            Ys[i * wcols + q] = (a0 + a1) * rinv[i];
        }
        // backward: L^T x = y
        for (int i = k - 1; i >= 0; --i) {
            double a0 = Ys[i * wcols + q], a1 = 0.0;
            int j = i + 1;
            for (; j + 1 < k; j += 2) {
                a0 = fma(-(double)Ls[j][i], Ys[j * wcols + q], a0);
                a1 = fma(-(double)Ls[j + 1][i], Ys[(j + 1) * wcols + q], a1);
            }
            if (j < k) a0 = fma(-(double)Ls[j][i], Ys[j * wcols + q], a0);
            Ys[i * wcols + q] = (a0 + a1) * rinv[i];
        }
    }
    __syncthreads();
    float* Wu = W + (size_t)u * r * wcols;
    for (int e = tid; e < r * wcols; e += blockDim.x) {
        const int a = e / wcols;
        Wu[e] = a < k ? (float)Ys[e] : 0.f;
    }
}

template <int NC>
size_t trsm_smem(int r) {
    return sizeof(double) * (NC * (size_t)r + kTB) + sizeof(float) * kTB * (kTB + 1);
}

template <int NC>
wc_status launch_trsm_t(const Shape& s, const float* Lg, const int32_t* rank, const double* Ct, float* W,
                        int* status, cudaStream_t st) {
    const size_t smem = trsm_smem<NC>(s.r);
    // two rows per thread where the panels are long (they hold 512 rows on average from r = 1024)
    auto kern = s.r >= 1024 ? trsm_kernel<NC, 2> : trsm_kernel<NC, 1>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return WC_ERR_CUDA;
    kern<<<dim3((s.dv + 1 + NC - 1) / NC, s.units), kTrsmThreads, smem, st>>>(Lg, rank, Ct, W, s.r, s.dv, status);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace

wc_status launch_gather(const Shape& s, const void* K, const int32_t* piv, const float* F, const int32_t* rank,
                        void* Ks, char* ws, cudaStream_t st) {
    const WsLayout L = make_layout(s);
    float* Lg = reinterpret_cast<float*>(ws + L.lg);
    int* status = reinterpret_cast<int*>(ws + L.status);
    // a row's copies take max(d, r) elements: give it that many threads (whole warps, at most
    // 256) and put several short rows in a block (many tiny blocks leave the GPU's block
    // scheduler the bottleneck)
    const int w = s.d > s.r ? s.d : s.r;
    const int tpr = w >= 256 ? 256 : (w + 31) / 32 * 32;
    const int rpb = 256 / tpr;
    dim3 grid((s.r + rpb - 1) / rpb, s.units);
    if (s.dtype == WC_BF16)
        gather_kernel<__nv_bfloat16><<<grid, rpb * tpr, 0, st>>>(static_cast<const __nv_bfloat16*>(K), piv, F, rank,
                                                                 static_cast<__nv_bfloat16*>(Ks), Lg, s.n, s.d, s.r,
                                                                 s.ldf, s.bins, tpr, status);
    else
        gather_kernel<float><<<grid, rpb * tpr, 0, st>>>(static_cast<const float*>(K), piv, F, rank,
                                                         static_cast<float*>(Ks), Lg, s.n, s.d, s.r, s.ldf, s.bins,
                                                         tpr, status);
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
    e.status = reinterpret_cast<int*>(ws + L.status);
    e.out = ws + L.c1part;
    e.d = s.d; e.dv = s.dv; e.r = s.r;
    e.nsplit = s.nsplit; e.split_len = split_keys(s.n, s.units, s.r);
    e.beta = (float)s.beta;
    e.group = 1; e.hq = s.hkv;
    e.mode = kExpmmPartial;
    if (s.center) {
        e.bias = reinterpret_cast<const float*>(ws + L.bias);
        e.bias_stride = center_bias_stride(s);
    }
    return launch_expmm_simt(e, s.dtype, s.units, st);
}

wc_status launch_solve(const Shape& s, const int32_t* piv, const int32_t* rank, float* W, char* ws,
                       cudaStream_t st) {
    const WsLayout L = make_layout(s);
    double* Ct = reinterpret_cast<double*>(ws + L.y);
    int* status = reinterpret_cast<int*>(ws + L.status);
    // a warp per coreset row, 8 rows a block
    merge_c1_kernel<<<dim3((s.r + 7) / 8, s.units), 256, 0, st>>>(
        reinterpret_cast<const float*>(ws + L.c1part), rank, Ct, s.nsplit, s.r, s.dv, piv,
        s.center ? reinterpret_cast<const double*>(ws + L.cdot) : nullptr,
        s.center ? reinterpret_cast<const double*>(ws + L.kk) : nullptr, s.bins, s.n_all, s.beta,
        reinterpret_cast<const double*>(ws + L.shift), 32, status);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
    // right-hand sides per block: 8 (the fewest re-reads of L, and each block
    // repeats the serial diagonal solves), fewer only while the blocks would
    // fill less than half of the GPU (one block per SM with two rows per
    // thread, two with one), within the shared memory that holds the columns
    // for this r
    const float* Lg = reinterpret_cast<const float*>(ws + L.lg);
    constexpr size_t kMax = 232448;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    auto smem_ok = [&](int nc) {
        return (nc == 8 ? trsm_smem<8>(s.r) : nc == 4 ? trsm_smem<4>(s.r) : nc == 2 ? trsm_smem<2>(s.r)
                                                                                  : trsm_smem<1>(s.r)) <= kMax;
    };
    int best = 0;
    for (int nc : {8, 4, 2, 1}) {
        if (!smem_ok(nc)) continue;
        best = nc;
        if ((long)s.units * ((s.dv + nc) / nc) * 2 >= (long)nsm * (s.r >= 1024 ? 1 : 2)) break;
    }
    // a single diagonal block (r <= 64): one block per unit, one thread per right-hand side
    if (s.r <= kSmallR) {
        const size_t smem = sizeof(double) * (size_t)s.r * (s.dv + 1);   // 132 KB at most (r = 64, dv = 256)
        if (cudaFuncSetAttribute(trsm_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return WC_ERR_CUDA;
        trsm_small_kernel<<<s.units, (s.dv + 1 + 31) / 32 * 32, smem, st>>>(Lg, rank, Ct, W, s.r, s.dv, status);
        return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
    }
    if (best == 8) return launch_trsm_t<8>(s, Lg, rank, Ct, W, status, st);
    if (best == 4) return launch_trsm_t<4>(s, Lg, rank, Ct, W, status, st);
    if (best == 2) return launch_trsm_t<2>(s, Lg, rank, Ct, W, status, st);
    if (best == 1) return launch_trsm_t<1>(s, Lg, rank, Ct, W, status, st);
    return WC_ERR_UNSUPPORTED;
}

}  // namespace wc

// center.cu — key statistics: centring and the factor's shift.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gist.science
// technical summary, "Methodik" item 3): softmax attention is invariant to a
// global centring of the keys, K <- K - kbar, and the method centres them.
// Per caller unit u (all n keys, bins included):
//   kbar_u   = (1/n) sum_i k_i                 fp64, two fixed-order passes
//   kk_u     = |kbar_u|^2                       fp64
//   c_i      = <k_i, kbar_u>                    fp64, every key
//   bias_i   = -beta log2(e) c_i                fp32, per bin unit, rows padded to
//                                               a multiple of 128 (zeros beyond)
// The centred kernel then factors as
//   exp(beta <k_s - kbar, k_j - kbar>) = exp(beta <k_s, k_j>) * 2^bias_j * exp(beta (kk - c_s)),
// so the C1 GEMM keeps the keys as given (a per-key logit bias, a per-row factor
// in the fp64 merge) and the selection streams centred fp32 keys.
#include "wc_common.cuh"
#include "wc_internal.h"

namespace wc {
namespace {

// Column sums of K over chunks of kCenterChunk keys: part[u][chunk][c].
template <typename T>
__global__ void key_sum_kernel(const T* __restrict__ K, double* part, int n, int d, int nchunk) {
    const int chunk = blockIdx.x, u = blockIdx.y;
    const int i0 = chunk * kCenterChunk, i1 = min(n, i0 + kCenterChunk);
    const T* Ku = K + (size_t)u * n * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        double acc = 0.0;
        for (int i = i0; i < i1; ++i) acc += (double)to_f32(Ku[(size_t)i * d + c]);
        part[((size_t)u * nchunk + chunk) * d + c] = acc;
    }
}

// kbar[u][c] = sum over chunks (in order) / n; kk[u] = |kbar|^2 (one block per unit).
__global__ void key_mean_kernel(const double* __restrict__ part, double* kbar, double* kk, int n, int d,
                                int nchunk) {
    const int u = blockIdx.x;
    __shared__ double sq[256];
    double mine = 0.0;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        double acc = 0.0;
        for (int ch = 0; ch < nchunk; ++ch) acc += part[((size_t)u * nchunk + ch) * d + c];
        const double m = acc / (double)n;
        kbar[(size_t)u * d + c] = m;
        mine += m * m;
    }
    sq[threadIdx.x] = mine;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int k = 0; k < (int)blockDim.x; ++k) t += sq[k];
        kk[u] = t;
    }
}

// c_i = <k_i, kbar> and the per-bin padded bias; one thread per key.
template <typename T>
__global__ void key_dot_mean_kernel(const T* __restrict__ K, const double* __restrict__ kbar, double* cdot,
                                    float* bias, int n, int d, int bins, int nb_pad, double beta_log2e) {
    const int u = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int nb = n / bins;
    if (i >= bins * nb_pad) return;
    const int b = i / nb_pad, il = i - b * nb_pad;  // bin and key within the padded bin row
    float* brow = bias + ((size_t)u * bins + b) * nb_pad;
    if (il >= nb) {
        brow[il] = 0.f;
        return;
    }
    const int key = b * nb + il;
    const T* k = K + ((size_t)u * n + key) * d;
    const double* m = kbar + (size_t)u * d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += (double)to_f32(k[c]) * m[c];
    cdot[(size_t)u * n + key] = acc;
    brow[il] = (float)(-beta_log2e * acc);
}

template <typename T>
wc_status launch_center_t(const Shape& s, const void* K, char* ws, cudaStream_t st) {
    const WsLayout L = make_layout(s);
    const int U = s.units_all, n = s.n_all, d = s.d;
    const int nchunk = (n + kCenterChunk - 1) / kCenterChunk;
    double* part = reinterpret_cast<double*>(ws + L.kpart);
    double* kbar = reinterpret_cast<double*>(ws + L.kbar);
    double* kk = reinterpret_cast<double*>(ws + L.kk);
    key_sum_kernel<T><<<dim3(nchunk, U), 128, 0, st>>>(static_cast<const T*>(K), part, n, d, nchunk);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
    key_mean_kernel<<<U, 256, 0, st>>>(part, kbar, kk, n, d, nchunk);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
    const int nb_pad = center_bias_stride(s);
    const int total = s.bins * nb_pad;
    key_dot_mean_kernel<T><<<dim3((total + 255) / 256, U), 256, 0, st>>>(
        static_cast<const T*>(K), kbar, reinterpret_cast<double*>(ws + L.cdot), reinterpret_cast<float*>(ws + L.bias),
        n, d, s.bins, nb_pad, s.beta * 1.4426950408889634);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

// M[u'] = max over bin unit u''s keys of beta |k_i|^2 (k_i - kbar when centred),
// in fp64.  A warp takes kShiftKeys keys at a time, lane l summing dimensions
// l, l + 32, ... of each (coalesced loads, all of them issued before the sums
// when the head width DT is a compile-time constant), then a fixed shuffle tree
// adds the lanes, so the result is deterministic; it may differ from the
// selection's own sum in the last bits, which scales W by 1 + O(1e-16 M) (the
// row normalisation cancels it).  The warp maxima meet in an atomic maximum on
// the bits (non-negative doubles order like their bits; a maximum is exact).
constexpr int kShiftBlocks = 2048;  // about two waves of 256-thread blocks on 148 SMs
constexpr int kShiftKeys = 4;

template <typename T, int DT>
__global__ void key_shift_kernel(const T* __restrict__ K, const double* __restrict__ kbar,
                                 unsigned long long* shift_bits, int n, int d_rt, int bins, double beta) {
    const int d = DT ? DT : d_rt;
    const int ub = blockIdx.y;               // bin unit: caller unit ub / bins, bin ub % bins
    const int nb = n / bins;
    const T* Kb = K + (size_t)ub * nb * d;   // the bin's keys are contiguous
    const double* m = kbar ? kbar + (size_t)(ub / bins) * d : nullptr;
    const int lane = threadIdx.x & 31, warps = blockDim.x >> 5;
    const int gw = blockIdx.x * warps + (int)(threadIdx.x >> 5), nw = gridDim.x * warps;
    double mx = 0.0;
    for (int i0 = gw * kShiftKeys; i0 < nb; i0 += nw * kShiftKeys) {
        double ss[kShiftKeys];
#pragma unroll
        for (int q = 0; q < kShiftKeys; ++q) {
            ss[q] = 0.0;
            if (i0 + q < nb) {
                const T* k = Kb + (size_t)(i0 + q) * d;
#pragma unroll
                for (int c = lane; c < d; c += 32) {
                    double x = (double)to_f32(k[c]);
                    if (m) x -= m[c];
                    ss[q] += x * x;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kShiftKeys; ++q) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss[q] += __shfl_xor_sync(0xffffffffu, ss[q], o);
            mx = fmax(mx, beta * ss[q]);
        }
    }
    if (lane == 0 && mx > 0.0) atomicMax(shift_bits + ub, (unsigned long long)__double_as_longlong(mx));
}

template <typename T>
wc_status launch_key_shift_t(const Shape& s, const void* K, char* ws, cudaStream_t st) {
    const WsLayout L = make_layout(s);
    const double* kbar = s.center ? reinterpret_cast<const double*>(ws + L.kbar) : nullptr;
    const int ub = s.units_all * s.bins, nb = s.n_all / s.bins;
    if (cudaMemsetAsync(ws + L.shift, 0, sizeof(double) * ub, st) != cudaSuccess) return WC_ERR_CUDA;
    const int per_bin = (kShiftBlocks + ub - 1) / ub, need = (nb + 8 * kShiftKeys - 1) / (8 * kShiftKeys);
    const dim3 grid(per_bin < need ? per_bin : need, ub);
    const T* Kt = static_cast<const T*>(K);
    auto* bits = reinterpret_cast<unsigned long long*>(ws + L.shift);
    if (s.d == 128)
        key_shift_kernel<T, 128><<<grid, 256, 0, st>>>(Kt, kbar, bits, s.n_all, s.d, s.bins, s.beta);
    else if (s.d == 64)
        key_shift_kernel<T, 64><<<grid, 256, 0, st>>>(Kt, kbar, bits, s.n_all, s.d, s.bins, s.beta);
    else
        key_shift_kernel<T, 0><<<grid, 256, 0, st>>>(Kt, kbar, bits, s.n_all, s.d, s.bins, s.beta);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace

int center_bias_stride(const Shape& s) { return (s.n_all / s.bins + 127) / 128 * 128; }

wc_status launch_key_shift(const Shape& s, const void* K, char* ws, cudaStream_t st) {
    if (s.dtype == WC_BF16) return launch_key_shift_t<__nv_bfloat16>(s, K, ws, st);
    return launch_key_shift_t<float>(s, K, ws, st);
}

wc_status launch_center(const Shape& s, const void* K, char* ws, cudaStream_t st) {
    if (s.dtype == WC_BF16) return launch_center_t<__nv_bfloat16>(s, K, ws, st);
    return launch_center_t<float>(s, K, ws, st);
}

}  // namespace wc

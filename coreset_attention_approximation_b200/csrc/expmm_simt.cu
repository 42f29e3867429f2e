// expmm_simt.cu — CUDA-core exp-GEMM with a running row maximum.
//
// Serves the fp32 workloads (whose 1e-5 tolerance tensor cores cannot meet)
// and any shape the tensor-core kernel does not take.  fp32 arithmetic,
// 32 x 32 tiles, 256 threads: thread (row = t / 8, sub = t % 8) owns logits
// (row, sub + 8k), k < 4, and output columns sub + 8q.
#include <math.h>

#include "wc_common.cuh"
#include "wc_expmm.cuh"

namespace wc {
namespace {

constexpr int BM = 32, BN = 32, kThreads = 256, kMaxQ = 32;

template <typename T, typename TC, int MODE>
__global__ void __launch_bounds__(kThreads) expmm_simt_kernel(const ExpmmArgs e) {
    extern __shared__ float sm[];
    const int d = e.d, dv = e.dv, lda = d + 1;
    float* As = sm;
    float* Bs = As + BM * lda;
    float* Cs = Bs + BN * lda;
    float* Ps = Cs + BN * dv;
    float* Ws = Ps + BM * (BN + 1);

    const int z = blockIdx.z;
    int unit, a_valid, b_lo, b_hi, split = 0;
    if (MODE == kExpmmPartial) {
        unit = z;
        a_valid = e.rank[unit];
        if (!in_bounds(a_valid >= 0 && a_valid <= e.r, e.status)) return;
        split = blockIdx.y;
        b_lo = split * e.split_len;
        b_hi = min(e.b_rows, b_lo + e.split_len);
    } else {
        const int hkv = e.hq / e.group;
        unit = (z / e.hq) * hkv + (z % e.hq) / e.group;
        a_valid = e.a_rows;
        b_lo = 0;
        b_hi = e.all_keys ? e.b_rows : e.rank[unit];
        if (!in_bounds(b_hi >= 0 && b_hi <= e.b_rows, e.status)) return;
    }
    const int a0 = blockIdx.x * BM;
    if (a0 >= a_valid) return;

    const T* A = static_cast<const T*>(e.A) + (size_t)z * e.a_stride;
    const T* B = static_cast<const T*>(e.B) + (size_t)unit * e.b_stride;
    const TC* C = static_cast<const TC*>(e.C) + (size_t)unit * e.c_stride;
    const float* wcol = e.wcol ? e.wcol + (size_t)unit * e.c_stride : nullptr;
    const float* bias = e.bias ? e.bias + (size_t)unit * e.bias_stride : nullptr;

    const int tid = threadIdx.x, row = tid / 8, sub = tid % 8;
    for (int x = tid; x < BM * d; x += kThreads) {
        const int i = x / d, c = x % d;
        As[i * lda + c] = (a0 + i < a_valid) ? to_f32(A[(size_t)(a0 + i) * d + c]) : 0.f;
    }

    float o[kMaxQ];
#pragma unroll
    for (int q = 0; q < kMaxQ; ++q) o[q] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int nq = dv / 8;

    for (int b0 = b_lo; b0 < b_hi; b0 += BN) {
        __syncthreads();
        for (int x = tid; x < BN * d; x += kThreads) {
            const int jj = x / d, c = x % d;
            Bs[jj * lda + c] = (b0 + jj < b_hi) ? to_f32(B[(size_t)(b0 + jj) * d + c]) : 0.f;
        }
        for (int x = tid; x < BN * dv; x += kThreads) {
            const int jj = x / dv, c = x % dv;
            Cs[jj * dv + c] = (b0 + jj < b_hi) ? to_f32(C[(size_t)(b0 + jj) * e.ldc + c]) : 0.f;
        }
        if (tid < BN) Ws[tid] = (b0 + tid < b_hi) ? (wcol ? wcol[(size_t)(b0 + tid) * e.ldc] : 1.f) : 0.f;
        __syncthreads();

        float sk[4];
        float mt = -INFINITY;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int jj = sub + 8 * k;
            float acc = 0.f;
            for (int c = 0; c < d; ++c) acc = fmaf(As[row * lda + c], Bs[jj * lda + c], acc);
            const float bj = (bias && b0 + jj < b_hi) ? bias[b0 + jj] * 0.6931471805599453f : 0.f;
            sk[k] = (b0 + jj < b_hi) ? fmaf(acc, e.beta, bj) : -INFINITY;
            mt = fmaxf(mt, sk[k]);
        }
#pragma unroll
        for (int o2 = 1; o2 < 8; o2 <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o2));
        const float m_new = fmaxf(m_run, mt);
        const float corr = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
        float lp = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int jj = sub + 8 * k;
            const float p = (sk[k] == -INFINITY) ? 0.f : expf(sk[k] - m_new);
            Ps[row * (BN + 1) + jj] = p;
            lp = fmaf(p, Ws[jj], lp);
        }
        l_run = l_run * corr + lp;
        m_run = m_new;
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kMaxQ; ++q) {
            if (q < nq) {
                const int col = sub + 8 * q;
                float acc = o[q] * corr;
                for (int jj = 0; jj < BN; ++jj) acc = fmaf(Ps[row * (BN + 1) + jj], Cs[jj * dv + col], acc);
                o[q] = acc;
            }
        }
    }
#pragma unroll
    for (int o2 = 1; o2 < 8; o2 <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, o2);

    const int a = a0 + row;
    if (a >= a_valid) return;
    if (MODE == kExpmmPartial) {
        float* out = static_cast<float*>(e.out) + (((size_t)unit * e.nsplit + split) * e.r + a) * c1_row(dv);
#pragma unroll
        for (int q = 0; q < kMaxQ; ++q)
            if (q < nq) out[sub + 8 * q] = o[q];
        if (sub == 0) {
            out[dv] = l_run;
            out[dv + 1] = m_run;
        }
    } else {
        float* out = static_cast<float*>(e.out) + ((size_t)z * e.a_rows + a) * dv;
#pragma unroll
        for (int q = 0; q < kMaxQ; ++q)
            if (q < nq) out[sub + 8 * q] = o[q] / l_run;
    }
}

template <typename T, typename TC, int MODE>
wc_status launch_t(const ExpmmArgs& e, int heads, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)(BM + BN) * (e.d + 1) + (size_t)BN * e.dv + BM * (BN + 1) + BN);
    auto kern = expmm_simt_kernel<T, TC, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return WC_ERR_CUDA;
    const int ysplit = MODE == kExpmmPartial ? e.nsplit : 1;
    dim3 grid((e.a_rows + BM - 1) / BM, ysplit, heads);
    kern<<<grid, kThreads, smem, st>>>(e);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // namespace

wc_status launch_expmm_simt(const ExpmmArgs& e, int dtype, int heads, cudaStream_t st) {
    if (e.dv % 8 != 0 || e.dv / 8 > kMaxQ) return WC_ERR_UNSUPPORTED;
    if (e.mode == kExpmmPartial) {
        if (dtype == WC_BF16) return launch_t<__nv_bfloat16, __nv_bfloat16, kExpmmPartial>(e, heads, st);
        return launch_t<float, float, kExpmmPartial>(e, heads, st);
    }
    if (dtype == WC_BF16) return launch_t<__nv_bfloat16, float, kExpmmRownorm>(e, heads, st);
    return launch_t<float, float, kExpmmRownorm>(e, heads, st);
}

}  // namespace wc

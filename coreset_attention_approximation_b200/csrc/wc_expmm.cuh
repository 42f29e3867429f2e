// wc_expmm.cuh — the exp-GEMM that both dense contractions of WildCat share:
//   O[a, :] = sum_b exp(beta <A_a, B_b> - m_a) C[b, :],  l_a = sum_b exp(...) w_b
// with a running row maximum m_a (rescaled as it grows).
//   weights: A = K_S, B = K, C = V, w = 1  -> partial (O, l, m) per key split
//   attend:  A = Q,  B = K_S, C = W[:, :dv], w = W[:, dv] -> out = O / l
#pragma once

#include "wc_internal.h"

namespace wc {

enum { kExpmmPartial = 0, kExpmmRownorm = 1 };

struct ExpmmArgs {
    const void* A;  int64_t a_stride; int a_rows;   // rows of A per head (coreset rows or queries)
    const void* B;  int64_t b_stride; int b_rows;   // rows of B per unit (keys or coreset rows)
    const void* C;  int64_t c_stride; int ldc;      // value rows (dtype, or fp32 W)
    const float* wcol;                              // rownorm: W[:, dv] with row stride ldc
    const int32_t* rank;                            // valid coreset rows per unit
    int* status;                                    // device status word (bounds checks of rank)
    int all_keys;                                   // rownorm: every one of the b_rows rows counts
    const float* bias;                              // partial: per-key logit bias (log2 units) or null
    int bias_stride;                                // floats per unit of bias
    void* out;
    int d, dv, r;
    int nsplit, split_len;
    float beta;
    int group;  // query heads per kv head (rownorm)
    int hq;     // query heads per batch (rownorm); kv heads per batch (partial)
    int mode;
};

wc_status launch_expmm_simt(const ExpmmArgs& e, int dtype, int heads, cudaStream_t st);

}  // namespace wc

// attend.cu — coreset attention.
//
// Method: WildCat: Near-Linear Attention in Theory and Practice (gptget.net
// page, Abstract): attend over only the small weighted coreset.
//   A = exp(beta Q K_S^T) W   (first rank[u] coreset rows),  out = A[:, :dv] / A[:, dv]
// Query head g of batch b reads kv unit b * Hkv + g / (Hq / Hkv).
#include "wc_common.cuh"
#include "wc_expmm.cuh"
#include "wc_internal.h"

namespace wc {

wc_status launch_attend(const Shape& s, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                        float* out, char* ws, cudaStream_t st) {
    if (tc_supported(s)) return launch_attend_tc(s, Q, Ks, W, rank, out, ws, st);
    ExpmmArgs e{};
    e.A = Q; e.a_stride = (int64_t)s.nq * s.d; e.a_rows = s.nq;
    e.B = Ks; e.b_stride = (int64_t)s.r * s.d; e.b_rows = s.r;
    e.C = W; e.c_stride = (int64_t)s.r * (s.dv + 1); e.ldc = s.dv + 1;
    e.wcol = W + s.dv;
    e.rank = rank;
    e.status = ws ? reinterpret_cast<int*>(ws + make_layout(s).status) : nullptr;
    e.all_keys = s.bins > 1;  // bins: padded rows carry zero weights, every row of the union counts
    e.out = out;
    e.d = s.d; e.dv = s.dv; e.r = s.r;
    e.nsplit = 1; e.split_len = s.r;
    e.beta = (float)s.beta;
    e.group = s.hq / s.hkv; e.hq = s.hq;
    e.mode = kExpmmRownorm;
    return launch_expmm_simt(e, s.dtype, s.batch * s.hq, st);
}

}  // namespace wc

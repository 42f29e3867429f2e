// wc_internal.h — workspace layout and kernel launchers of the WildCat library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/wildcat.h"

namespace wc {

constexpr int kMaxBlocksPerUnit = 512;   // select: thread blocks that share one unit
constexpr int kSplitKeys = 4096;         // weights: keys per partial sum of C1 (at least, for long heads)
// Keys per partial sum of C1 for units of n keys and r coreset rows: for long
// heads kSplitKeys, doubled while the grid keeps at least 8 waves of blocks
// (a block's fixed costs, start-up and the store of its partial sums, then
// weigh less); for heads of at most kSplitKeys keys whose row tiles leave SMs
// idle, up to 4 splits of whole 128-key tiles (so a few short heads still
// spread over the GPU, while many short heads keep one block each).
inline int split_keys(int n, int units, int r) {
    if (n > kSplitKeys) {
        const long row_tiles = (long)units * ((r + 127) / 128);
        int len = kSplitKeys;
        while (2L * len < n && row_tiles * ((n + 2L * len - 1) / (2L * len)) >= 8L * 148) len *= 2;
        return len;
    }
    const long tiles = (long)units * ((r + 127) / 128);
    int want = tiles >= 148 ? 1 : (int)((148 + tiles - 1) / tiles);
    if (want > 4) want = 4;
    const int q = ((n + want - 1) / want + 127) / 128 * 128;
    return q < 128 ? 128 : q;
}
constexpr int kCenterChunk = 1024;       // centring: keys per partial column sum
constexpr int kAttendFill = 148;         // attention: blocks resident at once (one per SM of a B200)
// Row of a C1 partial sum: O[0 .. dv), l, m, two unused floats (rows 16-byte aligned).
constexpr int c1_row(int dv) { return dv + 4; }
constexpr int kWsAlign = 256;

// One per unit, in the workspace; zeroed before every select launch.
struct UnitSync {
    uint32_t bar;                 // barrier arrivals (monotonic within a launch)
    uint32_t pivflag;             // j + 1 once the pivot of step j is published
    int32_t s;                    // published pivot
    int32_t stop;                 // 1 when the run ends at the published step
    double d_s;                   // residual diagonal at the published pivot
    unsigned long long hmax_bits; // M = max_i beta |k_i|^2 (bits of a non-negative double)
    uint32_t pad[8];
};
static_assert(sizeof(UnitSync) == 64, "UnitSync is 64 bytes");

// Byte offsets into the workspace (all kWsAlign-aligned).
struct WsLayout {
    size_t status;    // int32 first device error
    size_t sync;      // UnitSync[units]
    size_t partials;  // double[units][2][kMaxBlocksPerUnit]
    size_t kt;        // dtype[units][d][ldf]   transposed keys
    size_t lg;        // float[units][r][r]     gathered L = F[piv, :]
    size_t c1part;    // float[units][nsplit][r][c1_row(dv)]  (O | l | m | unused)
    size_t y;         // double[units][dv + 1][r]  C1, column-major, solved in place
    size_t v16;       // half[units][n][dv]     values for the tensor-core weights GEMM
    size_t w16;       // half[units][r][dv]     column-scaled weights for attention
    size_t sigma;     // float[units][dv]       their column scales
    size_t wn;        // float[units][r_pad]    normaliser column W[:, dv], zero from rank to r_pad
    // centring (sizes 0 unless shape.center): per caller unit
    size_t kpart;     // double[units][n / kCenterChunk][d]  partial column sums
    size_t kbar;      // double[units][d]       mean key
    size_t kk;        // double[units]          |mean|^2
    size_t cdot;      // double[units][n]       <k_i, mean>
    size_t bias;      // float[units * bins][stride]  -beta log2(e) <k_i, mean> per bin, padded
    size_t shift;     // double[units * bins]   M = max_i beta |k_i|^2 per bin unit (the factor's shift)
    size_t apart;     // float[B * hq][splits][nq][c1_row(dv)]  key-split attention rows (few queries only)
    size_t scratch_end;
    // room for outputs that wc_forward keeps in the workspace when not given
    size_t piv, rank, f, ks, w;
    size_t forward_end;
};

struct Shape {
    int32_t batch, hq, hkv, n, nq, d, dv, r;
    int32_t dtype;         // wc_dtype
    double beta, eps;
    uint64_t seed;
    uint64_t timeout_ns;
    int64_t ldf;
    int32_t units;         // batch * hkv
    int32_t esize;         // bytes per Q/K/V element
    int32_t nsplit;        // C1 partial sums
    int32_t r_pad;         // r rounded up to 128 (whole key tiles of the attention's normaliser column)
    int32_t bins;          // key bins per unit (1: none); select and weights run on the bin view
    int32_t center;        // subtract each unit's mean key before the selection and the weights
    int32_t unit_base;     // Philox unit index of the caller's first unit (0 for a whole problem)
    // the caller's problem, the same in the unit view and the bin view (sizes the workspace)
    int32_t units_all, n_all, r_all;
};

wc_status make_shape(const wc_shape* in, Shape* out);
// The per-bin problem: units * bins units of n / bins keys and r / bins pivots.
Shape bin_view(const Shape& s);
WsLayout make_layout(const Shape& s);

// Kernel launchers (each returns WC_OK or WC_ERR_CUDA / WC_ERR_UNSUPPORTED).
wc_status launch_read_probe(const void* buf, int64_t bytes, uint32_t* sink, cudaStream_t st);
wc_status launch_select(const Shape& s, const void* K, int32_t* piv, float* F, int32_t* rank,
                        char* ws, cudaStream_t st);
wc_status launch_gather(const Shape& s, const void* K, const int32_t* piv, const float* F,
                        const int32_t* rank, void* Ks, char* ws, cudaStream_t st);
wc_status launch_coreset_values(const Shape& s, const void* Ks, const void* K, const void* V,
                                const int32_t* rank, char* ws, cudaStream_t st);
wc_status launch_solve(const Shape& s, const int32_t* piv, const int32_t* rank, float* W, char* ws,
                       cudaStream_t st);
// Centring statistics of every caller unit (mean key, |mean|^2, <k_i, mean>,
// the per-bin logit bias); `s` may be either view.
wc_status launch_center(const Shape& s, const void* K, char* ws, cudaStream_t st);
int center_bias_stride(const Shape& s);  // floats per bin row of the bias
// M = max_i beta |k_i|^2 of every bin unit (centred keys when s.center), as the
// selection computes it; the weights step divides the shift back out.
wc_status launch_key_shift(const Shape& s, const void* K, char* ws, cudaStream_t st);
wc_status launch_attend(const Shape& s, const void* Q, const void* Ks, const float* W,
                        const int32_t* rank, float* out, char* ws, cudaStream_t st);
wc_status launch_wait_selftest(char* ws, uint64_t timeout_ns, cudaStream_t st);
// 2^x over an array: method 0 as the exp-GEMM's FMA-pipe polynomial, 1 on the exponential unit.
wc_status launch_exp2_selftest(const float* x, float* y, int64_t n, int method, cudaStream_t st);

// Tensor-core path (bf16 inputs, d and dv in {64, 128}).
bool tc_supported(const Shape& s);
// tensor-core attention: splits of the coreset when few query tiles would leave
// SMs idle (1 = none), and the floats of their partial rows in the workspace
int attend_splits(const Shape& s);
size_t attend_split_floats(const Shape& s);
wc_status launch_coreset_values_tc(const Shape& s, const void* Ks, const void* K, const void* V,
                                   const int32_t* rank, char* ws, cudaStream_t st);
wc_status launch_attend_tc(const Shape& s, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                           float* out, char* ws, cudaStream_t st);
wc_status launch_attend_tc_at(const Shape& s, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                              float* out, int* status, __half* W16, float* sigma, float* wn, cudaStream_t st);

}  // namespace wc

// expmm_tc.cu — tensor-core (tcgen05 / TMEM / TMA) exp-GEMM of WildCat.
//
// For a tile of 128 rows a of A (coreset keys for the weights, queries for
// attention) and the keys b of B in [b_lo, b_hi):
//   S = A B^T                    bf16 x bf16 -> fp32 in TMEM (tcgen05.mma)
//   P = 2^(S beta log2(e) - m)   fp16, in the softmax warps (running max m,
//                                rescaled only when it grows by more than 2^8)
//   O += P C                     fp16 x fp16 -> fp32 in TMEM (tcgen05.mma)
//   l += sum_b P w_b             fp32, in the softmax warps
// C = fp16 values (V, or the weights W scaled per column); w = 1 or the
// normaliser column W[:, dv].  Weights: the (O, l, m) of each key split are
// written for the solve (with centred keys a per-key logit bias is added to S);
// attention: out = O sigma / l, or, when the query tiles are too few to fill
// the GPU, (O sigma, l, m) per split of the coreset, combined by
// attend_combine_kernel.  The weight preparation (fp16 W, sigma, w) runs as
// clusters of 8 blocks whose column maxima meet in distributed shared memory.
//
// Warp roles (384 threads): warp 0 loads A once and then the key tiles, warp 1
// the value tiles (TMA, 3-stage rings); warp 2 owns TMEM and issues S = A B^T,
// warp 3 issues O += P C; warps 4..11 run the exponentials and the epilogue.
// A softmax warp w reads TMEM lanes 32 (w % 4) .. +31 (one tile row per
// thread) and takes every other key tile (parity (w - 4) / 4), so the two
// warps on an SM sub-partition alternate: one loads S and finds its row
// maxima while the other runs its exponentials.  They share one reference
// maximum per row (the shift of O), handed from tile to tile through shared
// memory at named barriers; O is rescaled only when the reference grows by
// more than 2^8.  S is triple buffered in TMEM (3 x 128 columns), O takes
// the remaining DV columns.  Operands use the 128-byte
// swizzled canonical layouts: A, B and P K-major, C MN-major.  Every wait is
// bounded; a wait that runs out records WC_ERR_TIMEOUT and the block winds
// down (drains its copies and MMAs, frees TMEM) instead of hanging.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "wc_common.cuh"
#include "wc_exp2.cuh"
#include "wc_expmm.cuh"
#include "wc_internal.h"
#include "wc_tc.cuh"

namespace wc {
namespace {

using namespace tc;

constexpr int BM = 128;              // rows per CTA (one TMEM lane per row)
constexpr int TILES = 1;             // row tiles per CTA
constexpr int BN = 128;              // keys per stage
constexpr int NB = 3;                // key-tile stages: released once S is computed
constexpr int NC = 3;                // value-tile stages: released once PV is computed
// warps: 0 key loader, 1 value loader, 2 S issuer, 3 PV issuer, 4..11 softmax
constexpr int kThreads = 384;
constexpr int NS = 3;                // S / P buffers in TMEM
// Register split (setmaxnreg): the block is launched with kRegsLaunch per
// thread; warps 0..3 drop to kRegsSide and warps 4..11 rise to kRegsSoftmax,
// which together use exactly the launch's registers (checked on the host).
constexpr int kRegsLaunch = 168;
constexpr int kRegsSide = 56;
constexpr int kRegsSoftmax = 224;
static_assert(128 * kRegsSide + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 units: P stays below 2^8 between rescales
constexpr uint64_t kTcTimeoutNs = 4000000000ull;
// Exponentials moved off the exponential unit: of each row's 128 key columns,
// kFmaExpCols run as exp2_fma2 on the FMA / ALU pipes (wc_exp2.cuh), the rest
// as ex2.approx on the exponential unit; placed at the row's last columns
// (kFmaExpSpread = 0) or at the last kFmaExpCols / 4 columns of every
// 32-column quarter (1).  Measured on the B200 with 0, 16, 32 and 48 columns
// in both placements: no split was faster than none (each 128-key tile is
// bound by shared-memory bandwidth, not by the exponential unit), so none is
// the default.
#ifndef WC_EXP2_FMA_COLS
#define WC_EXP2_FMA_COLS 0
#endif
#ifndef WC_EXP2_FMA_SPREAD
#define WC_EXP2_FMA_SPREAD 0
#endif
// The quarter of a tile's row before whose exponentials a softmax warp hands
// the reference to its partner; 0 (as soon as it is decided, so the two
// warps' exponentials overlap) measured 2-6 % faster than the last quarter.
#ifndef WC_HANDOFF_QUARTER
#define WC_HANDOFF_QUARTER 0
#endif
// Attention over short coresets (at most two 128-key tiles) with at least two
// query tiles a head runs on the paired-row-tile kernel (expmm_pair_kernel):
// there a CTA's fixed start-up and store dominate, and pairing halves them per
// row tile (measured 1.37-1.44x on the ViT- and diffusion-shaped heads).  With
// more key tiles it was slower than expmm_tc_kernel (0.51-0.53 against 0.57-0.60
// of the bf16 burst figure on the long workload's heads: the issuing thread
// waits for PV_p(t) before S_p(t + 1) may overwrite P_p(t)), and so are the
// weights.  WC_PAIR_TILES = 0 turns it off.
#ifndef WC_PAIR_TILES
#define WC_PAIR_TILES 1
#endif
constexpr bool kPairTiles = WC_PAIR_TILES != 0;
constexpr int kFmaExpCols = WC_EXP2_FMA_COLS;
constexpr int kHandQuarter = WC_HANDOFF_QUARTER;
constexpr int kFmaExpSpread = WC_EXP2_FMA_SPREAD;
static_assert(kFmaExpCols % 8 == 0 && kFmaExpCols >= 0 && kFmaExpCols <= BN, "whole column pairs per quarter");
static_assert(kHandQuarter >= 0 && kHandQuarter <= 3, "hand-over quarter");
__host__ __device__ constexpr bool fma_exp_col(int col) {
    return kFmaExpSpread ? (col % 32) >= 32 - kFmaExpCols / 4 : col >= BN - kFmaExpCols;
}

struct TcArgs {
    const int32_t* rank;
    void* out;
    const float* wn;     // rownorm: normaliser column, [units][r_pad]
    const float* sigma;  // rownorm: column scales of the fp16 weights, [units][dv]
    int* status;
    int a_rows;          // rows of A per head (r or n_q)
    int a_head_rows;     // row stride of A between heads in the 2-D view
    int b_rows;          // rows of B per unit (n or r)
    int nsplit, split_len;
    int r, r_pad;
    int hq, group;
    int all_keys;        // rownorm: all b_rows rows count (binned coresets), else rank[unit]
    float cb;            // beta * log2(e)
    const float* bias;   // kModeBias: per-key logit bias (log2 units), [units][bias_stride]
    int bias_stride;
};

// MODE: kExpmmPartial, kExpmmRownorm, kModeBias = partial sums of
// exp(beta <a, b_j> + bias_j) (the centred kernel: the bias tile arrives with
// the value tile), or kModeAttnSplit = attention over one split of the
// coreset (blockIdx.y), written as an unnormalised partial row (O scaled by the
// column scales | normaliser share | reference) for attend_combine_kernel.
constexpr int kModeBias = 2;
constexpr int kModeAttnSplit = 3;

template <int D, int DV>
struct Smem {
    static constexpr uint32_t kA = BM * D * 2;         // the row tile of A
    static constexpr uint32_t kB = BN * D * 2;         // one key tile (1024-aligned: swizzle atoms)
    static constexpr uint32_t kC = BN * DV * 2;        // one value tile
    static constexpr uint32_t A = 0;
    static constexpr uint32_t B0 = kA;                  // [NB] key tiles
    static constexpr uint32_t C0 = B0 + NB * kB;        // [NC] value tiles
    static constexpr uint32_t Wv = C0 + NC * kC;        // [NC][BN] normaliser weights (rownorm)
    static constexpr uint32_t Tok = Wv + NC * BN * 4;   // [2][BM] fp32: reference maxima, then sums
    static constexpr uint32_t Bar = Tok + 2 * BM * 4;
    static constexpr uint32_t kTotal = Bar + 256;
    static constexpr uint32_t kAlloc = kTotal;          // the base is 1024-aligned (checked in the kernel)
    static_assert(kAlloc <= 232448, "shared memory per block");
    static_assert(BM * c1_row(DV) * 4 <= NC * kC, "the epilogue stages O in the value ring");
};

// TMEM: S / P buffer b (b = key block % 3) at columns 128 b .. +127 (P as
// fp16 pairs over the first 64 columns of the S it came from), O at
// 384 .. 384+DV-1.
template <int D, int DV, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    expmm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                    const __grid_constant__ CUtensorMap mapC, const TcArgs args) {
    using L = Smem<D, DV>;
    // A holds queries (rows mapped to kv units by the query-head group), the
    // normaliser is weighted by the coreset's normaliser column, and the value
    // columns carry scales; only kExpmmRownorm divides the rows out in place
    constexpr bool kQueries = MODE == kExpmmRownorm || MODE == kModeAttnSplit;
    constexpr bool kNormOut = MODE == kExpmmRownorm;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = smem_raw;
    if (smem_u32(sm) & 1023u) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) record_status(args.status, WC_ERR_UNSUPPORTED);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::Bar);
    uint64_t* fullB = bars;                   // [NB]
    uint64_t* emptyB = fullB + NB;            // [NB]
    uint64_t* fullC = emptyB + NB;            // [NC]
    uint64_t* emptyC = fullC + NC;            // [NC]
    uint64_t* a_full = emptyC + NC;
    uint64_t* s_full = a_full + 1;            // [NS]
    uint64_t* p_full = s_full + NS;           // [NS]
    uint64_t* p_free = p_full + NS;           // [NS]
    uint64_t* drain = p_free + NS;            // [2] (S issuer, PV issuer)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int z = blockIdx.z;
    int unit, a_valid, b_lo, b_hi, split = 0, a_row0;
    if (!kQueries) {
        unit = z;
        a_valid = args.rank[unit];
        if (!in_bounds(a_valid >= 0 && a_valid <= args.r, args.status)) return;
        split = blockIdx.y;
        b_lo = split * args.split_len;
        b_hi = min(args.b_rows, b_lo + args.split_len);
        a_row0 = unit * args.a_head_rows + blockIdx.x * BM;
    } else {
        const int hkv = args.hq / args.group;
        unit = (z / args.hq) * hkv + (z % args.hq) / args.group;
        a_valid = args.a_rows;
        const int b_all = args.all_keys ? args.b_rows : args.rank[unit];
        if (!in_bounds(b_all >= 0 && b_all <= args.b_rows, args.status)) return;
        split = MODE == kModeAttnSplit ? (int)blockIdx.y : 0;
        b_lo = split * args.split_len;
        b_hi = min(b_all, b_lo + args.split_len);
        a_row0 = z * args.a_head_rows + blockIdx.x * BM;
    }
    const int a0 = blockIdx.x * BM;
    if (a0 >= a_valid) return;
    const int T = b_hi > b_lo ? (b_hi - b_lo + BN - 1) / BN : 0;
    const int b_row0 = unit * args.b_rows + b_lo;

    if (tid == 0) {
        for (int i = 0; i < NB; ++i) {
            mbar_init(&fullB[i], 1);
            mbar_init(&emptyB[i], 1);
        }
        for (int i = 0; i < NC; ++i) {
            mbar_init(&fullC[i], 1);
            mbar_init(&emptyC[i], 1);
        }
        mbar_init(a_full, 1);
        for (int x = 0; x < NS; ++x) {
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 4);
            mbar_init(&p_free[x], 1);
        }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 2) tmem_alloc<512>(tmem_slot);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tO0 = tmem + NS * BN;

    if (warp < 4) {
        reg_release<kRegsSide>();             // loaders and issuers: few registers
        if (warp <= 1) {
            // ------------------------------------------------------------ TMA producers
            // warp 0 loads A once, then the key tiles; warp 1 the value tiles (and w)
            const bool keys = warp == 0;
            if (lane == 0 && T > 0) {
                if (keys) {
                    tma_prefetch(&mapA);
                    tma_prefetch(&mapB);
                    mbar_expect_tx(a_full, L::kA);
    #pragma unroll
                    for (int c = 0; c < D / 64; ++c) tma_load_2d(sm + L::A + c * (BM * 128), &mapA, a_full, c * 64, a_row0);
                } else {
                    tma_prefetch(&mapC);
                }
                const int NR = keys ? NB : NC;
                uint64_t* fl = keys ? fullB : fullC;
                uint64_t* em = keys ? emptyB : emptyC;
                int issued = 0;
                for (int t = 0; t < T; ++t) {
                    const int s = t % NR;
                    if (t >= NR && !mbar_wait(&em[s], ((t / NR) - 1) & 1, abort_flag, args.status, kTcTimeoutNs))
                        break;
                    const int brow = b_row0 + t * BN;
                    if (keys) {
                        mbar_expect_tx(&fl[s], L::kB);
                        unsigned char* st = sm + L::B0 + s * L::kB;
    #pragma unroll
                        for (int c = 0; c < D / 64; ++c) tma_load_2d(st + c * (BN * 128), &mapB, &fl[s], c * 64, brow);
                    } else {
                        mbar_expect_tx(&fl[s], L::kC + (MODE != kExpmmPartial ? BN * 4 : 0));
                        unsigned char* st = sm + L::C0 + s * L::kC;
    #pragma unroll
                        for (int c = 0; c < DV / 64; ++c) tma_load_2d(st + c * (BN * 128), &mapC, &fl[s], c * 64, brow);
                        if (kQueries)
                            bulk_load(sm + L::Wv + s * BN * 4, args.wn + (size_t)unit * args.r_pad + b_lo + t * BN,
                                      BN * 4, &fl[s]);
                        if (MODE == kModeBias)
                            bulk_load(sm + L::Wv + s * BN * 4,
                                      args.bias + (size_t)unit * args.bias_stride + b_lo + t * BN, BN * 4, &fl[s]);
                    }
                    issued = t + 1;
                }
                // wind down: every copy this thread started has landed before the block exits
                if (*abort_flag) {
                    const uint64_t t0 = global_ns();
                    while (keys && !mbar_try_wait(a_full, 0) && global_ns() - t0 < 100000000ull) {
                    }
                    for (int t = issued - NR > 0 ? issued - NR : 0; t < issued; ++t) {
                        const uint64_t t1 = global_ns();
                        while (!mbar_try_wait(&fl[t % NR], (t / NR) & 1) && global_ns() - t1 < 100000000ull) {
                        }
                    }
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------------------ S issuer: S(t) = A B_t^T into buffer t % NS
            if (lane == 0 && T > 0) {
                constexpr uint32_t idS = idesc_f16(BM, BN, 1, 1, 0, 0);   // bf16 x bf16, both K-major
                const uint64_t dA = sdesc_sw128(smem_u32(sm + L::A), 16, 1024);
                const uint64_t dB = sdesc_sw128(smem_u32(sm + L::B0), 16, 1024);
                bool ok = mbar_wait(a_full, 0, abort_flag, args.status, kTcTimeoutNs);
                for (int t = 0; ok && t < T; ++t) {
                    const int x = t % NS;
                    ok = mbar_wait(&fullB[t % NB], (t / NB) & 1, abort_flag, args.status, kTcTimeoutNs);
                    // the buffer holds P(t - NS) until PV(t - NS) has completed
                    if (ok && t >= NS) ok = mbar_wait(&p_free[x], ((t / NS) - 1) & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t b = dB + (uint64_t)(((t % NB) * L::kB) >> 4);
    #pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // 16 elements = 32 bytes into the 128-byte row; 64-element chunks stacked
                        const uint64_t oa = (uint64_t)(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
                        const uint64_t ob = (uint64_t)(((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4);
                        mma_f16_ss(tmem + x * BN, dA + oa, b + ob, idS, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[x]);
                    mma_commit(&emptyB[t % NB]);
                }
                mma_commit(&drain[0]);
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(&drain[0], 0) && global_ns() - t0 < 1000000000ull) {
                }
            }
        } else if (warp == 3) {
            // ------------------------------------------------------------ PV issuer: O += P(t) C_t
            if (lane == 0 && T > 0) {
                constexpr uint32_t idO = idesc_f16(BM, DV, 0, 0, 0, 1);   // f16 P (TMEM) x f16 C (MN-major)
                const uint64_t dC = sdesc_sw128(smem_u32(sm + L::C0), BN * 128, 1024);
                bool ok = true;
                for (int t = 0; ok && t < T; ++t) {
                    const int x = t % NS;
                    ok = mbar_wait(&p_full[x], (t / NS) & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (ok) ok = mbar_wait(&fullC[t % NC], (t / NC) & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t c = dC + (uint64_t)(((t % NC) * L::kC) >> 4);
    #pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_f16_ts(tO0, tmem + x * BN + 8 * kk, c + (uint64_t)((kk * 16 * 128) >> 4), idO,
                                   (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&p_free[x]);
                    mma_commit(&emptyC[t % NC]);
                }
                mma_commit(&drain[1]);
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(&drain[1], 0) && global_ns() - t0 < 1000000000ull) {
                }
            }
        }
    } else {
        reg_claim<kRegsSoftmax>();            // softmax warps: a whole S row per thread
        // ------------------------------------------------------------ softmax + epilogue
        const int q = warp & 3;                 // TMEM lanes 32 q .. 32 q + 31
        const int par = (warp - 4) >> 2;        // this warp takes the key tiles t with t % 2 == par
        const int row = q * 32 + lane;
        // named barriers that hand the reference on: 1 + q from parity 0 to 1, 5 + q back
        const int id_in = par ? 1 + q : 5 + q;
        const int id_out = par ? 5 + q : 1 + q;
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        float* tok = reinterpret_cast<float*>(sm + L::Tok);   // [2][BM]
        const float cb = args.cb;
        float mO = -INFINITY;                   // the reference of O (log2 units) as this warp knows it
        float l = 0.f;                          // this warp's share of the normaliser, relative to mO
        bool ok = true;
        // Every iteration runs the same barrier steps whatever `ok` is, so a warp
        // that gave up still hands the reference on and its partner never hangs.
        for (int t = par; t < T; t += 2) {
            const int x = t % NS;
            const uint32_t tS = tmem + x * BN + lanes;
            ok = ok && mbar_wait(&s_full[x], (t / NS) & 1, abort_flag, args.status, kTcTimeoutNs);
            ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-collective
            const int valid = b_hi - (b_lo + t * BN);
            // pass 1: the whole row of S into registers, and its maximum
            float sv[BN];
            float mt = -INFINITY;
            if (ok && MODE == kModeBias) {
                // the logit bias arrives with the value tile
                ok = mbar_wait(&fullC[t % NC], (t / NC) & 1, abort_flag, args.status, kTcTimeoutNs);
                ok = __all_sync(0xffffffffu, ok);
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < 4; ++h) tmem_ld32(tS + 32 * h, sv + 32 * h);
                tmem_wait_ld();
                if (MODE == kModeBias) {
                    // logits in log2 units, biased: S cb + bias_j (pass 2 then only subtracts the reference)
                    const float* bv = reinterpret_cast<const float*>(sm + L::Wv + (t % NC) * BN * 4);
#pragma unroll
                    for (int j = 0; j < BN; j += 4) {
                        const float4 f = lds_f4_ordered(bv + j);
                        const float2 lo = fma2(make_float2(sv[j], sv[j + 1]), make_float2(cb, cb), make_float2(f.x, f.y));
                        const float2 hi =
                            fma2(make_float2(sv[j + 2], sv[j + 3]), make_float2(cb, cb), make_float2(f.z, f.w));
                        sv[j] = lo.x;
                        sv[j + 1] = lo.y;
                        sv[j + 2] = hi.x;
                        sv[j + 3] = hi.y;
                    }
                }
                if (valid < BN) {
#pragma unroll
                    for (int j = 0; j < BN; ++j)
                        if (j >= valid) sv[j] = -INFINITY;
                }
                float mq[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mq[i] = sv[i];
#pragma unroll
                for (int j = 8; j < BN; j += 2) mq[(j >> 1) & 7] = fmax3(mq[(j >> 1) & 7], sv[j], sv[j + 1]);
                mt = fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
                if (MODE != kModeBias) mt *= cb;
            }
            // the reference after tile t - 1 (decided by the partner)
            if (t > 0) {
                pair_sync(id_in);
                const float mp = tok[row];
                if (mp != mO) {
                    if (mO != -INFINITY) l *= ex2(mO - mp);
                    mO = mp;
                }
            }
            const bool grow = __any_sync(0xffffffffu, ok && mt > mO + kRescale);
            const float mn = grow ? fmaxf(mO, mt) : mO;
            const float mold = mO;
            if (grow) {
                if (mO != -INFINITY) l *= ex2(mO - mn);
                mO = mn;
            }
            if (t + 1 < T) tok[row] = mn;       // the partner reads it after this tile's hand-over below
            if (ok && kQueries) {
                // w arrives with the value tile; this stage cannot be reloaded before PV(t)
                ok = mbar_wait(&fullC[t % NC], (t / NC) & 1, abort_flag, args.status, kTcTimeoutNs);
                ok = __all_sync(0xffffffffu, ok);
            }
            bool handed = false;
            if (ok) {
                // pass 2: P = 2^(S cb - mO) as fp16 pairs over the first 64 columns
                const float* wv = reinterpret_cast<const float*>(sm + L::Wv + (t % NC) * BN * 4);
                const float nm = -mO;
                const float2 nm2 = make_float2(nm, nm), cb2 = make_float2(cb, cb);
                float2 lp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                make_float2(0.f, 0.f)};
                // Software-pipelined by 32-column quarter: iteration h issues the
                // exponentials of quarter h (results written over the logits) between
                // the packing and normaliser sums of quarter h - 1, whose inputs are
                // ready by then, so the warp's in-order issue does not wait on the
                // exponential unit's latency, and stores quarter h - 1 as fp16 pairs.
#pragma unroll
                for (int h = 0; h <= 4; ++h) {
                    if (h == kHandQuarter) {
                        // hand the reference on: the partner's exponentials may start
                        if (t + 1 < T) pair_arrive(id_out);
                        handed = true;
                    }
                    uint32_t packed[16];
                    float w[kQueries ? 32 : 1];
                    if (kQueries && h > 0) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 f = lds_f4_ordered(wv + 32 * (h - 1) + j);
                            w[j] = f.x;
                            w[j + 1] = f.y;
                            w[j + 2] = f.z;
                            w[j + 3] = f.w;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        if (h < 4) {
                            // logits of the pair in log2 units, shifted by the reference
                            const int c = 32 * h + j;
                            const float2 s2 = make_float2(sv[c], sv[c + 1]);
                            const float2 x2 = MODE == kModeBias ? add2(s2, nm2) : fma2(s2, cb2, nm2);
                            float2 p;
                            if (fma_exp_col(c)) {
                                p = exp2_fma2(x2);
                            } else {
                                p.x = ex2_ordered(x2.x);
                                p.y = ex2_ordered(x2.y);
                            }
                            sv[c] = p.x;
                            sv[c + 1] = p.y;
                        }
                        if (h > 0) {
                            const int c = 32 * (h - 1) + j;
                            const float2 p = make_float2(sv[c], sv[c + 1]);
                            if (kQueries)
                                lp[(j >> 1) & 3] = fma2(p, make_float2(w[j], w[j + 1]), lp[(j >> 1) & 3]);
                            else
                                lp[(j >> 1) & 3] = add2(lp[(j >> 1) & 3], p);
                            packed[j >> 1] = pack_half2_ordered(p.x, p.y);
                        }
                    }
                    if (h > 0) tmem_st16u(tS + 16 * (h - 1), packed);
                }
                const float2 l01 = add2(lp[0], lp[1]), l23 = add2(lp[2], lp[3]);
                l += (l01.x + l01.y) + (l23.x + l23.y);
                tmem_wait_st();
                if (grow && t > 0) {
                    // O holds key blocks 0..t-1 in the old reference: once the last of them
                    // has landed, rescale it in place (PV(t) is issued only after this)
                    ok = mbar_wait(&p_free[(t - 1) % NS], ((t - 1) / NS) & 1, abort_flag, args.status, kTcTimeoutNs);
                    ok = __all_sync(0xffffffffu, ok);
                    if (ok) {
                        tc_fence_after();
                        const float sc = (mold == -INFINITY) ? 0.f : ex2(mold - mn);
#pragma unroll
                        for (int c0 = 0; c0 < DV; c0 += 32) {
                            float o[32];
                            tmem_ld32(tO0 + lanes + c0, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] *= sc;
                            tmem_st32(tO0 + lanes + c0, o);
                        }
                        tmem_wait_st();
                    }
                }
                if (ok) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full[x]);
                }
            }
            // (if pass 2 was skipped, hand the reference on here: the partner never hangs)
            if (!handed && t + 1 < T) pair_arrive(id_out);
        }

        // ------------------------------------------------------------ epilogue
        // The warp that took the last tile (parity (T - 1) & 1; parity 1 when
        // T == 0) knows the final reference.  The other hands it log2 of its
        // share of the normaliser in its own reference; the last one adds the
        // two in the final reference and hands the total back.
        // the column scales of the attention output, loaded before the waits below
        float sgv[kQueries ? DV / 2 : 1];
        if (kQueries) {
            const float4* s4 = reinterpret_cast<const float4*>(args.sigma + (size_t)unit * DV + par * (DV / 2));
#pragma unroll
            for (int c = 0; c < DV / 2; c += 4) {
                const float4 f = __ldg(s4 + c / 4);
                sgv[c] = f.x;
                sgv[c + 1] = f.y;
                sgv[c + 2] = f.z;
                sgv[c + 3] = f.w;
            }
        }
        const bool last = par == ((T + 1) & 1);
        float* tl = tok + BM;                   // second slot: only the epilogue uses it
        float lt;
        // (its own barrier 9 + q first: its last hand-over may not have been taken yet)
        if (!last) {
            tl[row] = (l > 0.f) ? __log2f(l) + mO : -INFINITY;
            pair_arrive(9 + q);
            pair_sync(id_in);
            lt = tl[row];
        } else {
            pair_sync(9 + q);
            const float lo = tl[row];
            lt = l + ((lo == -INFINITY) ? 0.f : ex2(lo - mO));
            tl[row] = lt;
            pair_arrive(id_out);
        }
        if (ok && T > 0) {
            ok = mbar_wait(&p_free[(T - 1) % NS], ((T - 1) / NS) & 1, abort_flag, args.status, kTcTimeoutNs);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) tc_fence_after();
        }
        // O goes out through shared memory (the value ring is idle once PV(T - 1)
        // has completed): each warp stages half of the columns of its 32 rows
        // (staged rows DV + 4 floats apart, 16-byte aligned), then bulk
        // asynchronous copies move the rows to global memory: the partial sums'
        // rows are one contiguous run (the same row stride), attention rows go
        // one copy per row.
        constexpr int SST = c1_row(DV);
        float* stg = reinterpret_cast<float*>(sm + L::C0);
        const bool have_o = ok && T > 0;
        const uint32_t tO = tO0 + lanes + par * (DV / 2);
        const float inv = kNormOut ? 1.f / lt : 1.f;
        float* srow = stg + row * SST + par * (DV / 2);
#pragma unroll
        for (int c0 = 0; c0 < DV / 2; c0 += 32) {
            float o[32];
            if (have_o) {
                tmem_ld32(tO + c0, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                float4 v = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                if (kQueries) {
                    v.x *= sgv[c0 + c] * inv;
                    v.y *= sgv[c0 + c + 1] * inv;
                    v.z *= sgv[c0 + c + 2] * inv;
                    v.w *= sgv[c0 + c + 3] * inv;
                }
                *reinterpret_cast<float4*>(srow + c0 + c) = v;
            }
        }
        if (!kNormOut && last) *reinterpret_cast<float2*>(stg + row * SST + DV) = make_float2(lt, mO * kLn2);
        fence_async_smem();                     // the bulk copies read the staged rows through the async proxy
        softmax_sync();                         // all 8 softmax warps have staged their part
        const int rows = min(BM, a_valid - a0);
        const int st = tid - 4 * 32;            // 0 .. 255
        if (ok && !kNormOut && st == 0) {
            const size_t prow = kQueries ? ((size_t)z * args.nsplit + split) * args.a_rows + a0
                                         : ((size_t)unit * args.nsplit + split) * args.r + a0;
            bulk_store(static_cast<float*>(args.out) + prow * SST, stg, (uint32_t)(rows * SST * 4));
            bulk_commit();
            bulk_wait_read_all();
        }
        if (ok && kNormOut && st < rows) {
            bulk_store(static_cast<float*>(args.out) + ((size_t)z * args.a_rows + a0 + st) * DV, stg + st * SST,
                       (uint32_t)(DV * 4));
            bulk_commit();
            bulk_wait_read_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc<512>(tmem);
}

// ---------------------------------------------------------------------------
// Paired row tiles: one CTA computes two 128-row tiles of A (256 rows) against
// the same key and value tiles, each loaded once for both.  Softmax warps 4..7
// own row tile 0 and warps 8..11 row tile 1: a warp holds whole rows, so it
// keeps its own running maximum (no hand-over between warps), and the two
// warps of an SM sub-partition run their exponentials side by side on the
// exponential unit.  One thread issues every MMA, interleaving the two tiles
// so that each softmax has the other tile's MMAs to hide behind:
//   S0(0) S1(0) | PV0(t) S0(t+1) PV1(t) S1(t+1) | ...
// S_p(t+1) overwrites the TMEM columns from which PV_p(t) reads P_p(t); the
// issuing thread waits for PV_p(t) to complete first.
// TMEM: S_p at columns 128 p (P_p as fp16 pairs over its first 64 columns),
// O_p at 256 + DV p.  Modes: kExpmmPartial (the weights' partial sums) and
// kExpmmRownorm (attention).  The epilogue stages both tiles' rows in the
// operand rings (idle once the last MMA has completed) and stores them with
// bulk asynchronous copies.
template <int D, int DV>
struct SmemPair {
    static constexpr uint32_t kA = BM * D * 2;
    static constexpr uint32_t kB = BN * D * 2;
    static constexpr uint32_t kC = BN * DV * 2;
    // stages of the key and value rings: as many as fit beside both row tiles
    static constexpr int kStages = 2 * kA + 4 * (kB + kC + BN * 4) + 4096 <= 232448   ? 4
                                   : 2 * kA + 3 * (kB + kC + BN * 4) + 4096 <= 232448 ? 3
                                                                                       : 2;
    static constexpr uint32_t A = 0;                              // [2] row tiles
    static constexpr uint32_t B0 = 2 * kA;                        // [kStages] key tiles
    static constexpr uint32_t C0 = B0 + kStages * kB;             // [kStages] value tiles
    static constexpr uint32_t Wv = C0 + kStages * kC;             // [kStages][BN] normaliser weights
    static constexpr uint32_t Bar = Wv + kStages * BN * 4;
    static constexpr uint32_t kAlloc = Bar + 256;
    // epilogue staging of row tile p (rows c1_row(DV) floats apart) over the idle rings
    static constexpr uint32_t kStageBytes = (BM * c1_row(DV) * 4 + 1023) / 1024 * 1024;
    static_assert(2 * kStageBytes <= Wv, "both row tiles stage in the operand rings");
    static_assert(kAlloc <= 232448, "shared memory per block");
};

template <int D, int DV, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    expmm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                      const __grid_constant__ CUtensorMap mapC, const TcArgs args) {
    using L = SmemPair<D, DV>;
    constexpr int NR = L::kStages;
    constexpr bool kQueries = MODE == kExpmmRownorm;
    static_assert(MODE == kExpmmPartial || MODE == kExpmmRownorm, "paired tiles: weights or attention");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = smem_raw;
    if (smem_u32(sm) & 1023u) {
        if (threadIdx.x == 0) record_status(args.status, WC_ERR_UNSUPPORTED);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::Bar);
    uint64_t* fullB = bars;                   // [NR]
    uint64_t* emptyB = fullB + NR;            // [NR]
    uint64_t* fullC = emptyB + NR;            // [NR]
    uint64_t* emptyC = fullC + NR;            // [NR]
    uint64_t* a_full = emptyC + NR;
    uint64_t* s_full = a_full + 1;            // [2] per row tile
    uint64_t* p_full = s_full + 2;            // [2]
    uint64_t* pv_done = p_full + 2;           // [2]
    uint64_t* drain = pv_done + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int z = blockIdx.z;
    int unit, a_valid, b_lo, b_hi, split = 0, a_row0;
    if (!kQueries) {
        unit = z;
        a_valid = args.rank[unit];
        if (!in_bounds(a_valid >= 0 && a_valid <= args.r, args.status)) return;
        split = blockIdx.y;
        b_lo = split * args.split_len;
        b_hi = min(args.b_rows, b_lo + args.split_len);
        a_row0 = unit * args.a_head_rows + blockIdx.x * 2 * BM;
    } else {
        const int hkv = args.hq / args.group;
        unit = (z / args.hq) * hkv + (z % args.hq) / args.group;
        a_valid = args.a_rows;
        const int b_all = args.all_keys ? args.b_rows : args.rank[unit];
        if (!in_bounds(b_all >= 0 && b_all <= args.b_rows, args.status)) return;
        b_lo = 0;
        b_hi = b_all;
        a_row0 = z * args.a_head_rows + blockIdx.x * 2 * BM;
    }
    const int a0 = blockIdx.x * 2 * BM;
    if (a0 >= a_valid) return;
    const int T = b_hi > b_lo ? (b_hi - b_lo + BN - 1) / BN : 0;
    const int b_row0 = unit * args.b_rows + b_lo;

    if (tid == 0) {
        for (int i = 0; i < NR; ++i) {
            mbar_init(&fullB[i], 1);
            mbar_init(&emptyB[i], 1);
            mbar_init(&fullC[i], 1);
            mbar_init(&emptyC[i], 1);
        }
        mbar_init(a_full, 1);
        for (int p = 0; p < 2; ++p) {
            mbar_init(&s_full[p], 1);
            mbar_init(&p_full[p], 4);
            mbar_init(&pv_done[p], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 2) tmem_alloc<512>(tmem_slot);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        reg_release<kRegsSide>();
        if (warp <= 1) {
            // ------------------------------------------------------------ TMA producers
            // warp 0: both row tiles of A, then the key tiles; warp 1: the value tiles (and w)
            const bool keys = warp == 0;
            if (lane == 0 && T > 0) {
                if (keys) {
                    tma_prefetch(&mapA);
                    tma_prefetch(&mapB);
                    mbar_expect_tx(a_full, 2 * L::kA);
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_2d(sm + L::A + p * L::kA + c * (BM * 128), &mapA, a_full, c * 64, a_row0 + p * BM);
                } else {
                    tma_prefetch(&mapC);
                }
                uint64_t* fl = keys ? fullB : fullC;
                uint64_t* em = keys ? emptyB : emptyC;
                int issued = 0;
                for (int t = 0; t < T; ++t) {
                    const int s = t % NR;
                    if (t >= NR && !mbar_wait(&em[s], ((t / NR) - 1) & 1, abort_flag, args.status, kTcTimeoutNs))
                        break;
                    const int brow = b_row0 + t * BN;
                    if (keys) {
                        mbar_expect_tx(&fl[s], L::kB);
                        unsigned char* st = sm + L::B0 + s * L::kB;
#pragma unroll
                        for (int c = 0; c < D / 64; ++c) tma_load_2d(st + c * (BN * 128), &mapB, &fl[s], c * 64, brow);
                    } else {
                        mbar_expect_tx(&fl[s], L::kC + (kQueries ? BN * 4 : 0));
                        unsigned char* st = sm + L::C0 + s * L::kC;
#pragma unroll
                        for (int c = 0; c < DV / 64; ++c) tma_load_2d(st + c * (BN * 128), &mapC, &fl[s], c * 64, brow);
                        if (kQueries)
                            bulk_load(sm + L::Wv + s * BN * 4, args.wn + (size_t)unit * args.r_pad + b_lo + t * BN,
                                      BN * 4, &fl[s]);
                    }
                    issued = t + 1;
                }
                if (*abort_flag) {
                    const uint64_t t0 = global_ns();
                    while (keys && !mbar_try_wait(a_full, 0) && global_ns() - t0 < 100000000ull) {
                    }
                    for (int t = issued - NR > 0 ? issued - NR : 0; t < issued; ++t) {
                        const uint64_t t1 = global_ns();
                        while (!mbar_try_wait(&fl[t % NR], (t / NR) & 1) && global_ns() - t1 < 100000000ull) {
                        }
                    }
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------------------ MMA issuer (both row tiles)
            if (lane == 0) {
                constexpr uint32_t idS = idesc_f16(BM, BN, 1, 1, 0, 0);   // bf16 x bf16, both K-major
                constexpr uint32_t idO = idesc_f16(BM, DV, 0, 0, 0, 1);   // f16 P (TMEM) x f16 C (MN-major)
                const uint64_t dA = sdesc_sw128(smem_u32(sm + L::A), 16, 1024);
                const uint64_t dB = sdesc_sw128(smem_u32(sm + L::B0), 16, 1024);
                const uint64_t dC = sdesc_sw128(smem_u32(sm + L::C0), BN * 128, 1024);
                auto issue_s = [&](int p, int t) {
                    const uint64_t a = dA + (uint64_t)((p * L::kA) >> 4);
                    const uint64_t b = dB + (uint64_t)(((t % NR) * L::kB) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t oa = (uint64_t)(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
                        const uint64_t ob = (uint64_t)(((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4);
                        mma_f16_ss(tmem + p * BN, a + oa, b + ob, idS, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[p]);
                };
                auto issue_pv = [&](int p, int t) {
                    const uint64_t c = dC + (uint64_t)(((t % NR) * L::kC) >> 4);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_f16_ts(tmem + 2 * BN + p * DV, tmem + p * BN + 8 * kk, c + (uint64_t)((kk * 16 * 128) >> 4),
                                   idO, (t > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&pv_done[p]);
                };
                bool ok = T > 0 && mbar_wait(a_full, 0, abort_flag, args.status, kTcTimeoutNs);
                if (ok) ok = mbar_wait(&fullB[0], 0, abort_flag, args.status, kTcTimeoutNs);
                if (ok) {
                    tc_fence_after();
                    issue_s(0, 0);
                    issue_s(1, 0);
                    mma_commit(&emptyB[0]);
                }
                for (int t = 0; ok && t < T; ++t) {
                    const bool more = t + 1 < T;
                    ok = mbar_wait(&fullC[t % NR], (t / NR) & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (ok) ok = mbar_wait(&p_full[0], t & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(0, t);
                    if (more) {
                        ok = mbar_wait(&fullB[(t + 1) % NR], ((t + 1) / NR) & 1, abort_flag, args.status, kTcTimeoutNs);
                        // S_0(t + 1) overwrites the columns PV_0(t) reads P_0(t) from
                        if (ok) ok = mbar_wait(&pv_done[0], t & 1, abort_flag, args.status, kTcTimeoutNs);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(0, t + 1);
                    }
                    ok = mbar_wait(&p_full[1], t & 1, abort_flag, args.status, kTcTimeoutNs);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, t);
                    mma_commit(&emptyC[t % NR]);
                    if (more) {
                        ok = mbar_wait(&pv_done[1], t & 1, abort_flag, args.status, kTcTimeoutNs);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(1, t + 1);
                        mma_commit(&emptyB[(t + 1) % NR]);
                    }
                }
                mma_commit(drain);
            }
        }
    } else {
        reg_claim<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax + epilogue of row tile p
        const int p = (warp - 4) >> 2;          // row tile of this warp
        const int q = warp & 3;                 // TMEM lanes 32 q .. 32 q + 31
        const int row = q * 32 + lane;
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        const uint32_t tS = tmem + p * BN + lanes;
        const uint32_t tO = tmem + 2 * BN + p * DV + lanes;
        const float cb = args.cb;
        const float2 cb2 = make_float2(cb, cb);
        float mO = -INFINITY;                   // this row's reference (log2 units)
        float l = 0.f;                          // its normaliser share, relative to mO
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            ok = ok && mbar_wait(&s_full[p], t & 1, abort_flag, args.status, kTcTimeoutNs);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const int valid = b_hi - (b_lo + t * BN);
            float sv[BN];
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 4; ++h) tmem_ld32(tS + 32 * h, sv + 32 * h);
            tmem_wait_ld();
            if (valid < BN) {
#pragma unroll
                for (int j = 0; j < BN; ++j)
                    if (j >= valid) sv[j] = -INFINITY;
            }
            float mq[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mq[i] = sv[i];
#pragma unroll
            for (int j = 8; j < BN; j += 2) mq[(j >> 1) & 7] = fmax3(mq[(j >> 1) & 7], sv[j], sv[j + 1]);
            const float mt = fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7])) * cb;
            const bool grow = __any_sync(0xffffffffu, mt > mO + kRescale);
            if (grow) {
                const float mn = fmaxf(mO, mt);
                const float sc = (mO == -INFINITY) ? 0.f : ex2(mO - mn);
                l *= sc;
                if (t > 0) {
                    // O holds key tiles 0..t-1 in the old reference: rescale once PV(t - 1) has landed
                    ok = mbar_wait(&pv_done[p], (t - 1) & 1, abort_flag, args.status, kTcTimeoutNs);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < DV; c0 += 32) {
                        float o[32];
                        tmem_ld32(tO + c0, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= sc;
                        tmem_st32(tO + c0, o);
                    }
                    tmem_wait_st();
                }
                mO = mn;
            }
            if (kQueries) {
                // w arrives with the value tile; this stage cannot be reloaded before PV_1(t)
                ok = mbar_wait(&fullC[t % NR], (t / NR) & 1, abort_flag, args.status, kTcTimeoutNs);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            const float* wv = reinterpret_cast<const float*>(sm + L::Wv + (t % NR) * BN * 4);
            const float2 nm2 = make_float2(-mO, -mO);
            float2 lp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
            // quarter h's exponentials between the packing of quarter h - 1 (see expmm_tc_kernel)
#pragma unroll
            for (int h = 0; h <= 4; ++h) {
                uint32_t packed[16];
                float w[kQueries ? 32 : 1];
                if (kQueries && h > 0) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 f = lds_f4_ordered(wv + 32 * (h - 1) + j);
                        w[j] = f.x;
                        w[j + 1] = f.y;
                        w[j + 2] = f.z;
                        w[j + 3] = f.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    if (h < 4) {
                        const int c = 32 * h + j;
                        const float2 x2 = fma2(make_float2(sv[c], sv[c + 1]), cb2, nm2);
                        float2 pp;
                        if (fma_exp_col(c)) {
                            pp = exp2_fma2(x2);
                        } else {
                            pp.x = ex2_ordered(x2.x);
                            pp.y = ex2_ordered(x2.y);
                        }
                        sv[c] = pp.x;
                        sv[c + 1] = pp.y;
                    }
                    if (h > 0) {
                        const int c = 32 * (h - 1) + j;
                        const float2 pp = make_float2(sv[c], sv[c + 1]);
                        if (kQueries)
                            lp[(j >> 1) & 3] = fma2(pp, make_float2(w[j], w[j + 1]), lp[(j >> 1) & 3]);
                        else
                            lp[(j >> 1) & 3] = add2(lp[(j >> 1) & 3], pp);
                        packed[j >> 1] = pack_half2_ordered(pp.x, pp.y);
                    }
                }
                if (h > 0) tmem_st16u(tS + 16 * (h - 1), packed);
            }
            const float2 l01 = add2(lp[0], lp[1]), l23 = add2(lp[2], lp[3]);
            l += (l01.x + l01.y) + (l23.x + l23.y);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[p]);
        }

        // ------------------------------------------------------------ epilogue of row tile p
        // once every MMA has completed the operand rings are idle: row tile p stages its
        // rows (c1_row(DV) floats apart) at L::kStageBytes p, then bulk copies store them
        const float4* s4 = reinterpret_cast<const float4*>(args.sigma + (size_t)unit * DV);
        {
            const uint64_t t0 = global_ns();
            bool drained = false;
            while (!(drained = mbar_try_wait(drain, 0)) && global_ns() - t0 < 2000000000ull) {
            }
            if (!drained) {
                record_status(args.status, WC_ERR_TIMEOUT);
                ok = false;
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok) tc_fence_after();
        constexpr int SST = c1_row(DV);
        float* stg = reinterpret_cast<float*>(sm + p * L::kStageBytes);
        const bool have_o = ok && T > 0;
        const float inv = kQueries ? 1.f / l : 1.f;
        float* srow = stg + row * SST;
#pragma unroll
        for (int c0 = 0; c0 < DV; c0 += 32) {
            float o[32];
            if (have_o) {
                tmem_ld32(tO + c0, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                float4 v = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                if (kQueries) {
                    const float4 g = __ldg(s4 + (c0 + c) / 4);   // the column scales of the fp16 weights
                    v.x *= g.x * inv;
                    v.y *= g.y * inv;
                    v.z *= g.z * inv;
                    v.w *= g.w * inv;
                }
                *reinterpret_cast<float4*>(srow + c0 + c) = v;
            }
        }
        if (!kQueries) *reinterpret_cast<float2*>(srow + DV) = make_float2(l, mO * kLn2);
        fence_async_smem();
        asm volatile("bar.sync %0, 128;" ::"r"(1 + p) : "memory");   // the row tile's 4 warps have staged
        const int ap = a0 + p * BM;
        const int rows = min(BM, a_valid - ap);
        const int st = tid - 4 * 32 - p * 128;  // 0 .. 127 within the row tile
        if (ok && rows > 0) {
            if (!kQueries && st == 0) {
                const size_t prow = ((size_t)unit * args.nsplit + split) * args.r + ap;
                bulk_store(static_cast<float*>(args.out) + prow * SST, stg, (uint32_t)(rows * SST * 4));
                bulk_commit();
                bulk_wait_read_all();
            }
            if (kQueries && st < rows) {
                bulk_store(static_cast<float*>(args.out) + ((size_t)z * args.a_rows + ap + st) * DV, stg + st * SST,
                           (uint32_t)(DV * 4));
                bulk_commit();
                bulk_wait_read_all();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc<512>(tmem);
}

// Key-split attention: row q of query head h from its splits' partial rows
// (O_s | l_s | m_s, m in natural-log units):
//   out[h][q][c] = sum_s e_s O_s[c] / sum_s e_s l_s,  e_s = exp(m_s - max_s m_s).
// One warp per query row, lanes over the value columns.
template <int DV>
__global__ void attend_combine_kernel(const float* __restrict__ part, float* __restrict__ out, int nq, int nsplit,
                                      int rows_total) {
    constexpr int SST = c1_row(DV);
    const int wrow = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (wrow >= rows_total) return;
    const int h = wrow / nq, qr = wrow - h * nq;
    const size_t sstride = (size_t)nq * SST;                 // between splits
    const float* p = part + ((size_t)h * nsplit * nq + qr) * SST;
    float mx = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) mx = fmaxf(mx, p[sp * sstride + DV + 1]);
    float acc[DV / 32], lsum = 0.f;
#pragma unroll
    for (int k = 0; k < DV / 32; ++k) acc[k] = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) {
        const float* ps = p + sp * sstride;
        const float m = ps[DV + 1];
        const float e = m == -INFINITY ? 0.f : expf(m - mx);
        lsum = fmaf(e, ps[DV], lsum);
#pragma unroll
        for (int k = 0; k < DV / 32; ++k) acc[k] = fmaf(e, ps[lane + 32 * k], acc[k]);
    }
    const float inv = 1.f / lsum;
    float* o = out + (size_t)wrow * DV;
#pragma unroll
    for (int k = 0; k < DV / 32; ++k) o[lane + 32 * k] = acc[k] * inv;
}

// The exp-GEMM's two ways to compute 2^x, over an array (for tests):
// method 0 = exp2_fma2 (FMA / ALU pipes), 1 = ex2.approx.ftz (exponential unit).
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n, int method) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 2;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
        const bool two = i + 1 < n;
        const float a = x[i], b = two ? x[i + 1] : 0.f;
        float2 v;
        if (method == 0) {
            v = exp2_fma2(make_float2(a, b));
        } else {
            v.x = ex2(a);
            v.y = ex2(b);
        }
        y[i] = v.x;
        if (two) y[i + 1] = v.y;
    }
}

// V (bf16) -> fp16 copy for the value operand of the weights GEMM, 8 elements
// (16 bytes each way) a thread and iteration; count is a multiple of 8 (dv is).
__global__ void to_half_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, size_t count) {
    const uint4* s8 = reinterpret_cast<const uint4*>(src);
    uint4* d8 = reinterpret_cast<uint4*>(dst);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count / 8; i += (size_t)gridDim.x * blockDim.x) {
        const uint4 v = s8[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __half2 h = __floats2half2_rn(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
            o[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
        d8[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// The attention's weights as the tensor cores take them: per unit and value
// column c, sigma_c = max_s |W[s][c]| over the live rows (1 for an all-zero
// column), W16[s][c] = fp16(W[s][c] / sigma_c) (zero rows up to r), and the
// normaliser column wn[s] = W[s][dv] in fp32 (zero up to r_pad).  A cluster of
// kPrepCluster blocks per (unit, 32 columns); block q of the cluster takes rows
// 8 q + g + 64 k (warp g), so every block walks r / 64 rows.  The blocks'
// column maxima meet through distributed shared memory, then each block scales
// the rows it just read (from L2).
constexpr int kPrepCluster = 8;
constexpr int kPrepWarps = 8;

__global__ void __cluster_dims__(kPrepCluster, 1, 1) __launch_bounds__(kPrepWarps * 32)
    weights_prep_kernel(const float* __restrict__ W, const int32_t* __restrict__ rank, float* sigma, __half* W16,
                        float* wn, int r, int r_pad, int dv, int all_keys, int* status) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int q = (int)cluster.block_rank();
    const int u = blockIdx.x / kPrepCluster, lane = threadIdx.x & 31, g = threadIdx.x >> 5;
    const int c = blockIdx.y * 32 + lane;
    int k = all_keys ? r : rank[u];
    if (!in_bounds(k >= 0 && k <= r, status)) k = 0;   // (no early return: the cluster waits below)
    const float* Wu = W + (size_t)u * r * (dv + 1);
    const int s0 = q * kPrepWarps + g, step = kPrepCluster * kPrepWarps;
    float mx = 0.f;
    if (c < dv) {
#pragma unroll 4
        for (int s = s0; s < k; s += step) mx = fmaxf(mx, fabsf(Wu[(size_t)s * (dv + 1) + c]));
    }
    __shared__ float part[kPrepWarps][33];
    __shared__ float bmax[32];
    part[g][lane] = mx;
    __syncthreads();
    if (g == 0) {
        float m = part[0][lane];
#pragma unroll
        for (int i = 1; i < kPrepWarps; ++i) m = fmaxf(m, part[i][lane]);
        bmax[lane] = m;
    }
    cluster.sync();                            // every block's maxima are in its shared memory
    float m = 0.f;
#pragma unroll
    for (int p = 0; p < kPrepCluster; ++p) m = fmaxf(m, cluster.map_shared_rank(bmax, p)[lane]);
    cluster.sync();                            // no block leaves while a peer still reads its maxima
    const float sg = m > 0.f ? m : 1.f;
    if (c < dv) {
        if (q == 0 && g == 0) sigma[(size_t)u * dv + c] = sg;
        __half* Wh = W16 + (size_t)u * r * dv;
#pragma unroll 4
        for (int s = s0; s < r; s += step)
            Wh[(size_t)s * dv + c] = __float2half_rn(s < k ? Wu[(size_t)s * (dv + 1) + c] / sg : 0.f);
    }
    if (blockIdx.y == 0)
        for (int s = q * kPrepWarps * 32 + (int)threadIdx.x; s < r_pad; s += step * 32)
            wn[(size_t)u * r_pad + s] = s < k ? Wu[(size_t)s * (dv + 1) + dv] : 0.f;
}

wc_status launch_weights_prep(const Shape& s, const float* W, const int32_t* rank, __half* W16, float* sigma,
                              float* wn, int* status, cudaStream_t st) {
    weights_prep_kernel<<<dim3(s.units * kPrepCluster, (s.dv + 31) / 32), kPrepWarps * 32, 0, st>>>(
        W, rank, sigma, W16, wn, s.r, s.r_pad, s.dv, s.bins > 1, status);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D row-major view [rows][cols] of 2-byte elements, box = 64 columns x box_rows.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
              uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int DV, int MODE>
wc_status launch_tc_t(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& C, const TcArgs& a,
                      dim3 grid, cudaStream_t st) {
    using L = Smem<D, DV>;
    auto kern = expmm_tc_kernel<D, DV, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) != cudaSuccess)
        return WC_ERR_CUDA;
    // the register split needs the block launched with kRegsLaunch registers a thread
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return WC_ERR_CUDA;
    if (fa.numRegs < kRegsLaunch) return WC_ERR_UNSUPPORTED;
    kern<<<grid, kThreads, L::kAlloc, st>>>(A, B, C, a);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

template <int D, int DV, int MODE>
wc_status launch_pair_t(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& C, const TcArgs& a,
                        dim3 grid, cudaStream_t st) {
    using L = SmemPair<D, DV>;
    auto kern = expmm_pair_kernel<D, DV, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) != cudaSuccess)
        return WC_ERR_CUDA;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return WC_ERR_CUDA;
    if (fa.numRegs < kRegsLaunch) return WC_ERR_UNSUPPORTED;
    kern<<<grid, kThreads, L::kAlloc, st>>>(A, B, C, a);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

// Paired row tiles (two 128-row tiles of A per CTA): grid.x counts pairs.
template <int MODE>
wc_status launch_pair(int d, int dv, const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& C,
                      const TcArgs& a, dim3 grid, cudaStream_t st) {
    if (d == 64 && dv == 64) return launch_pair_t<64, 64, MODE>(A, B, C, a, grid, st);
    if (d == 64 && dv == 128) return launch_pair_t<64, 128, MODE>(A, B, C, a, grid, st);
    if (d == 128 && dv == 64) return launch_pair_t<128, 64, MODE>(A, B, C, a, grid, st);
    if (d == 128 && dv == 128) return launch_pair_t<128, 128, MODE>(A, B, C, a, grid, st);
    return WC_ERR_UNSUPPORTED;
}

template <int MODE>
wc_status launch_tc(int d, int dv, const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& C,
                    const TcArgs& a, dim3 grid, cudaStream_t st) {
    if (d == 64 && dv == 64) return launch_tc_t<64, 64, MODE>(A, B, C, a, grid, st);
    if (d == 64 && dv == 128) return launch_tc_t<64, 128, MODE>(A, B, C, a, grid, st);
    if (d == 128 && dv == 64) return launch_tc_t<128, 64, MODE>(A, B, C, a, grid, st);
    if (d == 128 && dv == 128) return launch_tc_t<128, 128, MODE>(A, B, C, a, grid, st);
    return WC_ERR_UNSUPPORTED;
}

}  // namespace

wc_status launch_exp2_selftest(const float* x, float* y, int64_t n, int method, cudaStream_t st) {
    const int64_t pairs = (n + 1) / 2;
    const int blocks = (int)(pairs < 256 * 1184 ? (pairs + 255) / 256 : 1184);
    exp2_selftest_kernel<<<blocks, 256, 0, st>>>(x, y, n, method);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

// the paired kernel's attention rule (see kPairTiles)
bool use_pair_tiles(const Shape& s) { return kPairTiles && s.r <= 2 * BN && s.nq > BM; }

int attend_splits(const Shape& s) {
    // the attention's query tiles alone fill the GPU: no split
    if (s.dtype != WC_BF16 || !((s.d == 64 || s.d == 128) && (s.dv == 64 || s.dv == 128))) return 1;
    const long base = (long)((s.nq + BM - 1) / BM) * s.batch * s.hq;
    const int tiles = (s.r + BN - 1) / BN;
    if (base == 0 || tiles < 2) return 1;
    // as many splits as keep every block in one wave (one block per SM): a
    // second wave would cost a whole block's fixed prologue and epilogue again
    int want = (int)(kAttendFill / base);
    if (want < 2) return 1;
    if (want > tiles) want = tiles;
    const int per = (tiles + want - 1) / want;               // key tiles per split
    return (tiles + per - 1) / per;
}

size_t attend_split_floats(const Shape& s) {
    const int ns = attend_splits(s);
    return ns > 1 ? (size_t)s.batch * s.hq * ns * s.nq * c1_row(s.dv) : 0;
}

bool tc_supported(const Shape& s) {
    return s.dtype == WC_BF16 && (s.d == 64 || s.d == 128) && (s.dv == 64 || s.dv == 128) && encode_fn() != nullptr;
}

wc_status launch_coreset_values_tc(const Shape& s, const void* Ks, const void* K, const void* V,
                                   const int32_t* rank, char* ws, cudaStream_t st) {
    const WsLayout Lw = make_layout(s);
    __half* V16 = reinterpret_cast<__half*>(ws + Lw.v16);
    const size_t nv = (size_t)s.units * s.n * s.dv;
    to_half_kernel<<<1184, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(V), V16, nv);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
    CUtensorMap mA, mB, mC;
    if (!make_map(&mA, Ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.units * s.r, BM) ||
        !make_map(&mB, K, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.units * s.n, BN) ||
        !make_map(&mC, V16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s.dv, (uint64_t)s.units * s.n, BN))
        return WC_ERR_CUDA;
    TcArgs a{};
    a.rank = rank;
    a.out = ws + Lw.c1part;
    a.status = reinterpret_cast<int*>(ws + Lw.status);
    a.a_rows = s.r;
    a.a_head_rows = s.r;
    a.b_rows = s.n;
    a.nsplit = s.nsplit;
    a.split_len = split_keys(s.n, s.units, s.r);
    a.r = s.r;
    a.r_pad = s.r_pad;
    a.hq = s.hkv;
    a.group = 1;
    a.cb = (float)(s.beta * 1.4426950408889634);
    dim3 grid((s.r + TILES * BM - 1) / (TILES * BM), s.nsplit, s.units);
    if (s.center) {
        a.bias = reinterpret_cast<const float*>(ws + Lw.bias);
        a.bias_stride = center_bias_stride(s);
        return launch_tc<kModeBias>(s.d, s.dv, mA, mB, mC, a, grid, st);
    }
    return launch_tc<kExpmmPartial>(s.d, s.dv, mA, mB, mC, a, grid, st);
}

wc_status launch_attend_tc(const Shape& s, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                           float* out, char* ws, cudaStream_t st) {
    const WsLayout Lw = make_layout(s);
    __half* W16 = reinterpret_cast<__half*>(ws + Lw.w16);
    float* sigma = reinterpret_cast<float*>(ws + Lw.sigma);
    float* wn = reinterpret_cast<float*>(ws + Lw.wn);
    if (launch_weights_prep(s, W, rank, W16, sigma, wn, reinterpret_cast<int*>(ws + Lw.status), st) != WC_OK)
        return WC_ERR_CUDA;
    CUtensorMap mA, mB, mC;
    if (!make_map(&mA, Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.batch * s.hq * s.nq, BM) ||
        !make_map(&mB, Ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.units * s.r, BN) ||
        !make_map(&mC, W16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s.dv, (uint64_t)s.units * s.r, BN))
        return WC_ERR_CUDA;
    TcArgs a{};
    a.rank = rank;
    a.out = out;
    a.wn = wn;
    a.sigma = sigma;
    a.status = reinterpret_cast<int*>(ws + Lw.status);
    a.a_rows = s.nq;
    a.a_head_rows = s.nq;
    a.b_rows = s.r;
    a.nsplit = 1;
    a.split_len = s.r;
    a.r = s.r;
    a.r_pad = s.r_pad;
    a.hq = s.hq;
    a.group = s.hq / s.hkv;
    a.all_keys = s.bins > 1;
    a.cb = (float)(s.beta * 1.4426950408889634);
    const int ns = attend_splits(s);
    if (ns <= 1) {
        if (use_pair_tiles(s)) {
            dim3 pgrid((s.nq + 2 * BM - 1) / (2 * BM), 1, s.batch * s.hq);
            return launch_pair<kExpmmRownorm>(s.d, s.dv, mA, mB, mC, a, pgrid, st);
        }
        dim3 grid((s.nq + TILES * BM - 1) / (TILES * BM), 1, s.batch * s.hq);
        return launch_tc<kExpmmRownorm>(s.d, s.dv, mA, mB, mC, a, grid, st);
    }
    // few query tiles: split the coreset over blockIdx.y, then combine the partial rows
    const int tiles = (s.r + BN - 1) / BN;
    float* part = reinterpret_cast<float*>(ws + Lw.apart);
    a.out = part;
    a.nsplit = ns;
    a.split_len = (tiles + ns - 1) / ns * BN;
    dim3 grid((s.nq + TILES * BM - 1) / (TILES * BM), ns, s.batch * s.hq);
    wc_status e = launch_tc<kModeAttnSplit>(s.d, s.dv, mA, mB, mC, a, grid, st);
    if (e != WC_OK) return e;
    const int rows = s.batch * s.hq * s.nq;
    const int blocks = (rows * 32 + 255) / 256;
    if (s.dv == 64)
        attend_combine_kernel<64><<<blocks, 256, 0, st>>>(part, out, s.nq, ns, rows);
    else
        attend_combine_kernel<128><<<blocks, 256, 0, st>>>(part, out, s.nq, ns, rows);
    return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

// Attention on the tensor cores with caller-chosen scratch pointers (status
// word, fp16 weights, column scales, normaliser column); used by the entry
// point that allocates nothing.
wc_status launch_attend_tc_at(const Shape& s, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                              float* out, int* status, __half* W16, float* sigma, float* wn, cudaStream_t st) {
    if (launch_weights_prep(s, W, rank, W16, sigma, wn, status, st) != WC_OK) return WC_ERR_CUDA;
    CUtensorMap mA, mB, mC;
    if (!make_map(&mA, Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.batch * s.hq * s.nq, BM) ||
        !make_map(&mB, Ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.d, (uint64_t)s.units * s.r, BN) ||
        !make_map(&mC, W16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s.dv, (uint64_t)s.units * s.r, BN))
        return WC_ERR_CUDA;
    TcArgs a{};
    a.rank = rank;
    a.out = out;
    a.wn = wn;
    a.sigma = sigma;
    a.status = status;
    a.a_rows = s.nq;
    a.a_head_rows = s.nq;
    a.b_rows = s.r;
    a.nsplit = 1;
    a.split_len = s.r;
    a.r = s.r;
    a.r_pad = s.r_pad;
    a.hq = s.hq;
    a.group = s.hq / s.hkv;
    a.all_keys = s.bins > 1;
    a.cb = (float)(s.beta * 1.4426950408889634);
    if (use_pair_tiles(s)) {
        dim3 pgrid((s.nq + 2 * BM - 1) / (2 * BM), 1, s.batch * s.hq);
        return launch_pair<kExpmmRownorm>(s.d, s.dv, mA, mB, mC, a, pgrid, st);
    }
    dim3 grid((s.nq + TILES * BM - 1) / (TILES * BM), 1, s.batch * s.hq);
    return launch_tc<kExpmmRownorm>(s.d, s.dv, mA, mB, mC, a, grid, st);
}

}  // namespace wc

/*
 * wildcat.h — C ABI of the B200 (sm_100a) WildCat coreset-attention library.
 *
 * WildCat approximates softmax attention by attending over a small weighted
 * coreset of the keys:
 *   1. select   randomly pivoted Cholesky (RPCholesky) on the exponential
 *               kernel H = exp(beta K K^T) picks r pivot keys S and the
 *               partial Cholesky factor F (n x r, F F^T ~ H).
 *               [WildCat: Near-Linear Attention in Theory and Practice,
 *                gist.science technical summary, "Methodik" item 1]
 *   2. weights  Nystrom weights on [V | 1]:
 *               W = h(K_S,K_S)^+ h(K_S,K) [V | 1]     (r x (dv+1))
 *               [same page, "Methodik" item 2: W = h(K_S,K_S)^+ h(K_S,K),
 *                compressed values V_S = W V; the extra column carries the
 *                softmax normaliser]
 *   3. attend   out = rownorm(exp(beta Q K_S^T) W): the last column of the
 *               product divides the others.
 *               [same title, gptget.net page, Abstract: attend over only a
 *                small weighted coreset]
 * h(x, y) = exp(beta <x, y>), beta = 1/sqrt(d) unless `scale` says otherwise.
 *
 * Conventions shared by every call
 *   - Pointers are DEVICE pointers owned by the caller; the library allocates
 *     no device memory.  Scratch lives in the caller's workspace `ws` of at
 *     least wc_workspace_bytes(shape) bytes, 256-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on it; argument errors are returned before any
 *     launch, launch errors as WC_ERR_CUDA.  Errors that a kernel meets on
 *     the device (a wait that ran out, a non-finite factor, and in the
 *     bounds-checked build libwildcat_debug.so an index outside its buffer)
 *     are recorded in the workspace and reported by wc_check_device_status.
 *   - No call allocates or synchronises (wc_check_device_status aside), so
 *     select, weights, attend and forward can be captured into a CUDA graph.
 *   - Tensors are dense, row-major, 16-byte aligned:
 *       Q   [B, Hq,  n_q, d]    dtype
 *       K   [B, Hkv, n_k, d]    dtype
 *       V   [B, Hkv, n_k, dv]   dtype
 *       piv [B, Hkv, r]         int32, pivot key indices in draw order;
 *                               entries >= rank are -1
 *       rank[B, Hkv]            int32, pivots accepted (<= r)
 *       F   [B, Hkv, r, ldf]    fp32, ldf = wc_f_ld(n_k); F[.., c, i] is the
 *                               factor entry of key i in column c of the
 *                               shifted kernel exp(beta K K^T - M_u), M_u =
 *                               max_i beta |k_i|^2 (see select); columns
 *                               >= rank and entries i >= n_k are zero
 *       Ks  [B, Hkv, r, d]      dtype, the pivot keys K[piv]; rows >= rank zero
 *       W   [B, Hkv, r, dv+1]   fp32; rows >= rank zero
 *       out [B, Hq,  n_q, dv]   fp32
 *     Query head g reads kv head g / (Hq / Hkv) (grouped-query attention).
 *   - Results are deterministic for a given shape, seed and GPU.
 *
 * Bins (shape.bins = B > 1)
 *   [same gist.science page, "Methodik" item 1, "Effizienz": the input is split
 *    into B bins processed in parallel, selection time O(n r^2 / B^3 + n r d / B^2)]
 *   Each unit's keys split into B contiguous bins of n_k / B keys; each bin
 *   selects r / B pivots on its own keys and solves its own weights (Philox
 *   unit index (b * Hkv + h) * B + bin), and attention runs over the union of
 *   the bins' coresets.  Layouts change as follows:
 *       piv [B, Hkv, r]         key indices within the unit; bin b's pivots at
 *                               positions b r/B .. (b+1) r/B - 1, -1 beyond its rank
 *       rank[B, Hkv, bins]      pivots accepted per bin
 *       F   [B, Hkv, bins, r/B, wc_f_ld(n_k / B)]   each bin's factor over its keys
 *       Ks, W                   as above (r rows per unit); rows of bin b beyond its
 *                               rank hold a copy of the bin's first pivot key in Ks
 *                               and zeros in W, so attention over all r rows equals
 *                               attention over the accepted pivots
 *
 * Centring (shape.center = 1)
 *   [same page, "Methodik" item 3: softmax attention is invariant to a global
 *    centring of the keys, K <- K - mean(K)]
 *   The selection and the weights use the centred keys of each unit; Ks holds
 *   the keys as given (K[piv]), and attention with them equals attention with
 *   the centred keys (the shift multiplies a query's row by one factor).
 */
#ifndef WILDCAT_H
#define WILDCAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WC_OK = 0,
    WC_ERR_INVALID = 1,      /* bad shape, null or misaligned pointer */
    WC_ERR_CUDA = 2,         /* a CUDA runtime call or launch failed */
    WC_ERR_TIMEOUT = 3,      /* a device-side wait ran out (recorded on the device) */
    WC_ERR_UNSUPPORTED = 4,  /* valid but not implemented (e.g. d not in {64, 128} on a path) */
    WC_ERR_WORKSPACE = 5,    /* ws_bytes < wc_workspace_bytes(shape) */
    WC_ERR_NUMERIC = 6,      /* non-finite value met on the device */
    WC_ERR_BOUNDS = 7        /* an index outside its buffer (pivot, rank), recorded by the
                                bounds-checked debug build (libwildcat_debug.so), which
                                skips the access instead of faulting */
} wc_status;

typedef enum { WC_F32 = 0, WC_BF16 = 1 } wc_dtype;

typedef struct {
    int32_t batch;    /* B >= 1, B * hq <= 65535 */
    int32_t hq;       /* query heads, a multiple of hkv */
    int32_t hkv;      /* key/value heads >= 1 */
    int32_t n_k;      /* keys per head, 1 <= n_k <= 2^26.  The selection keeps a
                         unit's residual diagonal in the shared memory of blocks
                         that run at the same time, which bounds the keys of one
                         unit (one bin with bins) to what the GPU holds at once:
                         about 3.6 million on a B200 (148 SMs x ~24.8k rows);
                         beyond, wc_select / wc_forward return WC_ERR_UNSUPPORTED
                         before the selection launches */
    int32_t n_q;      /* queries per head >= 0 */
    int32_t d;        /* key/query width, a multiple of 8, 8..256 */
    int32_t dv;       /* value width, a multiple of 8, 8..256 */
    int32_t r;        /* coreset size requested, 1 <= r <= min(n_k, 4096) */
    int32_t dtype;    /* wc_dtype of Q, K, V and Ks */
    float scale;      /* beta; 0 selects 1/sqrt(d) */
    float eps_stop;   /* stop rule: selection ends when the drawn pivot's residual
                         is <= eps_stop * max_i H_ii; 0 selects 2^-20 */
    uint32_t wait_timeout_ms;  /* bound on every device-side wait; 0 selects 10000 */
    uint64_t seed;    /* Philox4x32-10 key of the pivot draws */
    int32_t bins;     /* 0 or 1: one selection over each unit's n_k keys.  B > 1: the
                         divide-and-conquer selection; see "Bins" above.  n_k and r
                         must be multiples of B */
    int32_t center;   /* 0: keys as given.  1: each unit's mean key is subtracted
                         before the selection and the weights; see "Centring" above */
    int32_t unit_base; /* >= 0: the Philox unit index of this call's first (batch, kv head)
                          unit, i.e. the index of its first unit in a larger problem whose
                          units are split across calls (one call per GPU); 0 for a whole
                          problem.  Unit u of the call draws its pivots with Philox unit
                          index unit_base + u (times bins, plus the bin, with bins), so each
                          unit gets the pivots it gets in one call over the whole problem */
} wc_shape;

/* Row stride (elements) of F for n_k keys: n_k rounded up to a multiple of 64. */
int64_t wc_f_ld(int32_t n_k);

/* Workspace bytes that select, weights, attend and forward need for `shape`
 * when every output pointer is given (0 if the shape is invalid). */
size_t wc_workspace_bytes(const wc_shape* shape);

/* Workspace bytes for wc_forward when some of piv, rank, F, Ks, W are NULL:
 * the scratch above plus room for all five (0 if the shape is invalid). */
size_t wc_forward_workspace_bytes(const wc_shape* shape);

/*
 * select — RPCholesky [Methodik item 1].  For each (b, kv head) unit u = b*Hkv+h,
 * on the kernel shifted in the log domain, H = exp(beta K K^T - M_u) with
 * M_u = max_i beta |k_i|^2: every entry is then at most 1 (the factor cannot
 * overflow), and the pivots, the stop rule and the weights are those of the
 * unshifted kernel; F is the unshifted kernel's factor times exp(-M_u / 2).
 *   d_i = H_ii = exp(beta |k_i|^2 - M_u);   for j = 0 .. r-1:
 *     u_j = Philox4x32-10(ctr = (j, unit_base + u, 0, 0), key = seed).x0 * 2^-32
 *     s_j = smallest i with d_0 + ... + d_i > u_j * sum(d)  (inverse CDF)
 *     stop (rank = j) if sum(d) <= 0 or d_{s_j} <= eps_stop * max_i H_ii
 *     F[:, j] = (H[:, s_j] - F[:, :j] F[s_j, :j]^T) / sqrt(d_{s_j}),
 *               with the entries at earlier pivots set to zero
 *     d_i = max(d_i - F[i, j]^2, 0);  d_{s_j} = 0
 * Writes piv, F and rank.
 */
wc_status wc_select(const wc_shape* shape, const void* K, int32_t* piv, float* F,
                    int32_t* rank, void* ws, size_t ws_bytes, void* stream);

/*
 * weights — Nystrom weights [Methodik item 2] from select's outputs:
 *   Ks = K[piv];  C1 = exp(beta Ks K^T) [V | 1];  L = F[piv, :rank] (lower
 *   triangular, L L^T = h(K_S, K_S));  W = L^-T (L^-1 C1).
 * Writes Ks and W.
 */
wc_status wc_weights(const wc_shape* shape, const void* K, const void* V, const int32_t* piv,
                     const float* F, const int32_t* rank, void* Ks, float* W,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * attend — coreset attention [Abstract]: A = exp(beta Q Ks^T) W over the
 * first rank[u] coreset rows;  out[q, c] = A[q, c] / A[q, dv].
 */
wc_status wc_attend(const wc_shape* shape, const void* Q, const void* Ks, const float* W,
                    const int32_t* rank, float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * forward — select, weights and attend back to back on `stream` with no host
 * synchronisation.  piv, rank, F, Ks and W may be NULL, in which case they
 * live in the workspace, which must then hold wc_forward_workspace_bytes.
 */
wc_status wc_forward(const wc_shape* shape, const void* Q, const void* K, const void* V,
                     float* out, int32_t* piv, int32_t* rank, float* F, void* Ks, float* W,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, returns the first error a kernel recorded in `ws`
 * since the last check (WC_OK if none) and clears the record.
 */
wc_status wc_check_device_status(void* ws, void* stream);

/*
 * Exercises the bounded device-side wait that select uses between the
 * thread blocks of one unit: two blocks meet at a barrier that one of them
 * never reaches, so the other gives up after timeout_ms and records
 * WC_ERR_TIMEOUT in `ws` (read it with wc_check_device_status).  No fault,
 * no trap; the context stays usable.  ws needs 4096 bytes.
 */
wc_status wc_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t timeout_ms, void* stream);

/*
 * Evaluates over x[0 .. n) (device memory, fp32) the two ways the tensor-core
 * attention and weights kernels compute 2^x, writing y[0 .. n):
 *   method 0  a polynomial on the FMA / ALU pipes: x = n + f with n = rint(x)
 *             and f in [-1/2, 1/2] (additive range reduction after Cody and
 *             Waite), 2^f by a degree-3 relative-minimax (Remez) polynomial,
 *             2^n added to the exponent; relative error <= 2^-13.5 for
 *             -125 <= x <= 127, about 2^-125 returned below -125
 *   method 1  the exponential unit (ex2.approx.ftz.f32)
 * The kernels can run part of every row's exponentials with method 0 to
 * relieve the exponential unit (a build option, off by default: on the
 * measured workloads it was no faster).  For tests; asynchronous on `stream`;
 * WC_ERR_INVALID for n < 0, a null or misaligned pointer or another method.
 */
wc_status wc_selftest_exp2(const float* x, float* y, int64_t n, int32_t method, void* stream);

/*
 * Reads buf[0 .. bytes) (device memory, 16-byte aligned, bytes a positive
 * multiple of 16) once as a plain read-only stream and writes the XOR of its
 * 32-bit words to *sink (device memory, 4-byte aligned).  A measurement aid,
 * no step of the method: the read bandwidth it reaches (bytes / its time) is
 * the denominator to set beside the copy bandwidth for a kernel that, like
 * the select, reads far more than it writes.  Asynchronous on `stream`;
 * WC_ERR_INVALID for a null or misaligned pointer or a bad size.
 */
wc_status wc_read_bandwidth_probe(const void* buf, int64_t bytes, uint32_t* sink, void* stream);

/*
 * attend_noalloc — the same result as wc_attend, for callers that cannot
 * allocate device memory or pass a workspace (an allocator that must not be
 * re-entered, a process whose memory budget is fixed up front, a plugin that
 * only receives its tensors).  The paper has no counterpart; this is a
 * deployment variant of the attend step.
 *   - Scratch: a fixed 16 MiB array in device memory owned by the library
 *     (every GPU that loads the library holds it until the process exits).
 *     bf16 inputs with d, dv in {64, 128} use it; other shapes run on the
 *     CUDA-core kernel, which needs no scratch.  With units = batch * hkv and
 *     up(x) = x rounded up to a multiple of 256, a shape needs
 *         256 + up(2 * units * r * dv) + up(4 * units * dv)
 *             + up(4 * units * (r rounded up to 128))        bytes,
 *     and shapes that need more than 16 MiB (16777216 bytes) are refused with
 *     WC_ERR_WORKSPACE before any launch.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept per device number, for
 *     the device's primary context (the one the CUDA runtime uses); callers
 *     that make their own driver-API contexts current are not served.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 *   - Every call shares the one array and leaves its contents behind; the
 *     call clears what it needs cleared.  Calls whose execution overlaps on
 *     the GPU (other streams, other threads) race on it: serialise them.
 *   - The kernels record device-side errors (a wait that ran out, and in the
 *     bounds-checked build an index outside its buffer) in a status word at
 *     the start of the array, which each call clears first; they need it to
 *     wind down cleanly, and no call reports it (use wc_attend with a
 *     workspace and wc_check_device_status to read such errors).
 */
wc_status wc_attend_noalloc(const wc_shape* shape, const void* Q, const void* Ks, const float* W,
                            const int32_t* rank, float* out, void* stream);

/* Static text for a status code. */
const char* wc_status_string(wc_status status);

#ifdef __cplusplus
}
#endif
#endif

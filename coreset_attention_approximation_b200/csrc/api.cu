// api.cu — the C ABI (include/wildcat.h): argument checks, workspace layout,
// and the launch sequences of select, weights, attend and forward.
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <string.h>

#include "wc_common.cuh"
#include "wc_expmm.cuh"
#include "wc_internal.h"

namespace wc {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Row stride of F (and of the transposed keys): n rounded up to 64 elements, so
// every row of F starts on a 256-byte boundary.
static int64_t f_ld(int32_t n) { return ((int64_t)n + 63) / 64 * 64; }

wc_status make_shape(const wc_shape* in, Shape* o) {
    if (!in) return WC_ERR_INVALID;
    const wc_shape& s = *in;
    if (s.batch < 1 || s.hkv < 1 || s.hq < 1 || s.hq % s.hkv != 0) return WC_ERR_INVALID;
    if (s.n_k < 1 || s.n_k > (1 << 26) || s.n_q < 0) return WC_ERR_INVALID;
    if (s.d < 8 || s.d > 256 || s.d % 8 || s.dv < 8 || s.dv > 256 || s.dv % 8) return WC_ERR_INVALID;
    if (s.r < 1 || s.r > s.n_k || s.r > 4096) return WC_ERR_INVALID;
    if (s.dtype != WC_F32 && s.dtype != WC_BF16) return WC_ERR_INVALID;
    if (!(s.scale >= 0.f) || !isfinite(s.scale) || !(s.eps_stop >= 0.f) || !isfinite(s.eps_stop))
        return WC_ERR_INVALID;
    if ((long long)s.batch * s.hq > 65535) return WC_ERR_INVALID;  // grid z of the attend launch
    o->batch = s.batch; o->hq = s.hq; o->hkv = s.hkv;
    o->n = s.n_k; o->nq = s.n_q; o->d = s.d; o->dv = s.dv; o->r = s.r;
    o->dtype = s.dtype;
    o->beta = s.scale > 0.f ? (double)s.scale : 1.0 / sqrt((double)s.d);
    o->eps = s.eps_stop > 0.f ? (double)s.eps_stop : 0x1p-20;
    o->seed = s.seed;
    o->timeout_ns = (uint64_t)(s.wait_timeout_ms ? s.wait_timeout_ms : 10000u) * 1000000ull;
    o->ldf = f_ld(s.n_k);
    o->units = s.batch * s.hkv;
    o->esize = s.dtype == WC_BF16 ? 2 : 4;
    o->nsplit = (s.n_k + split_keys(s.n_k, o->units, s.r) - 1) / split_keys(s.n_k, o->units, s.r);
    o->r_pad = (s.r + 127) / 128 * 128;
    if (s.bins < 0 || (s.center != 0 && s.center != 1)) return WC_ERR_INVALID;
    o->bins = s.bins > 1 ? s.bins : 1;
    if (s.n_k % o->bins || s.r % o->bins) return WC_ERR_INVALID;
    o->center = s.center;
    if (s.unit_base < 0 || ((int64_t)s.unit_base + o->units) * o->bins > (int64_t)UINT32_MAX) return WC_ERR_INVALID;
    o->unit_base = s.unit_base;
    o->units_all = o->units;
    o->n_all = s.n_k;
    o->r_all = s.r;
    return WC_OK;
}

Shape bin_view(const Shape& s) {
    Shape b = s;
    if (s.bins <= 1) return b;
    b.hkv = s.hkv * s.bins;
    b.hq = s.hq * s.bins;
    b.units = s.units_all * s.bins;
    b.n = s.n_all / s.bins;
    b.r = s.r_all / s.bins;
    b.ldf = f_ld(b.n);
    b.nsplit = (b.n + split_keys(b.n, b.units, b.r) - 1) / split_keys(b.n, b.units, b.r);
    b.r_pad = (b.r + 127) / 128 * 128;
    return b;
}

WsLayout make_layout(const Shape& s) {
    // Every region is sized from the caller's problem (units_all, n_all, r_all,
    // bins) for the larger of its unit-view and bin-view needs, so the select,
    // weights and attend launchers agree on the offsets whichever view they get.
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, kWsAlign);
        return at;
    };
    const size_t U = (size_t)s.units_all, B = (size_t)s.bins;
    const size_t n = (size_t)s.n_all, r = (size_t)s.r_all, nb = n / B, rb = r / B;
    const size_t ldb = (size_t)f_ld((int32_t)nb);
    const int skb = split_keys((int)nb, (int)(U * B), (int)rb);
    const size_t nsb = (nb + skb - 1) / skb;
    const size_t r_pad = (r + 127) / 128 * 128;
    const size_t kt_unit = U * s.d * (size_t)f_ld((int32_t)n), kt_bin = U * B * s.d * ldb;
    L.status = take(256);
    L.sync = take(sizeof(UnitSync) * U * B);
    L.partials = take(sizeof(double) * U * B * 2 * kMaxBlocksPerUnit);
    // transposed keys for the selection: fp32 when centred (centred values are not bf16)
    L.kt = take((size_t)(s.center ? 4 : s.esize) * (kt_unit > kt_bin ? kt_unit : kt_bin));
    L.lg = take(sizeof(float) * U * B * rb * rb);
    L.c1part = take(sizeof(float) * U * B * nsb * rb * c1_row(s.dv));
    L.y = take(sizeof(double) * U * r * (s.dv + 1));
    const bool tc = s.dtype == WC_BF16;
    L.v16 = take(tc ? 2 * U * n * s.dv : 0);
    L.w16 = take(tc ? 2 * U * r * s.dv : 0);
    L.sigma = take(tc ? sizeof(float) * U * s.dv : 0);
    L.wn = take(tc ? sizeof(float) * U * r_pad : 0);
    const size_t C = s.center ? 1 : 0;
    L.kpart = take(C * sizeof(double) * U * ((n + kCenterChunk - 1) / kCenterChunk) * s.d);
    L.kbar = take(C * sizeof(double) * U * s.d);
    L.kk = take(C * sizeof(double) * U);
    L.cdot = take(C * sizeof(double) * U * n);
    L.bias = take(C * sizeof(float) * U * B * ((nb + 127) / 128 * 128));
    L.shift = take(sizeof(double) * U * B);
    L.apart = take(sizeof(float) * attend_split_floats(s));
    L.scratch_end = off;
    L.piv = take(sizeof(int32_t) * U * r);
    L.rank = take(sizeof(int32_t) * U * B);
    L.f = take(sizeof(float) * U * B * rb * ldb);
    L.ks = take((size_t)s.esize * U * r * s.d);
    L.w = take(sizeof(float) * U * r * (s.dv + 1));
    L.forward_end = off;
    return L;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static wc_status check_ws(const Shape& s, void* ws, size_t ws_bytes, bool forward_room) {
    if (!ws || ((uintptr_t)ws & (kWsAlign - 1))) return WC_ERR_INVALID;
    const WsLayout L = make_layout(s);
    if (ws_bytes < (forward_room ? L.forward_end : L.scratch_end)) return WC_ERR_WORKSPACE;
    return WC_OK;
}

}  // namespace wc

using namespace wc;

namespace {
// An NVTX range around each entry point, for profilers (no cost without one).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

extern "C" {

int64_t wc_f_ld(int32_t n_k) { return n_k < 1 ? 0 : f_ld(n_k); }

size_t wc_workspace_bytes(const wc_shape* shape) {
    Shape s;
    if (make_shape(shape, &s) != WC_OK) return 0;
    return make_layout(s).scratch_end;
}

size_t wc_forward_workspace_bytes(const wc_shape* shape) {
    Shape s;
    if (make_shape(shape, &s) != WC_OK) return 0;
    return make_layout(s).forward_end;
}

wc_status wc_select(const wc_shape* shape, const void* K, int32_t* piv, float* F, int32_t* rank, void* ws,
                    size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("wc_select");
    Shape s;
    wc_status e = make_shape(shape, &s);
    if (e != WC_OK) return e;
    if (!K || !piv || !F || !rank || !aligned16(K) || !aligned16(F) || !aligned16(piv)) return WC_ERR_INVALID;
    if ((e = check_ws(s, ws, ws_bytes, false)) != WC_OK) return e;
    char* w = static_cast<char*>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (s.center && (e = launch_center(s, K, w, st)) != WC_OK) return e;
    return launch_select(bin_view(s), K, piv, F, rank, w, st);
}

wc_status wc_weights(const wc_shape* shape, const void* K, const void* V, const int32_t* piv, const float* F,
                     const int32_t* rank, void* Ks, float* W, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("wc_weights");
    Shape s;
    wc_status e = make_shape(shape, &s);
    if (e != WC_OK) return e;
    if (!K || !V || !piv || !F || !rank || !Ks || !W) return WC_ERR_INVALID;
    if (!aligned16(K) || !aligned16(V) || !aligned16(F) || !aligned16(Ks) || !aligned16(W)) return WC_ERR_INVALID;
    if ((e = check_ws(s, ws, ws_bytes, false)) != WC_OK) return e;
    char* w = static_cast<char*>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape sb = bin_view(s);
    if (s.center && (e = launch_center(s, K, w, st)) != WC_OK) return e;
    if ((e = launch_key_shift(s, K, w, st)) != WC_OK) return e;
    if ((e = launch_gather(sb, K, piv, F, rank, Ks, w, st)) != WC_OK) return e;
    if ((e = launch_coreset_values(sb, Ks, K, V, rank, w, st)) != WC_OK) return e;
    return launch_solve(sb, piv, rank, W, w, st);
}

wc_status wc_attend(const wc_shape* shape, const void* Q, const void* Ks, const float* W, const int32_t* rank,
                    float* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("wc_attend");
    Shape s;
    wc_status e = make_shape(shape, &s);
    if (e != WC_OK) return e;
    if (s.nq == 0) return WC_OK;
    if (!Q || !Ks || !W || !rank || !out) return WC_ERR_INVALID;
    if (!aligned16(Q) || !aligned16(Ks) || !aligned16(W) || !aligned16(out)) return WC_ERR_INVALID;
    if ((e = check_ws(s, ws, ws_bytes, false)) != WC_OK) return e;
    return launch_attend(s, Q, Ks, W, rank, out, static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
}

wc_status wc_forward(const wc_shape* shape, const void* Q, const void* K, const void* V, float* out, int32_t* piv,
                     int32_t* rank, float* F, void* Ks, float* W, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("wc_forward");
    Shape s;
    wc_status e = make_shape(shape, &s);
    if (e != WC_OK) return e;
    if (!K || !V || (s.nq > 0 && (!Q || !out))) return WC_ERR_INVALID;
    const bool room = !piv || !rank || !F || !Ks || !W;
    if ((e = check_ws(s, ws, ws_bytes, room)) != WC_OK) return e;
    const WsLayout L = make_layout(s);
    char* w = static_cast<char*>(ws);
    if (!piv) piv = reinterpret_cast<int32_t*>(w + L.piv);
    if (!rank) rank = reinterpret_cast<int32_t*>(w + L.rank);
    if (!F) F = reinterpret_cast<float*>(w + L.f);
    if (!Ks) Ks = w + L.ks;
    if (!W) W = reinterpret_cast<float*>(w + L.w);
    if ((e = wc_select(shape, K, piv, F, rank, ws, ws_bytes, stream)) != WC_OK) return e;
    if ((e = wc_weights(shape, K, V, piv, F, rank, Ks, W, ws, ws_bytes, stream)) != WC_OK) return e;
    if (s.nq == 0) return WC_OK;
    return wc_attend(shape, Q, Ks, W, rank, out, ws, ws_bytes, stream);
}

wc_status wc_check_device_status(void* ws, void* stream) {
    if (!ws) return WC_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return WC_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return WC_ERR_CUDA;
    if (host != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return WC_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return WC_ERR_CUDA;
    }
    return static_cast<wc_status>(host);
}

wc_status wc_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t timeout_ms, void* stream) {
    if (!ws || ws_bytes < 4096 || ((uintptr_t)ws & (kWsAlign - 1))) return WC_ERR_INVALID;
    if (timeout_ms == 0 || timeout_ms > 60000) return WC_ERR_INVALID;
    return launch_wait_selftest(static_cast<char*>(ws), (uint64_t)timeout_ms * 1000000ull,
                                static_cast<cudaStream_t>(stream));
}

wc_status wc_selftest_exp2(const float* x, float* y, int64_t n, int32_t method, void* stream) {
    if (n < 0 || (method != 0 && method != 1)) return WC_ERR_INVALID;
    if (n == 0) return WC_OK;
    if (!x || !y || ((uintptr_t)x & 3u) || ((uintptr_t)y & 3u)) return WC_ERR_INVALID;
    return launch_exp2_selftest(x, y, n, method, static_cast<cudaStream_t>(stream));
}

wc_status wc_read_bandwidth_probe(const void* buf, int64_t bytes, uint32_t* sink, void* stream) {
    if (!buf || !sink || bytes <= 0 || (bytes & 15) || ((uintptr_t)buf & 15u) || ((uintptr_t)sink & 3u))
        return WC_ERR_INVALID;
    return launch_read_probe(buf, bytes, sink, static_cast<cudaStream_t>(stream));
}

const char* wc_status_string(wc_status status) {
    switch (status) {
        case WC_OK: return "ok";
        case WC_ERR_INVALID: return "invalid argument";
        case WC_ERR_CUDA: return "CUDA error";
        case WC_ERR_TIMEOUT: return "device-side wait timed out";
        case WC_ERR_UNSUPPORTED: return "unsupported shape";
        case WC_ERR_WORKSPACE: return "workspace too small";
        case WC_ERR_NUMERIC: return "non-finite value on the device";
        case WC_ERR_BOUNDS: return "index outside its buffer (debug build)";
    }
    return "unknown status";
}

}  // extern "C"

// gdn_api.cu -- the extern "C" entry points declared in include/gdn.h.
//
// Everything here runs on the host: argument validation (before any launch),
// workspace sizing, and dispatch to the kernels.  Dispatch rule: bf16 with
// dk = dv = 128 and chunk = 64 goes to the tensor-core kernels; every other
// supported shape and GDN_F32 go to the fp32 SIMT kernels.  Both run on the
// GPU; there is no host fallback.
#include <math.h>
#include <algorithm>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

using namespace gdn;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

gdn_status check_dims(const gdn_dims* d) {
    if (!d) return GDN_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 1 || d->H < 1) return GDN_ERR_INVALID_ARG;
    if (d->chunk != 16 && d->chunk != 32 && d->chunk != 64) return GDN_ERR_INVALID_ARG;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (d->gate != GDN_GATE_SCALAR && d->gate != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (!isfinite(d->scale)) return GDN_ERR_INVALID_ARG;
    // element counts must fit the kernels' 32-bit token index arithmetic
    if ((double)d->B * d->T * d->H * 128.0 > 9.0e18) return GDN_ERR_INVALID_ARG;
    if ((long long)d->B * d->H > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(d->dk) || !dim_ok(d->dv)) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

bool all_aligned(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && !aligned16(p)) return false;
    return true;
}

// Packed sequences: one row of T tokens in all (B = 1) split by device
// offsets into nseq sequences; tensor-core shapes only.
gdn_status check_varlen(const gdn_dims* d, int nseq) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (d->B != 1 || nseq < 1) return GDN_ERR_INVALID_ARG;
    if ((long long)nseq * d->H > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
    // chunk slots: ceil(T / 64) + nseq per head must fit an int
    if ((long long)d->H * ((d->T + 63) / 64 + (long long)nseq) > 0x7fffffffLL)
        return GDN_ERR_INVALID_ARG;
    if (!tc_supported(*d)) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

namespace gdn {
gdn_status validate_fwd_args(const gdn_dims* d, const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* h0, const void* o,
                             const float* hT) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, o, hT})) return GDN_ERR_INVALID_ARG;
    if (h0 && hT && h0 == hT) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

ConvLayout conv_layout(const gdn_dims& d, int K, size_t base) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t es = d.dtype == GDN_BF16 ? 2 : 4;
    const size_t tq = al((size_t)d.B * d.T * d.H * d.dk * es), tv = al((size_t)d.B * d.T * d.H * d.dv * es);
    ConvLayout c{};
    size_t o = al(base);
    c.qf = o; o += tq;
    c.kf = o; o += tq;
    c.vf = o; o += tv;
    c.dqf = o; o += tq;
    c.dkf = o; o += tq;
    c.dvf = o; o += tv;
    c.cws = o;
    o += al(std::max(gdn_short_conv_bwd_workspace(d.B, d.T, d.H, d.dk, K),
                     gdn_short_conv_bwd_workspace(d.B, d.T, d.H, d.dv, K)));
    c.end = o;
    return c;
}
}  // namespace gdn

extern "C" {

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT";
    }
    return "GDN_UNKNOWN_STATUS";
}

size_t gdn_chunk_fwd_workspace(const gdn_dims* d) {
    if (check_dims(d) != GDN_OK) return 0;
    return tc_supported(*d) ? tc_fwd_workspace(*d) : simt_fwd_workspace(*d);
}

size_t gdn_chunk_bwd_workspace(const gdn_dims* d) {
    if (check_dims(d) != GDN_OK) return 0;
    return tc_bwd_supported(*d) ? tc_bwd_workspace(*d) : simt_bwd_workspace(*d);
}

gdn_status gdn_chunk_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* h0, void* o,
                         float* hT, void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, o, hT})) return GDN_ERR_INVALID_ARG;
    if (h0 && hT && h0 == hT) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_fwd_workspace(d);
    if (ws_bytes < need || (need && !ws)) return GDN_ERR_WORKSPACE;
    if (ws && ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();  // clear a stale error so it is not reported as ours
    if (ws && cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (tc_supported(*d)) {
        if (!launch_tc_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st)) return GDN_ERR_CUDA;
    } else {
        launch_simt_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st);
    }
    return launch_status();
}

gdn_status gdn_chunk_bwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* h0, const void* dO,
                         const float* dhT, void* dq, void* dk, void* dv, float* dg,
                         float* dbeta, float* dh0, void* ws, size_t ws_bytes,
                         gdn_stream_t stream) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta)
        return GDN_ERR_INVALID_ARG;
    if ((h0 == nullptr) != (dh0 == nullptr)) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0}))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_bwd_workspace(d);
    if (ws_bytes < need || (need && !ws)) return GDN_ERR_WORKSPACE;
    if (ws && ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (ws && cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (tc_bwd_supported(*d)) {
        if (!launch_tc_bwd(*d, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, st))
            return GDN_ERR_CUDA;
    } else
        launch_simt_bwd(*d, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, st);
    return launch_status();
}

gdn_status gdn_chunk_fwd_save(const gdn_dims* d, const void* q, const void* k, const void* v,
                              const float* g, const float* beta, const float* h0, void* o,
                              float* hT, void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, o, hT})) return GDN_ERR_INVALID_ARG;
    if (h0 && hT && h0 == hT) return GDN_ERR_INVALID_ARG;
    const size_t need = std::max(gdn_chunk_bwd_workspace(d), gdn_chunk_fwd_workspace(d));
    if (ws_bytes < need || (need && !ws)) return GDN_ERR_WORKSPACE;
    if (ws && ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (ws && cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (tc_supported(*d)) {
        if (!launch_tc_fwd_save(*d, q, k, v, g, beta, h0, o, hT, ws, st)) return GDN_ERR_CUDA;
    } else {  // the general-shape backward recomputes: nothing to keep
        launch_simt_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st);
    }
    return launch_status();
}

gdn_status gdn_chunk_bwd_saved(const gdn_dims* d, const void* q, const void* k, const void* v,
                               const float* g, const float* beta, const float* h0, const void* dO,
                               const float* dhT, void* dq, void* dk, void* dv, float* dg,
                               float* dbeta, float* dh0, void* ws, size_t ws_bytes,
                               gdn_stream_t stream) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta)
        return GDN_ERR_INVALID_ARG;
    if ((h0 == nullptr) != (dh0 == nullptr)) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0}))
        return GDN_ERR_INVALID_ARG;
    const size_t need = std::max(gdn_chunk_bwd_workspace(d), gdn_chunk_fwd_workspace(d));
    if (ws_bytes < need || (need && !ws)) return GDN_ERR_WORKSPACE;
    if (ws && ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (ws && cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (tc_bwd_supported(*d)) {
        if (!launch_tc_bwd(*d, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, st,
                           nullptr, 0, true))
            return GDN_ERR_CUDA;
    } else
        launch_simt_bwd(*d, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, st);
    return launch_status();
}

static size_t saved_base(const gdn_dims* d) {
    return std::max(gdn_chunk_bwd_workspace(d), gdn_chunk_fwd_workspace(d));
}

size_t gdn_chunk_conv_saved_workspace(const gdn_dims* d, int K) {
    if (check_dims(d) != GDN_OK || K < 1 || K > 4) return 0;
    return conv_layout(*d, K, saved_base(d)).end;
}

gdn_status gdn_chunk_fwd_save_conv(const gdn_dims* d, int K, const void* xq, const void* xk,
                                   const void* xv, const float* wq, const float* wk, const float* wv,
                                   const float* g, const float* beta, const float* h0, void* o,
                                   float* hT, void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_status s = validate_fwd_args(d, xq, xk, xv, g, beta, h0, o, hT);
    if (s != GDN_OK) return s;
    if (K < 1 || K > 4 || !wq || !wk || !wv) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({wq, wk, wv})) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_conv_saved_workspace(d, K);
    if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
    if ((uintptr_t)ws & 255u) return GDN_ERR_WORKSPACE;
    const ConvLayout CL = conv_layout(*d, K, saved_base(d));
    char* base = (char*)ws;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (tc_supported(*d) && d->gate == GDN_GATE_SCALAR) {  // the prologue fused into the preparation
        if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return GDN_ERR_CUDA;
        if (!launch_tc_fwd_save_conv(*d, K, xq, xk, xv, wq, wk, wv, g, beta, h0, o, hT, ws, st))
            return GDN_ERR_CUDA;
        return launch_status();
    }
    // other shapes: the prologue as its own pass, then the saving forward
    const int B = d->B, T = d->T, H = d->H;
    if ((s = gdn_short_conv_fwd(B, T, H, d->dk, K, d->dtype, 1, xq, wq, base + CL.qf, stream)) != GDN_OK ||
        (s = gdn_short_conv_fwd(B, T, H, d->dk, K, d->dtype, 1, xk, wk, base + CL.kf, stream)) != GDN_OK ||
        (s = gdn_short_conv_fwd(B, T, H, d->dv, K, d->dtype, 0, xv, wv, base + CL.vf, stream)) != GDN_OK)
        return s;
    return gdn_chunk_fwd_save(d, base + CL.qf, base + CL.kf, base + CL.vf, g, beta, h0, o, hT, ws,
                              saved_base(d), stream);
}

gdn_status gdn_chunk_bwd_saved_conv(const gdn_dims* d, int K, const void* xq, const void* xk,
                                    const void* xv, const float* wq, const float* wk, const float* wv,
                                    const float* g, const float* beta, const float* h0, const void* dO,
                                    const float* dhT, void* dxq, void* dxk, void* dxv, float* dwq,
                                    float* dwk, float* dwv, float* dg, float* dbeta, float* dh0,
                                    void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_status s = check_dims(d);
    if (s != GDN_OK) return s;
    if (K < 1 || K > 4) return GDN_ERR_INVALID_ARG;
    if (!xq || !xk || !xv || !wq || !wk || !wv || !dxq || !dxk || !dxv || !dwq || !dwk || !dwv)
        return GDN_ERR_INVALID_ARG;
    if (!all_aligned({xq, xk, xv, wq, wk, wv, dxq, dxk, dxv, dwq, dwk, dwv}))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_conv_saved_workspace(d, K);
    if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
    if ((uintptr_t)ws & 255u) return GDN_ERR_WORKSPACE;
    const ConvLayout CL = conv_layout(*d, K, saved_base(d));
    char* base = (char*)ws;
    // the chunk backward for the filtered q, k, v kept by the forward ...
    s = gdn_chunk_bwd_saved(d, base + CL.qf, base + CL.kf, base + CL.vf, g, beta, h0, dO, dhT,
                            base + CL.dqf, base + CL.dkf, base + CL.dvf, dg, dbeta, dh0, ws,
                            saved_base(d), stream);
    if (s != GDN_OK) return s;
    // ... then the prologue's backward from their gradients
    const int B = d->B, T = d->T, H = d->H;
    void* cws = base + CL.cws;
    const size_t cb = CL.end - CL.cws;
    if ((s = gdn_short_conv_bwd(B, T, H, d->dk, K, d->dtype, 1, xq, wq, base + CL.dqf, dxq, dwq, cws, cb,
                                stream)) != GDN_OK ||
        (s = gdn_short_conv_bwd(B, T, H, d->dk, K, d->dtype, 1, xk, wk, base + CL.dkf, dxk, dwk, cws, cb,
                                stream)) != GDN_OK ||
        (s = gdn_short_conv_bwd(B, T, H, d->dv, K, d->dtype, 0, xv, wv, base + CL.dvf, dxv, dwv, cws, cb,
                                stream)) != GDN_OK)
        return s;
    return GDN_OK;
}

gdn_status gdn_recurrent_step(int N, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate,
                              float scale, const void* q, const void* k, const void* v,
                              const float* g, const float* beta, float* state, void* o,
                              gdn_stream_t stream) {
    if (N < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if ((long long)N * H > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (gate != GDN_GATE_SCALAR && gate != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, state, o})) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    cudaGetLastError();
    launch_recurrent_step(N, H, dk, dv, dtype, gate, scale, q, k, v, g, beta, state, o,
                          (cudaStream_t)stream);
    return launch_status();
}

gdn_status gdn_test_stalled_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                                const float* g, const float* beta, const float* h0, void* o,
                                float* hT, void* ws, size_t ws_bytes, int stall_at,
                                unsigned long long wait_ns, gdn_stream_t stream) {
    gdn_status s = validate_fwd_args(d, q, k, v, g, beta, h0, o, hT);
    if (s != GDN_OK) return s;
    if (stall_at < 0 || wait_ns == 0 || wait_ns > 1000000000ull) return GDN_ERR_INVALID_ARG;
    if (!tc_supported(*d) || !tc_fwd_whole_head(*d)) return GDN_ERR_UNSUPPORTED;
    const size_t need = tc_fwd_workspace(*d);
    if (!ws || ws_bytes < need || ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return GDN_ERR_CUDA;
    if (!launch_tc_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st, nullptr, 0, wait_ns, stall_at))
        return GDN_ERR_CUDA;
    return launch_status();
}

gdn_status gdn_query_device_status(void* ws, gdn_stream_t stream) {
    if (!ws) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (word == 0) return GDN_OK;
    const unsigned int zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return GDN_ERR_CUDA;
    return (word & 1u) ? GDN_ERR_DEVICE_TIMEOUT : GDN_ERR_INVALID_ARG;
}

size_t gdn_chunk_fwd_varlen_workspace(const gdn_dims* d, int nseq) {
    if (check_varlen(d, nseq) != GDN_OK) return 0;
    return tc_fwd_workspace(*d, nseq);
}

size_t gdn_chunk_bwd_varlen_workspace(const gdn_dims* d, int nseq) {
    if (check_varlen(d, nseq) != GDN_OK) return 0;
    return tc_bwd_workspace(*d, nseq);
}

gdn_status gdn_chunk_fwd_varlen(const gdn_dims* d, const int* cu_seqlens, int nseq, const void* q,
                                const void* k, const void* v, const float* g, const float* beta,
                                const float* h0, void* o, float* hT, void* ws, size_t ws_bytes,
                                gdn_stream_t stream) {
    gdn_status s = check_varlen(d, nseq);
    if (s != GDN_OK) return s;
    if (!cu_seqlens || ((uintptr_t)cu_seqlens & 3u)) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, o, hT})) return GDN_ERR_INVALID_ARG;
    if (h0 && hT && h0 == hT) return GDN_ERR_INVALID_ARG;
    const size_t need = tc_fwd_workspace(*d, nseq);
    if (!ws || ws_bytes < need || ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return GDN_ERR_CUDA;
    if (!launch_tc_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st, cu_seqlens, nseq))
        return GDN_ERR_CUDA;
    return launch_status();
}

gdn_status gdn_chunk_bwd_varlen(const gdn_dims* d, const int* cu_seqlens, int nseq, const void* q,
                                const void* k, const void* v, const float* g, const float* beta,
                                const float* h0, const void* dO, const float* dhT, void* dq,
                                void* dk, void* dv, float* dg, float* dbeta, float* dh0, void* ws,
                                size_t ws_bytes, gdn_stream_t stream) {
    gdn_status s = check_varlen(d, nseq);
    if (s != GDN_OK) return s;
    if (!cu_seqlens || ((uintptr_t)cu_seqlens & 3u)) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta)
        return GDN_ERR_INVALID_ARG;
    if ((h0 == nullptr) != (dh0 == nullptr)) return GDN_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0}))
        return GDN_ERR_INVALID_ARG;
    const size_t need = tc_bwd_workspace(*d, nseq);
    if (!ws || ws_bytes < need || ((uintptr_t)ws & 255u)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return GDN_ERR_CUDA;
    if (!launch_tc_bwd(*d, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, st,
                       cu_seqlens, nseq))
        return GDN_ERR_CUDA;
    return launch_status();
}

}  // extern "C"
